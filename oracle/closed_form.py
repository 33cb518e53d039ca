"""Brute-force closed-form unrolling of the two recurrences -- TEST INFRASTRUCTURE.

Only for tiny inputs: every state S_t is formed from S_0 and the inputs by
explicit products, with no recursion over t, so it is an independent route to
the same numbers as the eager recurrence (oracle/eager.c).

Mamba-2 (per (b,h); a_j = exp(dt_j A_h), s_i = dt_i if dt scales the input else 1):
    S_t = (prod_{j<=t} a_j) S_0 + sum_{i<=t} (prod_{i<j<=t} a_j) s_i x_i B_i^T
    y_t = S_t C_t + D_h x_t
Gated DeltaNet (per (b,h); M_j = alpha_j (I - beta_j k_j k_j^T) as a dense d_k x d_k matrix):
    S_t = S_0 M_1 ... M_t + sum_{i<=t} beta_i v_i k_i^T M_{i+1} ... M_t
    o_t = S_t q_t
Kimi Delta Attention (M_j = Diag(alpha_j) (I - beta_j k_j k_j^T), alpha_j a gate per key channel):
    the Gated DeltaNet form with that M_j.
These are the unrolled forms of the layer updates the ReplaySSM reports describe
("La fiche qu'on reecrit", blog.thibaultmonteiro.fr): a decay plus a rank-1 write
(Mamba-2), or the same with a delta-rule correction (Gated DeltaNet).
"""
from __future__ import annotations

import numpy as np


def mamba2_one_head(S0, A_h, D_h, x, dt, Bm, Cm, dt_scales_input=False):
    """S0[P,N]; x[T,P]; dt[T]; Bm,Cm[T,N].  Returns (y[T,P], S_T[P,N])."""
    T = x.shape[0]
    a = [np.exp(dt[j] * A_h) for j in range(T)]
    s = [dt[i] if dt_scales_input else 1.0 for i in range(T)]
    ys = []
    S_t = S0
    for t in range(T):
        S_t = float(np.prod(a[: t + 1])) * S0
        for i in range(t + 1):
            S_t = S_t + float(np.prod(a[i + 1: t + 1])) * s[i] * np.outer(x[i], Bm[i])
        ys.append(S_t @ Cm[t] + D_h * x[t])
    return np.array(ys), S_t


def gdn_one_head(S0, q, k, v, alpha, beta):
    """S0[d_v,d_k]; q,k[T,d_k]; v[T,d_v]; alpha,beta[T].  Returns (o[T,d_v], S_T)."""
    T, dk = k.shape
    M = [alpha[j] * (np.eye(dk) - beta[j] * np.outer(k[j], k[j])) for j in range(T)]

    def chain(i0, i1):  # M_{i0} ... M_{i1-1} (0-based, empty product = I)
        out = np.eye(dk)
        for j in range(i0, i1):
            out = out @ M[j]
        return out

    outs = []
    S_t = S0
    for t in range(T):
        S_t = S0 @ chain(0, t + 1)
        for i in range(t + 1):
            S_t = S_t + beta[i] * np.outer(v[i], k[i]) @ chain(i + 1, t + 1)
        outs.append(S_t @ q[t])
    return np.array(outs), S_t


def kda_one_head(S0, q, k, v, alpha, beta):
    """S0[d_v,d_k]; q,k[T,d_k]; v[T,d_v]; alpha[T,d_k]; beta[T].  Returns (o[T,d_v], S_T)."""
    T, dk = k.shape
    M = [np.diag(alpha[j]) @ (np.eye(dk) - beta[j] * np.outer(k[j], k[j])) for j in range(T)]

    def chain(i0, i1):  # M_{i0} ... M_{i1-1} (0-based, empty product = I)
        out = np.eye(dk)
        for j in range(i0, i1):
            out = out @ M[j]
        return out

    outs = []
    S_t = S0
    for t in range(T):
        S_t = S0 @ chain(0, t + 1)
        for i in range(t + 1):
            S_t = S_t + beta[i] * np.outer(v[i], k[i]) @ chain(i + 1, t + 1)
        outs.append(S_t @ q[t])
    return np.array(outs), S_t


def mamba2(S0, A, D, x, dt, Bm, Cm, dt_scales_input=False):
    """All (b,h). S0[B,H,P,N]; x[B,T,H,P]; dt[B,T,H]; Bm,Cm[B,T,G,N]. Returns y[B,T,H,P], S_T."""
    Bn, H, P, N = S0.shape
    G = Bm.shape[2]
    T = x.shape[1]
    y = np.empty((Bn, T, H, P))
    S = np.empty_like(S0)
    for b in range(Bn):
        for h in range(H):
            g = h // (H // G)
            yy, S[b, h] = mamba2_one_head(S0[b, h], A[h], D[h], x[b, :, h], dt[b, :, h],
                                          Bm[b, :, g], Cm[b, :, g], dt_scales_input)
            y[b, :, h] = yy
    return y, S


def gdn(S0, q, k, v, alpha, beta):
    """All (b,h). S0[B,H,d_v,d_k]; q,k[B,T,H,d_k]; v[B,T,H,d_v]; alpha,beta[B,T,H]."""
    Bn, H, P, N = S0.shape
    T = q.shape[1]
    o = np.empty((Bn, T, H, P))
    S = np.empty_like(S0)
    for b in range(Bn):
        for h in range(H):
            oo, S[b, h] = gdn_one_head(S0[b, h], q[b, :, h], k[b, :, h], v[b, :, h],
                                       alpha[b, :, h], beta[b, :, h])
            o[b, :, h] = oo
    return o, S


def kda(S0, q, k, v, alpha, beta):
    """All (b,h). S0[B,H,d_v,d_k]; q,k[B,T,H,d_k]; v[B,T,H,d_v]; alpha[B,T,H,d_k]; beta[B,T,H]."""
    Bn, H, P, N = S0.shape
    T = q.shape[1]
    o = np.empty((Bn, T, H, P))
    S = np.empty_like(S0)
    for b in range(Bn):
        for h in range(H):
            oo, S[b, h] = kda_one_head(S0[b, h], q[b, :, h], k[b, :, h], v[b, :, h],
                                       alpha[b, :, h], beta[b, :, h])
            o[b, :, h] = oo
    return o, S
