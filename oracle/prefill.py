"""Chunked Mamba-2 prefill -- TEST INFRASTRUCTURE.

Only tests/ may import this.  A prompt of T tokens is processed in chunks of Q
tokens: within a chunk the outputs come from the chunk's own inputs through the
decayed pairwise products (C_t . B_s), plus the state at the chunk's start read
with the query; the state is then carried to the next chunk by one decay and a
rank-Q update.  It reaches the eager recurrence's numbers (y_t = S_t C_t + D x_t,
S_t = e^{dt_t A} S_{t-1} + s_t x_t B_t^T) by another route, and its final state is
the checkpoint a decode would start from (rssm_import_state).  The same
checkpoint + inputs algebra as the replay read, with the "buffer" being the chunk
(blog.thibaultmonteiro.fr, "Tenir le journal plutot que le solde").

Per chunk, with Lam_t = sum of dt_j A over the chunk's tokens j <= t:
    y_t = e^{Lam_t} (S_start C_t) + sum_{s <= t} e^{Lam_t - Lam_s} (C_t . B_s) s_s x_s + D x_t
    S_end = e^{Lam_last} S_start + sum_s e^{Lam_last - Lam_s} s_s x_s B_s^T
"""
from __future__ import annotations

import numpy as np


def mamba2_one_head(S0, A_h, D_h, x, dt, Bm, Cm, chunk, dt_scales_input=False):
    """S0 [P, N]; x [T, P]; dt [T]; Bm, Cm [T, N].  Returns (y [T, P], S_T [P, N])."""
    T = x.shape[0]
    S = np.array(S0, dtype=np.float64, copy=True)
    y = np.empty((T, x.shape[1]))
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        lam = np.cumsum(dt[t0:t1] * A_h)                    # [Q]
        s = dt[t0:t1] if dt_scales_input else np.ones(t1 - t0)
        CB = Cm[t0:t1] @ Bm[t0:t1].T                        # [Q, Q]: C_t . B_s
        Ldec = np.exp(lam[:, None] - lam[None, :])          # e^{Lam_t - Lam_s}
        mask = np.tril(np.ones((t1 - t0, t1 - t0)))
        Wts = mask * Ldec * CB * s[None, :]                 # weight of x_s in y_t
        y[t0:t1] = np.exp(lam)[:, None] * (Cm[t0:t1] @ S.T) + Wts @ x[t0:t1] + D_h * x[t0:t1]
        carry = np.exp(lam[-1] - lam) * s                   # [Q]
        S = np.exp(lam[-1]) * S + (x[t0:t1] * carry[:, None]).T @ Bm[t0:t1]
    return y, S


def mamba2(S0, A, D, x, dt, Bm, Cm, chunk, dt_scales_input=False):
    """All (b, h).  S0 [B, H, P, N]; x [B, T, H, P]; dt [B, T, H]; Bm, Cm [B, T, G, N]."""
    Bn, H, P, N = S0.shape
    G = Bm.shape[2]
    T = x.shape[1]
    y = np.empty((Bn, T, H, P))
    S = np.empty_like(S0)
    for b in range(Bn):
        for h in range(H):
            g = h // (H // G)
            y[b, :, h], S[b, h] = mamba2_one_head(S0[b, h], A[h], D[h], x[b, :, h], dt[b, :, h],
                                                  Bm[b, :, g], Cm[b, :, g], chunk, dt_scales_input)
    return y, S
