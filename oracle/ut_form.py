"""Chunked (WY / UT) form of the delta-rule fold -- TEST INFRASTRUCTURE.

Only tests/ may import this.  It folds L buffered entries into a checkpoint in
one step per head instead of L sequential row updates, and is pinned against the
sequential fold of oracle/replay.py (tests/test_oracle_ut.py): a second,
independent route to the same numbers, and the algebra a chunked flush kernel
would use.  The pages name the delta-rule layers (Gated DeltaNet, Kimi Delta
Attention) and say their updates have the same checkpoint + buffer form
(blog.thibaultmonteiro.fr, "La fiche qu'on reecrit a chaque token"); this
module only restates that algebra, in float64, with dense numpy linear algebra.

Per row s of the state (d_k wide) the entries i = 0..L-1 apply
    s_i = g_i (.) s_{i-1} + w_i k_i,     w_i = beta_i (v_i[row] - (g_i (.) s_{i-1}) . k_i)
with g_i the gate (GDN: a scalar on every channel; KDA: one per key channel).
With G_i = g_0 (.) ... (.) g_i and D_ij = G_i / G_j (the gates of entries j+1..i):
    s_i = G_i (.) s_0 + sum_{j<=i} w_j D_ij (.) k_j
so the w of one row solve the unit lower-triangular system
    w_i + beta_i sum_{j<i} ((D_ij (.) k_j) . k_i) w_j = beta_i (v_i[row] - (G_i (.) s_0) . k_i),
whose matrix is shared by every row of the head, and the folded row is
    s_L = G_{L-1} (.) s_0 + sum_j w_j D_{L-1,j} (.) k_j.
"""
from __future__ import annotations

import numpy as np


def _gates(alpha: np.ndarray, N: int) -> np.ndarray:
    """alpha [L] (one gate per entry) or [L, N] -> [L, N]."""
    a = np.asarray(alpha, dtype=np.float64)
    return np.repeat(a[:, None], N, axis=1) if a.ndim == 1 else a


def fold_one_head(S0: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: np.ndarray,
                  beta: np.ndarray) -> np.ndarray:
    """S0 [P, N]; k [L, N]; v [L, P]; alpha [L] or [L, N]; beta [L].  Returns S_L [P, N]."""
    L, N = k.shape
    if L == 0:
        return S0.copy()
    g = _gates(alpha, N)
    # D[i, j] = prod_{j < l <= i} g_l (per channel), for j <= i; products, no division
    D = np.zeros((L, L, N))
    for j in range(L):
        acc = np.ones(N)
        D[j, j] = acc
        for i in range(j + 1, L):
            acc = acc * g[i]
            D[i, j] = acc
    G = np.cumprod(g, axis=0)                         # G_i = g_0 ... g_i
    # system matrix, shared by the rows: unit lower triangular
    Mt = np.eye(L)
    for i in range(L):
        for j in range(i):
            Mt[i, j] = beta[i] * np.dot(D[i, j] * k[j], k[i])
    # right-hand sides of every row at once: [L, P]
    a = np.stack([S0 @ (G[i] * k[i]) for i in range(L)])     # (G_i (.) s_0) . k_i per row
    rhs = beta[:, None] * (v - a)
    w = np.linalg.solve(Mt, rhs)                      # [L, P]
    out = G[L - 1][None, :] * S0
    for j in range(L):
        out = out + np.outer(w[j], D[L - 1, j] * k[j])
    return out


def fold(S: np.ndarray, e: dict) -> np.ndarray:
    """All heads of one sequence.  S [H, P, N]; e as the replay oracle buffers it:
    k [L, H, N], v [L, H, P], alpha [L, H] or [L, H, N], beta [L, H]."""
    H = S.shape[0]
    out = np.empty_like(S)
    for h in range(H):
        al = e["alpha"][:, h]
        out[h] = fold_one_head(S[h], e["k"][:, h], e["v"][:, h], al, e["beta"][:, h])
    return out
