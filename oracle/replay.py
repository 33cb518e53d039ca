"""fp64 replay formulation of SSM decode (checkpoint + input buffer) -- TEST INFRASTRUCTURE.

This restates, in float64 and in plain numpy, how the ReplaySSM reports compute
a token's output from a checkpoint and a buffer of recent inputs without writing
state, and how the checkpoint is rewritten only when the buffer is full
("Tenir le journal plutot que le solde", blog.thibaultmonteiro.fr;
"L'astuce du checkpoint et du tampon", irisproject.cloud).  The bookkeeping
(ring slots, lazy flush, verify/commit) is oracle/ring.py's.  The algebra is the
unrolled recurrence, read from the checkpoint S_c and the buffered entries
1..L (L includes the token being decoded):

Mamba-2 (a_i = exp(dt_i A_h), s_i = dt_i if dt scales the input else 1):
    y = (prod_{i<=L} a_i) (S^ C) + sum_{i<=L} (prod_{i<j<=L} a_j) (B_i . C) s_i x_i + D x_L
    fold:  S_c <- (prod_i a_i) S_c + sum_i (prod_{j>i} a_j) s_i x_i B_i^T
Gated DeltaNet (backward sweep applying the delta-rule factors to q):
    r <- q;  for j = L..1: c_j = beta_j (k_j . r);  r <- alpha_j (r - c_j k_j)
    o = S^ r + sum_j c_j v_j
    fold:  for j = 1..L: S_c <- alpha_j S_c (I - beta_j k_j k_j^T) + beta_j v_j k_j^T
Kimi Delta Attention (alpha_j a gate per key channel; the same sweep with
Diag(alpha_j) in place of the scalar):
    r <- q;  for j = L..1: c_j = beta_j (k_j . r);  r <- alpha_j (.) (r - c_j k_j)
    o = S^ r + sum_j c_j v_j
    fold:  for j = 1..L: S_c <- S_c Diag(alpha_j) (I - beta_j k_j k_j^T) + beta_j v_j k_j^T
S^ is the read copy: the fp32 checkpoint itself, or its bf16 / per-row fp8
rounding (oracle/quant.py); rounding of the copy never feeds the fold, which
always starts from the full-precision checkpoint ("Deux precisions pour le prix
d'une", irisproject.cloud).  Decay products are explicit fp64 products.
A verify of K drafts gives draft m the entries up to and including itself.
"""
from __future__ import annotations

import numpy as np

from . import quant
from .ring import RingModel


class ReplayOracle:
    """One layer, all sequences.  Holds the checkpoint in float64."""

    def __init__(self, kind: str, S0: np.ndarray, window: int, max_draft: int = 1,
                 read_dtype: str = "f64", params: dict | None = None, ngroups: int = 1,
                 dt_scales_input: bool = False):
        self.kind = kind
        Bn, H, P, N = S0.shape
        self.B, self.H, self.P, self.N = Bn, H, P, N
        self.G = ngroups if kind == "mamba2" else H
        self.read_dtype = read_dtype
        self.params = params or {}
        self.dt_scales_input = dt_scales_input
        self.ring = RingModel(Bn, window, max_draft)
        self.R = self.ring.R
        self.ckpt = np.array(S0, dtype=np.float64, copy=True)
        self.rc = quant.read_copy(self.ckpt, read_dtype)
        self.buf = {}  # name -> [B, R, ...] ring of buffered inputs
        if kind == "mamba2":
            self.buf["x"] = np.zeros((Bn, self.R, H, P))
            self.buf["dt"] = np.zeros((Bn, self.R, H))
            self.buf["B"] = np.zeros((Bn, self.R, self.G, N))
        else:
            self.buf["k"] = np.zeros((Bn, self.R, H, N))
            self.buf["v"] = np.zeros((Bn, self.R, H, P))
            self.buf["alpha"] = np.zeros((Bn, self.R, H, N) if kind == "kda" else (Bn, self.R, H))
            self.buf["beta"] = np.zeros((Bn, self.R, H))

    # ---------------------------------------------------------------- entries
    def _entries(self, b: int, n0: int, n1: int) -> dict:
        """Buffered inputs of tokens n0..n1-1 of sequence b, each [L, ...]."""
        idx = [n % self.R for n in range(n0, n1)]
        return {k: v[b, idx] for k, v in self.buf.items()}

    # ---------------------------------------------------------------- algebra
    def _fold_seq(self, S: np.ndarray, e: dict) -> np.ndarray:
        """Fold entries e (length L) into S[H,P,N] of one sequence."""
        if self.kind == "mamba2":
            A = self.params["A"]
            L = e["dt"].shape[0]
            a = np.exp(e["dt"] * A[None, :])  # [L,H]
            out = np.prod(a, axis=0)[:, None, None] * S
            hpg = self.H // self.G
            for i in range(L):
                w = np.prod(a[i + 1:], axis=0)  # [H]
                s = e["dt"][i] if self.dt_scales_input else np.ones(self.H)
                Bh = np.repeat(e["B"][i], hpg, axis=0)  # [H,N]
                out = out + (w * s)[:, None, None] * e["x"][i][:, :, None] * Bh[:, None, :]
            return out
        out = S.copy()
        if self.kind == "kda":
            for i in range(e["k"].shape[0]):
                k, v = e["k"][i], e["v"][i]  # [H,N], [H,P]
                al, be = e["alpha"][i], e["beta"][i]  # [H,N], [H]
                u = al[:, None, :] * out
                uk = np.einsum("hpn,hn->hp", u, k)
                out = u - be[:, None, None] * uk[:, :, None] * k[:, None, :] \
                    + be[:, None, None] * v[:, :, None] * k[:, None, :]
            return out
        for i in range(e["k"].shape[0]):
            k, v = e["k"][i], e["v"][i]  # [H,N], [H,P]
            al, be = e["alpha"][i], e["beta"][i]
            Sk = np.einsum("hpn,hn->hp", out, k)
            out = al[:, None, None] * (out - be[:, None, None] * Sk[:, :, None] * k[:, None, :]) \
                + be[:, None, None] * v[:, :, None] * k[:, None, :]
        return out

    def _read_seq(self, rc: np.ndarray, e: dict, q: dict) -> np.ndarray:
        """Output of one query token from the read copy rc[H,P,N] and entries e
        (the last entry is the query token itself).  q holds the query token's
        C (Mamba-2) or q (GDN) and, for Mamba-2, its x for the skip term."""
        if self.kind == "mamba2":
            A, D = self.params["A"], self.params["D"]
            hpg = self.H // self.G
            L = e["dt"].shape[0]
            a = np.exp(e["dt"] * A[None, :])
            Ch = np.repeat(q["C"], hpg, axis=0)  # [H,N]
            y = np.prod(a, axis=0)[:, None] * np.einsum("hpn,hn->hp", rc, Ch)
            for i in range(L):
                w = np.prod(a[i + 1:], axis=0)
                s = e["dt"][i] if self.dt_scales_input else np.ones(self.H)
                Bh = np.repeat(e["B"][i], hpg, axis=0)
                y = y + (w * s * np.sum(Bh * Ch, axis=1))[:, None] * e["x"][i]
            return y + D[:, None] * q["x"]
        r = q["q"].copy()  # [H,N]
        o = np.zeros((self.H, self.P))
        for j in range(e["k"].shape[0] - 1, -1, -1):
            c = e["beta"][j] * np.sum(e["k"][j] * r, axis=1)  # [H]
            al = e["alpha"][j] if self.kind == "kda" else e["alpha"][j][:, None]
            r = al * (r - c[:, None] * e["k"][j])
            o = o + c[:, None] * e["v"][j]
        return o + np.einsum("hpn,hn->hp", rc, r)

    def _fold_and_requant(self, b: int, n0: int, n1: int):
        if n1 > n0:
            self.ckpt[b] = self._fold_seq(self.ckpt[b], self._entries(b, n0, n1))
            self.rc[b] = quant.read_copy(self.ckpt[b], self.read_dtype)

    # ---------------------------------------------------------------- API
    def _run(self, toks: dict, K: int, verify: bool) -> np.ndarray:
        ck0 = self.ring.ckpt_pos.copy()
        sp0 = self.ring.seq_pos.copy()
        if verify:
            mask, _ = self.ring.verify(K)
        else:
            mask, _ = self.ring.decode()
        out = np.empty((self.B, K, self.H, self.P))
        for b in range(self.B):
            if mask[b]:
                self._fold_and_requant(b, int(ck0[b]), int(sp0[b]))
            for j in range(K):
                n = int(sp0[b]) + j
                s = n % self.R
                for k in self.buf:
                    self.buf[k][b, s] = toks[k][b, j]
            ck = int(self.ring.ckpt_pos[b])
            for j in range(K):
                n = int(sp0[b]) + j
                e = self._entries(b, ck, n + 1)
                qtok = {k: toks[k][b, j] for k in toks}
                out[b, j] = self._read_seq(self.rc[b], e, qtok)
        return out

    def decode(self, tok: dict) -> np.ndarray:
        """tok: one token, arrays [B,...] (as from inputs.token). Returns y[B,H,P]."""
        toks = {k: v[:, None] for k, v in tok.items()}
        return self._run(toks, 1, verify=False)[:, 0]

    def verify(self, toks: dict) -> np.ndarray:
        """toks: K drafts, arrays [B,K,...]. Returns y[B,K,H,P]; appends drafts uncommitted."""
        K = next(iter(toks.values())).shape[1]
        return self._run(toks, K, verify=True)

    def commit(self, accept) -> np.ndarray:
        return self.ring.commit(accept)

    def flush(self):
        ck0 = self.ring.ckpt_pos.copy()
        mask = self.ring.flush()
        for b in np.nonzero(mask)[0]:
            self._fold_and_requant(int(b), int(ck0[b]), int(self.ring.seq_pos[b]))
        return mask

    def export(self) -> np.ndarray:
        """Committed state (checkpoint with committed entries folded in), not mutating."""
        out = self.ckpt.copy()
        for b in range(self.B):
            ck, sp = int(self.ring.ckpt_pos[b]), int(self.ring.seq_pos[b])
            if sp > ck:
                out[b] = self._fold_seq(self.ckpt[b], self._entries(b, ck, sp))
        return out


class LowPrecEagerOracle:
    """Eager recurrence whose single state is stored rounded ("bf16" | "fp8") every
    token: dequantise, update in fp64, output from the updated value, requantise.
    This is the single shared low-precision state that accumulates rounding error
    (the third difficulty of "Trois ennuis nes de la meme fusion",
    blog.thibaultmonteiro.fr), used as the comparator of the dual-precision path."""

    def __init__(self, kind: str, S0: np.ndarray, dtype: str, params: dict | None = None,
                 ngroups: int = 1, dt_scales_input: bool = False):
        self.kind, self.dtype = kind, dtype
        self.params = params or {}
        self.G = ngroups
        self.dt_scales_input = dt_scales_input
        self.S = quant.read_copy(S0, dtype)

    def decode(self, tok: dict) -> np.ndarray:
        from . import eager  # C oracle step on the dequantised state
        S = np.ascontiguousarray(self.S.copy())
        y = eager.step(self.kind, S, tok, self.params, self.dt_scales_input)
        self.S = quant.read_copy(S, self.dtype)
        return y
