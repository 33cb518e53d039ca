"""Seeded synthetic inputs for SSM-layer decode (Mamba-2, Gated DeltaNet, Kimi Delta Attention).

This module is the only code shared by the CUDA path's tests/benchmark and the
CPU oracle. It draws random numbers and rounds them to their storage dtype; it
holds none of the decode method's arithmetic (no recurrence, no decay products,
no quantisation of state).

Stream layout.  Every (seed, token t, sequence b) has its own numpy
``Generator(PCG64(SeedSequence([seed, t, b])))``, so any subset of sequences or
steps can be regenerated without materialising the rest.  Per-layer constants
(A_h, D_h) come from ``SeedSequence([seed, CONST_TAG])`` and the initial state of
sequence b from ``SeedSequence([seed, CONST_TAG, b])``.  Draw order per token:
Mamba-2 x, dt, B, C; Gated DeltaNet and KDA q, k, v, beta, alpha.

Distributions (the decode workloads of the ReplaySSM reports, restated):
  Mamba-2: x, B, C ~ N(0,1); dt = softplus(N(0,1) - 2); A_h = -exp(U(0,1));
           D_h ~ N(0,1); S_0 ~ N(0, 0.1^2).
  GDN:     q, k = v/|v| with v ~ N(0,1) per head; v ~ N(0,1);
           beta = sigmoid(N(0,1)); alpha = exp(-softplus(N(0,1))); S_0 ~ N(0, 0.1^2).
  KDA:     as GDN, with alpha drawn the same way for every key channel (alpha[H, d_k]).
x, B, C (q, k, v) are rounded to the workload's input dtype before either side
sees them, so buffering them in that dtype is lossless; dt, alpha, beta, A, D are
rounded to fp32.  Every array is returned as float64 holding exactly the rounded
values (what the oracle consumes) and, via ``to_torch``, in the storage dtype.
"""
from __future__ import annotations

import dataclasses
import numpy as np

CONST_TAG = 0xC0_57_A1_7E  # keeps constant streams apart from token streams (t >= 0)
ACCEPT_TAG = 1_000_000  # accept-length streams: SeedSequence([seed, ACCEPT_TAG + round])


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes and seeds of one decode workload for one SSM layer."""

    name: str
    kind: str  # "mamba2" | "gdn" | "kda"
    batch: int
    nheads: int
    headdim: int  # P: Mamba-2 headdim, GDN d_v
    dstate: int  # N: Mamba-2 dstate, GDN d_k
    ngroups: int  # Mamba-2 B/C groups (GDN: = nheads)
    window: int  # W, buffer window
    steps: int  # decode steps (or verify rounds for speculative workloads)
    seed: int
    read_dtype: str  # "f32" | "bf16" | "fp8" : replay read copy
    input_dtype: str  # "f32" | "bf16"
    max_draft: int = 1
    draft_k: int = 0  # >0: speculative verify workload with K drafts per round
    state_std: float = 0.1

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def state_shape(self):
        return (self.batch, self.nheads, self.headdim, self.dstate)


# The five decode workloads.  Names say what they are and their sizes.
WORKLOADS = {
    "mamba2_tiny_b2_h4_p16_n16_w4": Workload(
        "mamba2_tiny_b2_h4_p16_n16_w4", "mamba2", 2, 4, 16, 16, 1, 4, 32, 0, "f32", "f32"),
    "mamba2_nemotron_b256_h128_p64_n128_g8_w16": Workload(
        "mamba2_nemotron_b256_h128_p64_n128_g8_w16", "mamba2", 256, 128, 64, 128, 8, 16, 256, 1,
        "bf16", "bf16"),
    "mamba2_specverify_b512_h128_p64_n128_g8_w16_k4": Workload(
        "mamba2_specverify_b512_h128_p64_n128_g8_w16_k4", "mamba2", 512, 128, 64, 128, 8, 16, 128,
        2, "bf16", "bf16", max_draft=4, draft_k=4),
    "gdn_b256_h32_dk128_dv128_w16": Workload(
        "gdn_b256_h32_dk128_dv128_w16", "gdn", 256, 32, 128, 128, 32, 16, 256, 3, "bf16", "bf16"),
    "mamba2_fp8drift_b256_h128_p64_n128_g8": Workload(
        "mamba2_fp8drift_b256_h128_p64_n128_g8", "mamba2", 256, 128, 64, 128, 8, 16, 4096, 4,
        "fp8", "bf16"),
    # Kimi Delta Attention layer (per-channel gate), the GDN layer's shapes
    "kda_b256_h32_dk128_dv128_w16": Workload(
        "kda_b256_h32_dk128_dv128_w16", "kda", 256, 32, 128, 128, 32, 16, 256, 5, "bf16", "bf16"),
    # prompt prefill of the Nemotron-scale layer: 512 prompt tokens per sequence
    # (steps = prompt length), handing its final state to the decode checkpoint
    "mamba2_prefill_b256_h128_p64_n128_g8_t512": Workload(
        "mamba2_prefill_b256_h128_p64_n128_g8_t512", "mamba2", 256, 128, 64, 128, 8, 16, 512, 6,
        "bf16", "bf16"),
}
TINY, NEMOTRON, SPECVERIFY, GDN, FP8DRIFT, KDA, PREFILL = WORKLOADS.values()


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _softplus(z: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, z)


def round_to(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float data to the storage dtype (via fp32, torch's cast) and return it as
    float64 holding exactly the rounded values."""
    import torch

    f = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return f.astype(np.float64)
    if dtype == "bf16":
        return torch.from_numpy(f).to(torch.bfloat16).to(torch.float64).numpy()
    raise ValueError(dtype)


def constants(wl: Workload, seqs=None, f64: bool = True) -> dict:
    """Per-layer constants and the initial state S_0[seqs], fp32 values held in
    float64 (``f64=True``, what the oracle consumes) or in float32."""
    seqs = range(wl.batch) if seqs is None else seqs
    out = {}
    if wl.kind == "mamba2":
        g = _rng(wl.seed, CONST_TAG)
        out["A"] = round_to(-np.exp(g.uniform(0.0, 1.0, wl.nheads)), "f32")
        out["D"] = round_to(g.standard_normal(wl.nheads), "f32")
    s0 = np.empty((len(seqs), wl.nheads, wl.headdim, wl.dstate), np.float32)
    for i, b in enumerate(seqs):
        s0[i] = _rng(wl.seed, CONST_TAG, b).normal(0.0, wl.state_std,
                                                    (wl.nheads, wl.headdim, wl.dstate))
    out["S0"] = s0.astype(np.float64) if f64 else s0
    return out


def _token_one_seq(wl: Workload, t: int, b: int) -> dict:
    g = _rng(wl.seed, t, b)
    H, P, N = wl.nheads, wl.headdim, wl.dstate
    f32 = np.float32
    if wl.kind == "mamba2":
        G = wl.ngroups
        return {
            "x": g.standard_normal((H, P), dtype=f32),
            "dt": _softplus(g.standard_normal(H) - 2.0),
            "B": g.standard_normal((G, N), dtype=f32),
            "C": g.standard_normal((G, N), dtype=f32),
        }
    q = g.standard_normal((H, N), dtype=f32)
    k = g.standard_normal((H, N), dtype=f32)
    v = g.standard_normal((H, P), dtype=f32)
    beta = 1.0 / (1.0 + np.exp(-g.standard_normal(H)))
    alpha = np.exp(-_softplus(g.standard_normal((H, N) if wl.kind == "kda" else H)))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return {"q": q, "k": k, "v": v, "beta": beta, "alpha": alpha}


def token(wl: Workload, t: int, seqs=None) -> dict:
    """Inputs of absolute token index t for the given sequences.

    Returns float64 arrays shaped [len(seqs), ...] holding the dtype-rounded
    values: Mamba-2 x[b,H,P], dt[b,H], B[b,G,N], C[b,G,N]; GDN q,k[b,H,N],
    v[b,H,P], beta,alpha[b,H]; KDA as GDN with alpha[b,H,N].
    """
    seqs = list(range(wl.batch)) if seqs is None else list(seqs)
    parts = [_token_one_seq(wl, t, b) for b in seqs]
    out = {k: np.stack([p[k] for p in parts]) for k in parts[0]}
    wide = ("x", "B", "C") if wl.kind == "mamba2" else ("q", "k", "v")
    for k in out:
        out[k] = round_to(out[k], wl.input_dtype if k in wide else "f32")
    return out


def tokens(wl: Workload, t0: int, T: int, seqs=None) -> dict:
    """T consecutive tokens t0..t0+T-1 stacked on axis 1: x[b,T,H,P] etc."""
    steps = [token(wl, t0 + j, seqs) for j in range(T)]
    return {k: np.stack([s[k] for s in steps], axis=1) for k in steps[0]}


def accept_lengths(wl: Workload, rnd: int, seqs=None) -> np.ndarray:
    """Per-sequence accepted draft counts for verify round ``rnd``: U{0..K}."""
    a = _rng(wl.seed, ACCEPT_TAG + rnd).integers(0, wl.draft_k + 1, wl.batch)
    return a if seqs is None else a[list(seqs)]


def to_torch(a: np.ndarray, dtype: str):
    """float64 numpy -> torch CPU tensor in the storage dtype ("f32" | "bf16")."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(torch.float32) if dtype == "f32" else t.to(torch.float32).to(torch.bfloat16)
