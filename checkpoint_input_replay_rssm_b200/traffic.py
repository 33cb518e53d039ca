"""Algorithmic HBM bytes of the decode kernels, per (sequence, head) per token.

The bytes each kernel must move at minimum, counted from the data it reads and
writes (no re-reads): the state tile, the buffered entries it replays or folds,
the token's inputs, the output, the ring append.  Group-shared Mamba-2 B/C data
is charged 1/(heads per group) to each head.  Plain decode cycles through
buffer lengths L0 = W (fold step), 1, 2, ..., W-1, so the per-token figure is the
mean over one window.  These are the per-unit figures the benchmark's roofline
uses (achieved = bytes per launch / launch time).
"""
from __future__ import annotations

import dataclasses

SB = {"f32": 4, "bf16": 2, "fp8": 1}


@dataclasses.dataclass
class Shape:
    kind: str = "mamba2"
    headdim: int = 64
    dstate: int = 128
    heads_per_group: int = 16
    window: int = 16
    read_dtype: str = "bf16"   # replay read copy (f32 = the checkpoint itself)
    input_dtype: str = "bf16"


def _entry_bytes(s: Shape) -> float:
    """Bytes of one buffered entry as the replay/fold reads it (per head)."""
    ib = SB[s.input_dtype]
    if s.kind == "mamba2":
        return s.headdim * ib + 4 + s.dstate * ib / s.heads_per_group
    return (s.headdim + s.dstate) * ib + 8  # v, k, alpha, beta


def _token_io(s: Shape, T: int = 1) -> dict:
    ib = SB[s.input_dtype]
    if s.kind == "mamba2":
        inputs = s.headdim * ib + 4 + 2 * s.dstate * ib / s.heads_per_group
    else:
        inputs = (s.headdim + 2 * s.dstate) * ib + 8
    return {"inputs": T * inputs, "output": T * s.headdim * 4, "append": T * _entry_bytes(s)}


def state_tile(s: Shape, dtype: str) -> float:
    extra = s.headdim * 4 if dtype == "fp8" else 0  # per-row scales
    return s.headdim * s.dstate * SB[dtype] + extra


def replay_step(s: Shape, L0: int, fold: bool) -> dict:
    """One replay decode launch's bytes per (b, h) with L0 committed entries buffered."""
    io = _token_io(s)
    d = {"inputs": io["inputs"], "output": io["output"], "append": io["append"]}
    if fold:
        d["ckpt_read"] = state_tile(s, "f32")
        d["ckpt_write"] = state_tile(s, "f32")
        d["copy_write"] = state_tile(s, s.read_dtype) if s.read_dtype != "f32" else 0.0
        d["buffer_read"] = L0 * _entry_bytes(s)
    else:
        d["copy_read"] = state_tile(s, s.read_dtype)
        d["buffer_read"] = L0 * _entry_bytes(s)
    return d


def replay_decode_per_token(s: Shape) -> dict:
    """Mean over one window of plain decode (one fold step, W - 1 read steps)."""
    W = s.window
    steps = [replay_step(s, W, True)] + [replay_step(s, L0, False) for L0 in range(1, W)]
    keys = sorted({k for st in steps for k in st})
    return {k: sum(st.get(k, 0.0) for st in steps) / W for k in keys}


def eager_decode_per_token(s: Shape, state_dtype: str = "f32") -> dict:
    io = _token_io(s)
    t = state_tile(s, state_dtype)
    return {"inputs": io["inputs"], "output": io["output"], "state_read": t, "state_write": t}


STATE_KEYS = ("copy_read", "ckpt_read", "ckpt_write", "copy_write", "buffer_read", "append",
              "state_read", "state_write")


def total(d: dict) -> float:
    return float(sum(d.values()))


def state_bytes(d: dict) -> float:
    """State traffic only (checkpoint, copy, buffer), without the token's inputs/output."""
    return float(sum(v for k, v in d.items() if k in STATE_KEYS))


def verify_round(s: Shape, K: int, L0: int, fold: bool) -> dict:
    """One replay verify launch of K drafts, per (b, h)."""
    io = _token_io(s, K)
    d = {"inputs": io["inputs"], "output": io["output"], "append": io["append"],
         "buffer_read": L0 * _entry_bytes(s)}
    if fold:
        d["ckpt_read"] = state_tile(s, "f32")
        d["ckpt_write"] = state_tile(s, "f32")
        d["copy_write"] = state_tile(s, s.read_dtype) if s.read_dtype != "f32" else 0.0
    else:
        d["copy_read"] = state_tile(s, s.read_dtype)
    return d


def eager_verify_round(s: Shape, K: int, state_dtype: str = "f32") -> dict:
    io = _token_io(s, K)
    t = state_tile(s, state_dtype)
    return {"inputs": io["inputs"], "output": io["output"], "state_read": t,
            "snapshot_write": K * t}
