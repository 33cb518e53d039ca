"""Algorithmic HBM bytes of the decode kernels, per (sequence, head) per call.

The bytes each kernel must move at minimum, counted from the data it reads and
writes (no re-reads): the state tile, the buffered entries it replays or folds,
the call's tokens, the output, the ring append and the prep -> read hand-off
(replay coefficients).  Group-shared Mamba-2 B/C data is charged 1/(heads per
group) to each head.  A replay decode runs two kernels: the prep/flush kernel
(coefficients, and the fold when the buffer is full) and the replay-read kernel
(read copy + buffered inputs -> output).  Plain decode cycles through buffer
lengths L0 = W (fold step), 1, 2, ..., W-1, so the per-token figure is the mean
over one window.  These are the per-unit figures of the benchmark's roofline
(achieved = bytes per launch / launch time).
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


def state_tile(s: Shape, dtype: str) -> float:
    extra = s.headdim * 4 if dtype == "fp8" else 0  # per-row scales
    return s.headdim * s.dstate * SB[dtype] + extra


def _grp(s: Shape) -> float:
    return s.heads_per_group if s.kind == "mamba2" else 1


def _x_row(s: Shape) -> float:  # Mamba-2 x / GDN v of one token, one head
    return s.headdim * SB[s.input_dtype]


def _key_row(s: Shape) -> float:  # Mamba-2 B (charged per head) / GDN, KDA k
    return s.dstate * SB[s.input_dtype] / _grp(s)


def _scalars(s: Shape) -> float:  # per-token fp32 gates: dt; alpha + beta; KDA alpha[d_k] + beta
    return {"mamba2": 4.0, "gdn": 8.0}.get(s.kind, s.dstate * 4.0 + 4.0)


def _handoff(s: Shape, L0: int, T: int) -> float:
    """Prep -> read hand-off per (b, h): coefficients over the replayed entries and
    a decay per query; GDN and KDA also hand over the swept query (d_k fp32)."""
    per_query = (L0 + T) * 4 + 4 + (0 if s.kind == "mamba2" else s.dstate * 4)
    return T * per_query


def replay_step_split(s: Shape, L0: int, fold: bool, T: int = 1) -> dict:
    """Bytes per (b, h) of one replay decode (T = 1) or verify (T = K) call, by kernel.

    L0 committed entries are buffered before the call; ``fold`` when they are
    folded into the checkpoint by this call (then the read kernel skips the head).
    """
    x, k = _x_row(s), _key_row(s)
    scal = _scalars(s)
    q = k  # Mamba-2 C (group-shared), GDN / KDA q
    prep = {
        "buffer_read": L0 * (k + scal) + (L0 * x if fold else 0.0),
        "inputs": T * (q + k + scal + x),
        "append": T * (x + k + scal),
    }
    read = {}
    if fold:
        prep["ckpt_read"] = state_tile(s, "f32")
        prep["ckpt_write"] = state_tile(s, "f32")
        prep["copy_write"] = state_tile(s, s.read_dtype) if s.read_dtype != "f32" else 0.0
        prep["output"] = T * s.headdim * 4
    else:
        prep["handoff_write"] = _handoff(s, L0, T)
        read = {
            "copy_read": state_tile(s, s.read_dtype),
            "buffer_read": L0 * x,
            "inputs": T * x + (q if s.kind == "mamba2" else 0.0),
            "handoff_read": prep["handoff_write"],
            "output": T * s.headdim * 4,
        }
    return {"prep": prep, "read": read}


def replay_decode_window(s: Shape) -> dict:
    """Per-kernel bytes per (b, h) per token, averaged over one window of plain decode."""
    W = s.window
    steps = [replay_step_split(s, W, True)] + [replay_step_split(s, L0, False) for L0 in range(1, W)]
    out = {}
    for kern in ("prep", "read"):
        keys = sorted({k for st in steps for k in st[kern]})
        out[kern] = {k: sum(st[kern].get(k, 0.0) for st in steps) / W for k in keys}
    return out


def replay_decode_per_token(s: Shape) -> dict:
    """All replay bytes per (b, h) per token (both kernels), mean over a window."""
    w = replay_decode_window(s)
    out = {}
    for kern in w.values():
        for k, v in kern.items():
            out[k] = out.get(k, 0.0) + v
    return out


def eager_decode_per_token(s: Shape, state_dtype: str = "f32") -> dict:
    x, k = _x_row(s), _key_row(s)
    t = state_tile(s, state_dtype)
    return {"inputs": 2 * k + x + _scalars(s),
            "output": s.headdim * 4, "state_read": t, "state_write": t}


STATE_KEYS = ("copy_read", "ckpt_read", "ckpt_write", "copy_write", "buffer_read", "append",
              "handoff_write", "handoff_read", "state_read", "state_write")


def total(d: dict) -> float:
    return float(sum(d.values()))


def state_bytes(d: dict) -> float:
    """State traffic only (checkpoint, copy, buffer, hand-off), without the call's
    inputs and outputs."""
    return float(sum(v for k, v in d.items() if k in STATE_KEYS))


def eager_verify_round(s: Shape, K: int, state_dtype: str = "f32") -> dict:
    t = state_tile(s, state_dtype)
    return {"inputs": K * (2 * _key_row(s) + _x_row(s) + 4), "output": K * s.headdim * 4,
            "state_read": t, "snapshot_write": K * t}
