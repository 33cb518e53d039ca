"""Helpers for the GPU parity tests (imported by test_gpu_*.py; not collected)."""
from __future__ import annotations

import numpy as np

from checkpoint_input_replay_rssm_b200 import inputs as I

WIDE = {"mamba2": ("x", "B", "C"), "gdn": ("q", "k", "v"), "kda": ("q", "k", "v")}


def make_layer(wl: I.Workload, mode="replay", state_dtype=None, max_draft=None, dt_scales=False,
               consts=None):
    import torch

    from checkpoint_input_replay_rssm_b200 import rssm

    cfg = rssm.make_config(kind=wl.kind, mode=mode, state_dtype=state_dtype or wl.read_dtype,
                           input_dtype=wl.input_dtype, batch=wl.batch, nheads=wl.nheads,
                           headdim=wl.headdim, dstate=wl.dstate, ngroups=wl.ngroups,
                           window=wl.window,
                           max_draft=wl.max_draft if max_draft is None else max_draft,
                           dt_scales_input=dt_scales)
    L = rssm.Layer(cfg)
    c = consts if consts is not None else I.constants(wl, f64=False)
    if wl.kind == "mamba2":
        L.set_params(torch.tensor(c["A"], dtype=torch.float32, device="cuda"),
                     torch.tensor(c["D"], dtype=torch.float32, device="cuda"))
    L.import_state(torch.from_numpy(np.ascontiguousarray(c["S0"], dtype=np.float32)).cuda())
    return L, c


def to_device(tok: dict, wl: I.Workload, with_T: bool = True) -> dict:
    """numpy float64 token arrays ([B,...] or [B,T,...]) -> CUDA tensors [B,T,...]."""
    out = {}
    for k, v in tok.items():
        t = I.to_torch(v, wl.input_dtype if k in WIDE[wl.kind] else "f32")
        if not with_T:
            t = t.unsqueeze(1)
        out[k] = t.contiguous().cuda()
    return out


def rel_err(y, ref) -> float:
    """max |y - ref| / RMS(ref): the per-step tolerance metric."""
    rms = float(np.sqrt(np.mean(np.square(ref))))
    return float(np.max(np.abs(np.asarray(y, np.float64) - ref))) / max(rms, 1e-30)


def oracle_params(c):
    return {"A": c.get("A"), "D": c.get("D")}
