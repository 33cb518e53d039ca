"""The synthetic hybrid decode step (five Mamba-2 layers per attention layer,
random weights): the SSM layers decoded by replay and by the eager baseline
must give the same hidden states through the whole stack -- with the fp32 read
path within the bf16 rounding of the stack's projections (a few ulps of bf16
where an SSM output rounds the other way), with the bf16 read copy within its
own tolerance -- and every SSM layer's counters must follow the ring model."""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200.hybrid import HybridShape, HybridStack
from oracle.ring import RingModel

pytestmark = pytest.mark.gpu

SHAPE = HybridShape(batch=4, blocks=2, ssm_per_block=5, d_model=256, nheads=8, headdim=32, dstate=64, ngroups=2,
                    window=4, n_q_heads=4, n_kv_heads=2, head_dim=64, context=64)


def _run(mode, read_dtype, steps=12):
    import torch

    st = HybridStack(SHAPE, ssm_mode=mode, read_dtype=read_dtype, seed=5, max_steps=steps)
    g = torch.Generator(device="cuda").manual_seed(9)
    outs = []
    for _ in range(steps):
        x = torch.randn((SHAPE.batch, SHAPE.d_model), generator=g, device="cuda").to(torch.bfloat16)
        outs.append(st.step(x).float().cpu().numpy())
    torch.cuda.synchronize()
    return st, np.stack(outs)


def test_replay_and_eager_steps_agree():
    st_r, xr = _run("replay", "f32")
    st_e, xe = _run("eager", "f32")
    _, xb = _run("replay", "bf16")
    rms = lambda a: float(np.sqrt(np.mean(np.square(a))))
    scale = rms(xe)
    assert np.isfinite(xr).all() and np.isfinite(xb).all()
    assert rms(xr - xe) <= 1e-2 * scale and np.max(np.abs(xr - xe)) <= 1e-1 * scale
    assert rms(xb - xe) <= 5e-2 * scale
    rm = RingModel(SHAPE.batch, SHAPE.window, 1)
    for _ in range(12):
        rm.decode()
    for L in st_r.ssm_layers():
        sp, ck, pe, fc = L.counters()
        assert np.array_equal(sp, rm.seq_pos) and np.array_equal(ck, rm.ckpt_pos)
        assert np.array_equal(fc, rm.flush_count)
        assert L.status()[0] == 0
    assert len(st_r.ssm_layers()) == SHAPE.blocks * SHAPE.ssm_per_block
