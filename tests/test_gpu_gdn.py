"""Gated DeltaNet decode on the GPU against the fp64 CPU oracle (tolerances as for Mamba-2)."""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from oracle import eager
from oracle.replay import LowPrecEagerOracle, ReplayOracle
from oracle.ring import RingModel
from tests.gpu_common import make_layer, rel_err, to_device

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _run(wl, mode, dtypes, steps, seqs=None, emulate=False):
    import torch

    full = I.constants(wl, f64=False)
    layers = {d: make_layer(wl, mode=mode, state_dtype=d, consts=full)[0] for d in dtypes}
    del full
    c = I.constants(wl, seqs)
    seqs = list(range(wl.batch)) if seqs is None else list(seqs)
    S = np.ascontiguousarray(c["S0"].copy())
    emu = {}
    if emulate:
        for d in dtypes:
            if mode == "replay":
                emu[d] = ReplayOracle("gdn", c["S0"], wl.window, read_dtype=d)
            elif d != "f32":
                emu[d] = LowPrecEagerOracle("gdn", c["S0"], d)
    worst = {d: 0.0 for d in dtypes}
    worst_emu = {d: 0.0 for d in dtypes}
    for t in range(steps):
        tok = I.token(wl, t)
        dev = to_device(tok, wl, with_T=False)
        ys = {d: L.decode(dev) for d, L in layers.items()}
        sub = {k: v[seqs] for k, v in tok.items()}
        o_ref = eager.gdn_step(S, sub["q"], sub["k"], sub["v"], sub["alpha"], sub["beta"])
        for d, y in ys.items():
            yc = y[seqs, 0].double().cpu().numpy()
            worst[d] = max(worst[d], rel_err(yc, o_ref))
            if d in emu:
                worst_emu[d] = max(worst_emu[d], rel_err(yc, emu[d].decode(sub)))
    torch.cuda.synchronize()
    return layers, worst, worst_emu, S


def _gdn_tiny(**kw):
    base = dict(name="gdn_tiny", kind="gdn", batch=2, nheads=3, headdim=16, dstate=16, ngroups=3,
                window=4, steps=30, seed=21, read_dtype="f32", input_dtype="f32")
    base.update(kw)
    return I.Workload(**base)


def test_tiny_replay_and_eager_fp32():
    wl = _gdn_tiny()
    for mode in ("replay", "eager"):
        layers, worst, _, S = _run(wl, mode, ["f32"], wl.steps)
        assert worst["f32"] <= 1e-4, (mode, worst)
        exp = layers["f32"].export_state().double().cpu().numpy()
        assert rel_err(exp, S) <= 1e-5
        sp, ck, pe, fc = layers["f32"].counters()
        rm = RingModel(wl.batch, wl.window, 1, mode=mode)
        for _ in range(wl.steps):
            rm.decode()
        assert sp.tolist() == rm.seq_pos.tolist() and fc.tolist() == rm.flush_count.tolist()


@pytest.mark.parametrize("N,P,W", [(16, 8, 3), (32, 40, 5), (64, 72, 7), (128, 24, 2), (128, 128, 16)])
def test_ragged_shapes_all_read_copies(N, P, W):
    wl = _gdn_tiny(batch=3, nheads=2, ngroups=2, headdim=P, dstate=N, window=W, steps=2 * W + 3)
    _, worst, worst_emu, _ = _run(wl, "replay", ["f32", "bf16", "fp8"], wl.steps, emulate=True)
    assert worst["f32"] <= TOL["f32"], worst
    assert worst["bf16"] <= TOL["bf16"], worst
    assert worst_emu["bf16"] <= 2e-3, worst_emu
    assert worst_emu["fp8"] <= 6e-2, worst_emu


@pytest.mark.parametrize("sd", ["f32", "bf16", "fp8"])
def test_eager_baselines(sd):
    wl = _gdn_tiny(batch=2, nheads=2, ngroups=2, headdim=24, dstate=32, window=4, steps=16)
    _, worst, worst_emu, _ = _run(wl, "eager", [sd], wl.steps, emulate=True)
    if sd == "f32":
        assert worst[sd] <= 1e-4
    else:
        assert worst_emu[sd] <= (2e-2 if sd == "bf16" else 6e-2), worst_emu


def test_gdn_layer_full_size_sampled():
    """Batch 256 x 32 heads x 128 x 128, W = 16, 256 steps, bf16 read copy and fp32
    read path; 16 sequences (first, last, both sides of the halfway and quarter
    marks) at every step against the fp64 oracle, every counter exact."""
    wl = I.GDN
    seqs = [0, 1, 2, 63, 64, 100, 127, 128, 129, 150, 191, 192, 200, 230, 254, 255]
    layers, worst, _, S = _run(wl, "replay", ["bf16", "f32"], wl.steps, seqs=seqs)
    assert worst["bf16"] <= TOL["bf16"], worst
    assert worst["f32"] <= TOL["f32"], worst
    rm = RingModel(wl.batch, wl.window, 1)
    for _ in range(wl.steps):
        rm.decode()
    for L in layers.values():
        sp, ck, pe, fc = L.counters()
        assert np.array_equal(sp, rm.seq_pos) and np.array_equal(ck, rm.ckpt_pos)
        assert np.array_equal(fc, rm.flush_count)
        assert rel_err(L.export_state()[seqs].double().cpu().numpy(), S) <= 1e-5
        assert L.status()[0] == 0
