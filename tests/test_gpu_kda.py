"""Kimi Delta Attention (gate per key channel) decode on the GPU against the fp64 CPU
oracle, through the C ABI: replay (fp32 read path, bf16 and fp8 read copies),
the eager baselines, verify / commit, flush and export, and the full-size layer
(batch 256 x 32 heads x d_k = d_v = 128, W = 16) on sampled sequences.
Tolerances as for the other kinds: 1e-4 x RMS (fp32 path), 2e-2 x RMS (bf16
copy), 6e-2 x RMS against the emulated fp8 copy; counters bit-exact."""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from oracle import eager
from oracle.replay import LowPrecEagerOracle, ReplayOracle
from oracle.ring import RingModel
from tests.gpu_common import make_layer, rel_err, to_device
from tests.test_gpu_spec import _spec_run

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
                emu[d] = ReplayOracle("kda", c["S0"], wl.window, read_dtype=d)
            elif d != "f32":
                emu[d] = LowPrecEagerOracle("kda", c["S0"], d)
    worst = {d: 0.0 for d in dtypes}
    worst_emu = {d: 0.0 for d in dtypes}
    for t in range(steps):
        tok = I.token(wl, t)
        dev = to_device(tok, wl, with_T=False)
        ys = {d: L.decode(dev) for d, L in layers.items()}
        sub = {k: v[seqs] for k, v in tok.items()}
        o_ref = eager.kda_step(S, sub["q"], sub["k"], sub["v"], sub["alpha"], sub["beta"])
        for d, y in ys.items():
            yc = y[seqs, 0].double().cpu().numpy()
            worst[d] = max(worst[d], rel_err(yc, o_ref))
            if d in emu:
                worst_emu[d] = max(worst_emu[d], rel_err(yc, emu[d].decode(sub)))
    torch.cuda.synchronize()
    return layers, worst, worst_emu, S


def _kda_tiny(**kw):
    base = dict(name="kda_tiny", kind="kda", batch=2, nheads=3, headdim=16, dstate=16, ngroups=3,
                window=4, steps=30, seed=51, read_dtype="f32", input_dtype="f32")
    base.update(kw)
    return I.Workload(**base)


def test_token_inputs_have_a_gate_per_key_channel():
    tok = I.token(_kda_tiny(), 0)
    assert tok["alpha"].shape == (2, 3, 16)
    assert len(np.unique(tok["alpha"])) > 16  # not one value per head


def test_tiny_replay_and_eager_fp32():
    wl = _kda_tiny()
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
    wl = _kda_tiny(batch=3, nheads=2, ngroups=2, headdim=P, dstate=N, window=W, steps=2 * W + 3)
    _, worst, worst_emu, _ = _run(wl, "replay", ["f32", "bf16", "fp8"], wl.steps, emulate=True)
    assert worst["f32"] <= TOL["f32"], worst
    assert worst["bf16"] <= TOL["bf16"], worst
    assert worst_emu["bf16"] <= 2e-3, worst_emu
    assert worst_emu["fp8"] <= 6e-2, worst_emu


@pytest.mark.parametrize("sd", ["f32", "bf16", "fp8"])
def test_eager_baselines(sd):
    wl = _kda_tiny(batch=2, nheads=2, ngroups=2, headdim=24, dstate=32, window=4, steps=16)
    _, worst, worst_emu, _ = _run(wl, "eager", [sd], wl.steps, emulate=True)
    if sd == "f32":
        assert worst[sd] <= 1e-4
    else:
        assert worst_emu[sd] <= (2e-2 if sd == "bf16" else 6e-2), worst_emu


def test_spec_verify_kda():
    wl = I.Workload("kda_spec", "kda", 6, 2, 24, 32, 2, 6, 0, 52, "f32", "f32", max_draft=3, draft_k=3)
    _spec_run(wl, 14, list(range(6)), {"r32": ("replay", "f32"), "rbf": ("replay", "bf16"),
                                       "e32": ("eager", "f32")},
              {"r32": 1e-4, "rbf": 2e-2, "e32": 1e-4})


def test_flush_and_export_match_the_oracle():
    import torch

    wl = _kda_tiny(batch=3, nheads=2, ngroups=2, headdim=32, dstate=64, window=5, steps=0)
    L, _ = make_layer(wl, "replay", "bf16")
    c = I.constants(wl)
    rp = ReplayOracle("kda", c["S0"], wl.window, read_dtype="bf16")
    for t in range(7):  # one fold at step 5, two committed entries left
        tok = I.token(wl, t)
        L.decode(to_device(tok, wl, with_T=False))
        rp.decode(tok)
    torch.cuda.synchronize()
    exp = L.export_state().double().cpu().numpy()
    assert rel_err(exp, rp.export()) <= 1e-5
    L.flush()
    rp.flush()
    sp, ck, pe, fc = L.counters()
    assert np.array_equal(ck, rp.ring.ckpt_pos) and np.array_equal(fc, rp.ring.flush_count)
    assert rel_err(L.export_state().double().cpu().numpy(), rp.export()) <= 1e-5
    tok = I.token(wl, 7)
    y = L.decode(to_device(tok, wl, with_T=False))[:, 0].double().cpu().numpy()
    assert rel_err(y, rp.decode(tok)) <= 2e-3  # same bf16 copy on both sides
    assert L.status()[0] == 0


def test_kda_layer_full_size_sampled():
    """Batch 256 x 32 heads x 128 x 128, W = 16, bf16 read copy and fp32 read path,
    256 steps (16 folds); 16 sequences (first, last, both sides of the halfway and
    quarter marks) at every step against the fp64 oracle, counters exact."""
    wl = I.KDA
    steps = wl.steps
    seqs = [0, 1, 2, 63, 64, 100, 127, 128, 129, 150, 191, 192, 200, 230, 254, 255]
    layers, worst, _, S = _run(wl, "replay", ["bf16", "f32"], steps, seqs=seqs)
    assert worst["bf16"] <= TOL["bf16"], worst
    assert worst["f32"] <= TOL["f32"], worst
    rm = RingModel(wl.batch, wl.window, 1)
    for _ in range(steps):
        rm.decode()
    for L in layers.values():
        sp, ck, pe, fc = L.counters()
        assert np.array_equal(sp, rm.seq_pos) and np.array_equal(ck, rm.ckpt_pos)
        assert np.array_equal(fc, rm.flush_count)
        assert rel_err(L.export_state()[seqs].double().cpu().numpy(), S) <= 1e-5
        assert L.status()[0] == 0
