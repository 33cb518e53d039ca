"""Mamba-2 decode on the GPU against the fp64 CPU oracle.

Tolerances (per step, max |y - y_oracle| <= tol * RMS(y_oracle)): 1e-4 for the
fp32 read path and 2e-2 for the bf16 read copy against the fp64 oracle.  The e4m3
copy's own rounding is larger than any fp8 tolerance against fp64 at these
shapes, so the fp8 path is checked against the oracle that applies the same e4m3
rounding to its checkpoint: the stored codes must agree except for rare one-step
differences where the fp32 and fp64 checkpoints straddle a rounding boundary, and
outputs within 6e-2 * RMS (one such step at a row's largest element moves an
output by up to amax/14 times |C_n|, a few percent of RMS).
"""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from oracle import eager
from oracle.replay import LowPrecEagerOracle, ReplayOracle
from oracle.ring import RingModel
from tests.gpu_common import make_layer, oracle_params, rel_err, to_device

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2, "fp8": 2e-2}


def _run_decode(wl, mode, read_dtypes, steps, seqs=None, dt_scales=False, emulate=False,
                return_emu=False):
    """Decode `steps` tokens with one GPU layer per read dtype; compare every step
    against the fp64 eager oracle (and the emulated-rounding oracles)."""
    import torch

    full = I.constants(wl, f64=False)
    layers = {d: make_layer(wl, mode=mode, state_dtype=d, dt_scales=dt_scales, consts=full)[0]
              for d in read_dtypes}
    del full
    c = I.constants(wl, seqs)
    seqs = list(range(wl.batch)) if seqs is None else list(seqs)
    S = np.ascontiguousarray(c["S0"].copy())
    emu = {}
    if emulate:
        for d in read_dtypes:
            if mode == "replay":
                emu[d] = ReplayOracle("mamba2", c["S0"], wl.window, params=oracle_params(c),
                                      ngroups=wl.ngroups, read_dtype=d, dt_scales_input=dt_scales)
            elif d != "f32":
                emu[d] = LowPrecEagerOracle("mamba2", c["S0"], d, oracle_params(c), wl.ngroups,
                                            dt_scales)
    worst = {d: 0.0 for d in read_dtypes}
    worst_emu = {d: 0.0 for d in read_dtypes}
    for t in range(steps):
        tok = I.token(wl, t)
        dev = to_device(tok, wl, with_T=False)
        ys = {d: L.decode(dev) for d, L in layers.items()}
        sub = {k: v[seqs] for k, v in tok.items()}
        y_ref = eager.mamba2_step(S, c["A"], c["D"], sub["x"], sub["dt"], sub["B"], sub["C"], dt_scales)
        for d, y in ys.items():
            yc = y[seqs, 0].double().cpu().numpy()
            e = rel_err(yc, y_ref)
            worst[d] = max(worst[d], e)
            if d in emu:
                worst_emu[d] = max(worst_emu[d], rel_err(yc, emu[d].decode(sub)))
    torch.cuda.synchronize()
    if return_emu:
        return layers, worst, worst_emu, S, emu
    return layers, worst, worst_emu, S


def test_tiny_replay_and_eager_fp32_match_oracle():
    """Tiny layer (B2 H4 P16 N16 W4, fp32, 32 steps): replay-fp32 and eager-fp32."""
    wl = I.TINY
    for mode in ("replay", "eager"):
        layers, worst, _, S = _run_decode(wl, mode, ["f32"], wl.steps)
        assert worst["f32"] <= 1e-4, (mode, worst)
        L = layers["f32"]
        sp, ck, pe, fc = L.counters()
        rm = RingModel(wl.batch, wl.window, 1, mode=mode)
        for _ in range(wl.steps):
            rm.decode()
        assert sp.tolist() == rm.seq_pos.tolist() and ck.tolist() == rm.ckpt_pos.tolist()
        assert fc.tolist() == rm.flush_count.tolist() and pe.tolist() == rm.pending.tolist()
        exp = L.export_state().double().cpu().numpy()
        assert rel_err(exp, S) <= 1e-5
        assert L.status()[0] == 0


def fp8_codes_match(L, emu_ckpt, shape):
    """The GPU's e4m3 read copy against the oracle's e4m3 rounding of its own (fp64)
    checkpoint: codes may differ only where the fp32 and fp64 checkpoints straddle a
    rounding boundary -- rarely, and then by one e4m3 step."""
    import torch

    from oracle import quant

    Bn, H, P, N = shape
    g_codes = L.region("rc_off", "rc_bytes", torch.uint8).view(torch.float8_e4m3fn).float().view(Bn, H, P, N)
    g_scale = L.region("rc_scale_off", "rc_scale_bytes", torch.float32).view(Bn, H, P)
    o_codes, o_scale = quant.e4m3_rows(emu_ckpt.astype(np.float32))
    g = g_codes.double().cpu().numpy()
    assert np.allclose(g_scale.double().cpu().numpy(), o_scale, rtol=2 ** -20, atol=0)
    diff = g != o_codes
    assert diff.mean() <= 1e-3, diff.mean()
    if diff.any():
        grid = np.sort(np.unique(np.abs(torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
                                        .float().numpy())))
        gi = np.searchsorted(grid, np.abs(g[diff]))
        oi = np.searchsorted(grid, np.abs(o_codes[diff]))
        assert np.all(np.abs(gi - oi) <= 1) and np.all(np.sign(g[diff]) * np.sign(o_codes[diff]) >= 0)


@pytest.mark.parametrize("N,P,W,H,G", [(16, 8, 3, 4, 2), (32, 40, 5, 6, 3), (64, 24, 8, 4, 1),
                                       (128, 72, 2, 2, 2), (128, 64, 16, 8, 1)])
def test_ragged_shapes_all_read_copies(N, P, W, H, G):
    """Rows not a multiple of the rows per pass, 1, 2 or 4 heads per CTA, short windows."""
    wl = I.TINY.replace(batch=3, nheads=H, ngroups=G, headdim=P, dstate=N, window=W, steps=3 * W + 2,
                        seed=11)
    layers, worst, worst_emu, _, emu = _run_decode(wl, "replay", ["f32", "bf16", "fp8"], wl.steps,
                                                   emulate=True, return_emu=True)
    assert worst["f32"] <= TOL["f32"], worst
    assert worst["bf16"] <= TOL["bf16"], worst
    assert worst_emu["bf16"] <= 2e-3, worst_emu
    assert worst_emu["fp8"] <= 6e-2, worst_emu
    fp8_codes_match(layers["fp8"], emu["fp8"].ckpt, (wl.batch, H, P, N))


@pytest.mark.parametrize("sd", ["f32", "bf16", "fp8"])
def test_eager_baselines(sd):
    """Eager read-modify-write with the state stored in fp32, bf16 or fp8 (the single
    shared low-precision state), against fp64 and the emulated-rounding eager oracle."""
    wl = I.TINY.replace(batch=3, nheads=6, ngroups=3, headdim=40, dstate=32, window=4, steps=20,
                        seed=12)
    _, worst, worst_emu, _ = _run_decode(wl, "eager", [sd], wl.steps, emulate=True)
    if sd == "f32":
        assert worst[sd] <= 1e-4
    else:
        assert worst_emu[sd] <= (2e-2 if sd == "bf16" else 6e-2), worst_emu


def test_eager_stream_many_heads_per_cta():
    """The streamed fp32 eager decode at 1 280 heads (about four per CTA of its
    persistent grid, so every shared-memory stage is reused and its mbarrier phase
    flips), 6 steps; six sequences against the fp64 eager oracle, the counters of
    all of them against the plain count."""
    wl = I.TINY.replace(batch=80, nheads=16, ngroups=2, headdim=64, dstate=128, window=4, steps=6, seed=21)
    seqs = [0, 1, 39, 40, 78, 79]
    layers, worst, _, _ = _run_decode(wl, "eager", ["f32"], wl.steps, seqs=seqs)
    assert worst["f32"] <= 1e-4, worst
    sp, ck, pe, fc = layers["f32"].counters()
    assert sp.tolist() == [wl.steps] * wl.batch and ck.tolist() == [wl.steps] * wl.batch


def test_dt_scaled_input_term():
    wl = I.TINY.replace(batch=2, nheads=4, ngroups=2, headdim=16, dstate=16, window=3, steps=12, seed=13)
    for mode in ("replay", "eager"):
        _, worst, _, _ = _run_decode(wl, mode, ["f32"], wl.steps, dt_scales=True)
        assert worst["f32"] <= 1e-4


def test_nemotron_layer_full_size_sampled():
    """Batch 256 x 128 heads x 64 x 128 (4 MiB fp32 state per sequence), W = 16,
    256 steps, bf16 read copy and fp32 read path in the launch configuration the
    benchmark times; outputs of 16 sequences (first, last, both sides of the
    halfway and quarter marks) at every one of the 256 steps against the fp64
    oracle, counters of every sequence against the ring model."""
    wl = I.NEMOTRON
    seqs = [0, 1, 2, 63, 64, 100, 127, 128, 129, 150, 191, 192, 200, 230, 254, 255]
    layers, worst, _, S = _run_decode(wl, "replay", ["bf16", "f32"], wl.steps, seqs=seqs)
    assert worst["bf16"] <= TOL["bf16"], worst
    assert worst["f32"] <= TOL["f32"], worst
    rm = RingModel(wl.batch, wl.window, 1)
    for _ in range(wl.steps):
        rm.decode()
    for L in layers.values():
        sp, ck, pe, fc = L.counters()
        assert np.array_equal(sp, rm.seq_pos) and np.array_equal(ck, rm.ckpt_pos)
        assert np.array_equal(fc, rm.flush_count) and np.array_equal(pe, rm.pending)
        exp = L.export_state()[seqs].double().cpu().numpy()
        assert rel_err(exp, S) <= 1e-5
        assert L.status()[0] == 0
