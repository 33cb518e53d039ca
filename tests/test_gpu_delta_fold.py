"""The Gated DeltaNet and Kimi Delta Attention decode fold at d_k = d_v = 128
against the fp64 CPU oracle: windows from 1 to 32 entries (ragged lengths
included), both input dtypes, every read copy, buffers of different lengths
folding on different calls, and the read copy checked bit for bit against the
rounding of the fp32 checkpoint.

The low-precision copies are compared with the oracle's emulated copy (the
rounding of its fp64 checkpoint).  An fp32 checkpoint within eps of the fp64
one rounds to the neighbouring bf16 code in about 2 eps / 2^-8 of its elements,
and one such code moves an output by up to 2^-7 |S||r|, about 3e-3 x RMS for an
element and query entry at three standard deviations over 128 channels; the
bf16 bound, 5e-3, allows one or two such flips over a run.  That the copy is
exactly the rounding of the checkpoint is checked bit for bit by
test_read_copy_is_the_rounded_checkpoint_after_folds."""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from oracle import eager
from oracle.replay import ReplayOracle
from oracle.ring import RingModel
from tests.gpu_common import make_layer, rel_err, to_device

pytestmark = pytest.mark.gpu


def _wl(kind, W, input_dtype, batch=3, nheads=2):
    return I.Workload(name=f"{kind}_fold_w{W}", kind=kind, batch=batch, nheads=nheads, headdim=128, dstate=128,
                      ngroups=nheads, window=W, steps=3 * W + 2, seed=400 + W, read_dtype="f32",
                      input_dtype=input_dtype)


def _run(wl, dtypes):
    import torch

    full = I.constants(wl, f64=False)
    layers = {d: make_layer(wl, mode="replay", state_dtype=d, consts=full)[0] for d in dtypes}
    c = I.constants(wl)
    S = np.ascontiguousarray(c["S0"].copy())
    emu = {d: ReplayOracle(wl.kind, c["S0"], wl.window, read_dtype=d) for d in dtypes}
    step = eager.kda_step if wl.kind == "kda" else eager.gdn_step
    worst = {d: 0.0 for d in dtypes}
    worst_emu = {d: 0.0 for d in dtypes}
    for t in range(wl.steps):
        tok = I.token(wl, t)
        dev = to_device(tok, wl, with_T=False)
        ys = {d: L.decode(dev) for d, L in layers.items()}
        o_ref = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        for d, y in ys.items():
            yc = y[:, 0].double().cpu().numpy()
            worst[d] = max(worst[d], rel_err(yc, o_ref))
            worst_emu[d] = max(worst_emu[d], rel_err(yc, emu[d].decode(tok)))
    torch.cuda.synchronize()
    return layers, worst, worst_emu, S


@pytest.mark.parametrize("kind", ["gdn", "kda"])
@pytest.mark.parametrize("W", [1, 5, 13, 16, 17, 27, 32])
def test_fold_all_read_copies(kind, W):
    wl = _wl(kind, W, "bf16")
    layers, worst, worst_emu, S = _run(wl, ["f32", "bf16", "fp8"])
    assert worst["f32"] <= 1e-4, worst
    assert worst["bf16"] <= 2e-2, worst
    assert worst_emu["bf16"] <= 5e-3, worst_emu
    assert worst_emu["fp8"] <= 6e-2, worst_emu
    exp = layers["f32"].export_state().double().cpu().numpy()
    assert rel_err(exp, S) <= 1e-4
    sp, ck, pe, fc = layers["f32"].counters()
    rm = RingModel(wl.batch, W, 1)
    for _ in range(wl.steps):
        rm.decode()
    assert sp.tolist() == rm.seq_pos.tolist() and ck.tolist() == rm.ckpt_pos.tolist()
    assert fc.tolist() == rm.flush_count.tolist()
    for L in layers.values():
        assert L.status()[0] == 0


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_fold_fp32_inputs(kind):
    wl = _wl(kind, 16, "f32")
    _, worst, worst_emu, _ = _run(wl, ["f32", "bf16"])
    assert worst["f32"] <= 1e-4, worst
    assert worst_emu["bf16"] <= 5e-3, worst_emu


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_fold_with_staggered_buffers(kind):
    """Sequences whose buffers fold on different calls: one verify of 4 drafts
    with accept lengths 0..4 leaves the buffers at different lengths, so every
    later fold call serves some sequences from the fold kernel and leaves the
    rest to the read kernel.  Compared with the oracle's bf16 read copy."""
    import torch

    wl = _wl(kind, 16, "bf16", batch=10)
    full = I.constants(wl, f64=False)
    layer = make_layer(wl, mode="replay", state_dtype="bf16", max_draft=4, consts=full)[0]
    c = I.constants(wl)
    orc = ReplayOracle(kind, c["S0"], wl.window, max_draft=4, read_dtype="bf16")
    toks = I.tokens(wl, 0, 4)
    y = layer.verify(4, to_device(toks, wl))
    worst = rel_err(y.double().cpu().numpy(), orc.verify(toks))
    accept = np.arange(wl.batch, dtype=np.int32) % 5
    layer.commit(torch.from_numpy(accept).cuda())
    orc.commit(accept)
    for t in range(4, 44):
        tok = I.token(wl, t)
        y = layer.decode(to_device(tok, wl, with_T=False))[:, 0].double().cpu().numpy()
        worst = max(worst, rel_err(y, orc.decode(tok)))
    torch.cuda.synchronize()
    assert worst <= 5e-3, worst
    sp, ck, pe, fc = layer.counters()
    assert sp.tolist() == orc.ring.seq_pos.tolist() and ck.tolist() == orc.ring.ckpt_pos.tolist()
    assert fc.tolist() == orc.ring.flush_count.tolist()
    assert layer.status()[0] == 0


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_read_copy_is_the_rounded_checkpoint_after_folds(kind):
    """After several folds the read copy equals the rounding of the
    fp32 checkpoint, bit for bit: bf16 round-to-nearest-even, and for fp8 the
    per-row scale amax / 448 (correctly rounded) with e4m3(value / scale)
    (torch's casts, which the oracle's quantisers are pinned to)."""
    import torch

    wl = _wl(kind, 16, "bf16", batch=4)
    full = I.constants(wl, f64=False)
    layers = {d: make_layer(wl, mode="replay", state_dtype=d, consts=full)[0] for d in ("bf16", "fp8")}
    for t in range(3 * wl.window + 5):
        dev = to_device(I.token(wl, t), wl, with_T=False)
        for L in layers.values():
            L.decode(dev)
    torch.cuda.synchronize()
    rows = wl.batch * wl.nheads * wl.headdim
    L = layers["bf16"]
    ck = L.region("ckpt_off", "ckpt_bytes", torch.float32).view(rows, wl.dstate)
    rc = L.region("rc_off", "rc_bytes", torch.int16).view(rows, wl.dstate)
    assert torch.equal(ck.to(torch.bfloat16).view(torch.int16), rc)
    L = layers["fp8"]
    ck = L.region("ckpt_off", "ckpt_bytes", torch.float32).view(rows, wl.dstate)
    rc = L.region("rc_off", "rc_bytes", torch.uint8).view(rows, wl.dstate)
    sc = L.region("rc_scale_off", "rc_scale_bytes", torch.float32).view(rows)
    amax = ck.abs().amax(dim=1)
    # a tensor divisor: torch turns division by a Python scalar into a product
    # with its reciprocal, which is not the correctly rounded quotient
    want_sc = torch.where(amax > 0, amax / torch.full_like(amax, 448.0), torch.ones_like(amax))
    assert torch.equal(sc, want_sc)
    codes = (ck / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(codes, rc)
    for L in layers.values():
        assert L.status()[0] == 0
