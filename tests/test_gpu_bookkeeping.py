"""Integer bookkeeping and invariants of the device state (bit-exact where integer).

* counters after every op of a random decode/verify/commit/flush sequence equal
  the ring model's, and every live buffered entry sits in slot n mod R holding
  exactly token n's inputs;
* the fp32 checkpoint is byte-identical whatever read copy is kept (rounding of
  the copy never feeds the recurrent update), and a verify that needs no fold
  leaves it untouched;
* flush and export agree; import/export round-trips;
* device-detected misuse sets the error word without trapping; host misuse is
  refused synchronously.
"""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from checkpoint_input_replay_rssm_b200 import rssm
from oracle.ring import RingModel
from tests.gpu_common import make_layer, to_device

pytestmark = pytest.mark.gpu


def _wl(**kw):
    base = dict(batch=4, nheads=4, ngroups=2, headdim=24, dstate=32, window=5, steps=0, seed=50,
                input_dtype="bf16", max_draft=3, draft_k=3)
    base.update(kw)
    return I.TINY.replace(**base)


def _buffer_check(L, wl, rm, history):
    """Every live entry n of every sequence is in slot n mod R with token n's bits."""
    import torch

    R = int(L.layout.ring)
    xb = L.region("xbuf_off", "xbuf_bytes", torch.int16).view(wl.batch, wl.nheads, R, wl.headdim).cpu()
    for b in range(wl.batch):
        for n in rm.live_entries(b):
            want = I.to_torch(history[(b, n)], "bf16").view(torch.int16)
            assert torch.equal(xb[b, :, n % R], want), (b, n)


def test_random_op_sequence_counters_and_slots():
    import torch

    wl = _wl()
    L, _ = make_layer(wl, "replay", "bf16")
    rm = RingModel(wl.batch, wl.window, wl.max_draft)
    rng = np.random.default_rng(0)
    history = {}  # (b, absolute token n) -> x of that token
    t_draw = 0
    for step in range(120):
        op = rng.choice(["decode", "verify", "flush"], p=[0.5, 0.4, 0.1])
        if op == "decode":
            tok = I.token(wl, t_draw); t_draw += 1
            for b in range(wl.batch):
                history[(b, int(rm.seq_pos[b]))] = tok["x"][b]
            L.decode(to_device(tok, wl, with_T=False))
            rm.decode()
        elif op == "verify":
            K = int(rng.integers(1, wl.max_draft + 1))
            toks = I.tokens(wl, t_draw, K); t_draw += K
            for b in range(wl.batch):
                for m in range(K):
                    history[(b, int(rm.seq_pos[b]) + m)] = toks["x"][b, m]
            L.verify(K, to_device(toks, wl))
            rm.verify(K)
            sp, ck, pe, fc = L.counters()
            assert pe.tolist() == rm.pending.tolist()
            _buffer_check(L, wl, rm, history)
            a = rng.integers(0, K + 1, wl.batch)
            L.commit(torch.tensor(a, dtype=torch.int32, device="cuda"))
            rm.commit(a)
        else:
            L.flush()
            rm.flush()
        sp, ck, pe, fc = L.counters()
        assert sp.tolist() == rm.seq_pos.tolist(), step
        assert ck.tolist() == rm.ckpt_pos.tolist(), step
        assert pe.tolist() == rm.pending.tolist(), step
        assert fc.tolist() == rm.flush_count.tolist(), step
        _buffer_check(L, wl, rm, history)
    assert L.status()[0] == 0


def test_checkpoint_identical_across_read_copies_and_untouched_by_verify():
    import torch

    wl = _wl(input_dtype="f32")
    layers = {d: make_layer(wl, "replay", d)[0] for d in ("f32", "bf16", "fp8")}
    t = 0
    for rnd in range(20):
        if rnd % 3 == 2:
            K = 2
            toks = to_device(I.tokens(wl, t, K), wl); t += K
            before = {d: L.region("ckpt_off", "ckpt_bytes", torch.int32).clone() for d, L in layers.items()}
            lens = [L.counters() for L in layers.values()][0]
            no_fold = (lens[0] - lens[1] + K <= wl.window)
            for L in layers.values():
                L.verify(K, toks)
            for d, L in layers.items():
                now = L.region("ckpt_off", "ckpt_bytes", torch.int32).view(wl.batch, -1)
                was = before[d].view(wl.batch, -1)
                for b in range(wl.batch):
                    if no_fold[b]:
                        assert torch.equal(now[b], was[b])
            acc = torch.tensor([1, 0, 2, 1], dtype=torch.int32, device="cuda")
            for L in layers.values():
                L.commit(acc)
        else:
            dev = to_device(I.token(wl, t), wl, with_T=False); t += 1
            for L in layers.values():
                L.decode(dev)
    ck = {d: L.region("ckpt_off", "ckpt_bytes", torch.int32) for d, L in layers.items()}
    assert torch.equal(ck["f32"], ck["bf16"]) and torch.equal(ck["f32"], ck["fp8"])
    assert layers["f32"].counters()[3].min() >= 2  # several folds happened


def test_flush_equals_export_and_import_round_trip():
    import torch

    wl = _wl(input_dtype="f32")
    L, c = make_layer(wl, "replay", "bf16")
    S0 = torch.from_numpy(c["S0"]).cuda()
    assert torch.equal(L.export_state(), S0)  # empty buffer: the checkpoint itself
    for t in range(7):
        L.decode(to_device(I.token(wl, t), wl, with_T=False))
    e1 = L.export_state()
    L.flush()
    sp, ck, _, fc = L.counters()
    assert (sp == ck).all() and (fc == 2).all()  # one fold at token 5 (W = 5), then the flush
    assert torch.equal(L.export_state(), e1)
    assert torch.equal(L.region("ckpt_off", "ckpt_bytes", torch.float32).view_as(e1), e1)
    L.import_state(S0)
    sp, ck, pe, fc = L.counters()
    assert (sp == 0).all() and (ck == 0).all() and (fc == 0).all()
    assert torch.equal(L.export_state(), S0)


def test_device_errors_set_the_error_word_without_trapping():
    import torch

    wl = _wl()
    L, _ = make_layer(wl, "replay", "bf16")
    L.decode(to_device(I.token(wl, 0), wl, with_T=False))
    L.verify(2, to_device(I.tokens(wl, 1, 2), wl))
    L.commit(torch.tensor([1, 3, -1, 2], dtype=torch.int32, device="cuda"))
    st, info = L.status()
    assert st == rssm.RSSM_EDEVICE and info[0] == rssm.RSSM_DEV_BAD_ACCEPT and info[1] in (1, 2)
    sp = L.counters()[0]
    assert sp.tolist() == [2, 1, 1, 3]  # bad accept lengths count as 0
    L.clear_status()
    assert L.status()[0] == 0
    # corrupt sequence 2's counters from the host: seq_pos far beyond the window
    off = L.layout.seq_pos_off
    seq = L.workspace[off:off + 8 * wl.batch].view(torch.int64)
    seq[2] = 1000
    y = torch.full((wl.batch, 1, wl.nheads, wl.headdim), 7.0, device="cuda")
    L.decode(to_device(I.token(wl, 5), wl, with_T=False), y=y)
    st, info = L.status()
    assert st == rssm.RSSM_EDEVICE and info[0] == rssm.RSSM_DEV_BAD_COUNTERS and info[1] == 2
    assert (y[2] == 7.0).all() and not (y[0] == 7.0).all()
    assert L.counters()[0][2] == 1000  # skipped, unchanged


def test_host_misuse_is_refused():
    import torch

    wl = _wl()
    L, _ = make_layer(wl, "replay", "bf16")
    dev1 = to_device(I.token(wl, 0), wl, with_T=False)
    with pytest.raises(rssm.RssmError) as e:
        L.commit(torch.zeros(wl.batch, dtype=torch.int32, device="cuda"))
    assert e.value.status == rssm.RSSM_ESTATE
    with pytest.raises(rssm.RssmError) as e:
        L.verify(4, to_device(I.tokens(wl, 0, 4), wl))
    assert e.value.status == rssm.RSSM_EINVAL
    L.verify(2, to_device(I.tokens(wl, 0, 2), wl))
    for call in (lambda: L.decode(dev1), lambda: L.flush(),
                 lambda: L.verify(1, to_device(I.tokens(wl, 0, 1), wl))):
        with pytest.raises(rssm.RssmError) as e:
            call()
        assert e.value.status == rssm.RSSM_ESTATE
    L.commit(torch.zeros(wl.batch, dtype=torch.int32, device="cuda"))
    L.decode(dev1)
    assert L.status()[0] == 0


def test_flush_kernel_launched_only_when_a_buffer_can_be_full():
    """Plain decode from an empty buffer: the flush kernel runs exactly on the
    calls that find the buffer full (every W-th), so those calls launch one
    kernel more; counters changed behind the library's back so that a fold is
    due when none was scheduled are reported, not silently mis-served."""
    import torch

    wl = _wl()
    W = wl.window
    L, _ = make_layer(wl, "replay", "bf16")
    per_call = []
    for t in range(2 * W + 1):
        l0 = L.launches()
        L.decode(to_device(I.token(wl, t), wl, with_T=False))
        per_call.append(L.launches() - l0)
    fold_calls = [t for t in range(2 * W + 1) if per_call[t] == per_call[0] + 1]
    assert fold_calls == [W, 2 * W], per_call
    assert L.counters()[3].tolist() == [2] * wl.batch
    assert L.status()[0] == 0

    L2, _ = make_layer(wl, "replay", "bf16")
    for t in range(3):
        L2.decode(to_device(I.token(wl, t), wl, with_T=False))
    off = L2.layout.seq_pos_off
    seq = L2.workspace[off:off + 8 * wl.batch].view(torch.int64)
    seq[1] = W  # buffer of sequence 1 now claims W entries
    y = torch.full((wl.batch, 1, wl.nheads, wl.headdim), 7.0, device="cuda")
    L2.decode(to_device(I.token(wl, 3), wl, with_T=False), y=y)
    st, info = L2.status()
    assert st == rssm.RSSM_EDEVICE and info[0] == rssm.RSSM_DEV_BAD_COUNTERS and info[1] == 1
    assert (y[1] == 7.0).all() and not (y[0] == 7.0).all()
    assert L2.counters()[0].tolist() == [4, W, 4, 4]
