"""Speculative verify + rollback as a buffer-pointer move, on the GPU.

Each round verifies K drafts for every sequence, then commits a per-sequence
accept length a ~ U{0..K}.  The integer bookkeeping (counters, flush schedule,
ring slots) must equal the ring model bit for bit on every sequence; draft
outputs must equal the eager fp64 drafts run from the committed state, and the
committed state must equal the eager state after the accepted tokens.
"""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from oracle import eager
from oracle.ring import RingModel
from tests.gpu_common import make_layer, oracle_params, rel_err, to_device

pytestmark = pytest.mark.gpu


def _spec_run(wl, rounds, seqs, layers_spec, tols):
    import torch

    full = I.constants(wl, f64=False)
    layers = {name: make_layer(wl, mode=mode, state_dtype=sd, consts=full)[0]
              for name, (mode, sd) in layers_spec.items()}
    del full
    c = I.constants(wl, seqs)
    S_ref = np.ascontiguousarray(c["S0"].copy())
    rm = RingModel(wl.batch, wl.window, wl.max_draft)
    K = wl.draft_k
    worst = {n: 0.0 for n in layers}
    for r in range(rounds):
        toks = I.tokens(wl, r * K, K)
        dev = to_device(toks, wl)
        ys = {n: L.verify(K, dev) for n, L in layers.items()}
        S_tmp = S_ref.copy()
        states = []
        for m in range(K):
            tok = {k: v[seqs, m] for k, v in toks.items()}
            y_m = eager.step(wl.kind, S_tmp, tok, oracle_params(c))
            states.append(S_tmp.copy())
            for n, y in ys.items():
                worst[n] = max(worst[n], rel_err(y[seqs, m].double().cpu().numpy(), y_m))
        a = I.accept_lengths(wl, r)
        acc = torch.tensor(a, dtype=torch.int32, device="cuda")
        for L in layers.values():
            L.commit(acc)
        rm.verify(K)
        rm.commit(a)
        for i, b in enumerate(seqs):
            if a[b] > 0:
                S_ref[i] = states[a[b] - 1][i]
    for n, w in worst.items():
        assert w <= tols[n], (n, worst)
    for n, L in layers.items():
        sp, ck, pe, fc = L.counters()
        assert np.array_equal(sp, rm.seq_pos), n
        assert np.array_equal(pe, rm.pending), n
        if layers_spec[n][0] == "replay":
            assert np.array_equal(ck, rm.ckpt_pos) and np.array_equal(fc, rm.flush_count), n
        else:
            assert np.array_equal(ck, rm.seq_pos), n
        assert rel_err(L.export_state()[seqs].double().cpu().numpy(), S_ref) <= 1e-5, n
        assert L.status()[0] == 0
    return layers, rm


def test_spec_verify_mamba2_batch512_k4():
    """Nemotron-scale layer at batch 512, K = 4; replay (bf16 copy, fp32 path) and the
    eager snapshot baseline, all 128 rounds of the workload (many folds per sequence
    at W = 16); floats on 16 sequences, integers on all 512."""
    wl = I.SPECVERIFY
    seqs = list(range(3, 512, 32))  # 16 sequences
    _spec_run(wl, wl.steps, seqs,
              {"replay_bf16": ("replay", "bf16"), "replay_f32": ("replay", "f32"),
               "eager_f32": ("eager", "f32")},
              {"replay_bf16": 2e-2, "replay_f32": 1e-4, "eager_f32": 1e-4})


def test_spec_verify_small_all_k():
    """Every K up to max_draft with tight windows (flush on most verifies) and ragged rows."""
    for K, W in ((1, 1), (2, 2), (3, 4), (8, 8)):
        wl = I.TINY.replace(batch=5, nheads=4, ngroups=2, headdim=16, dstate=32, window=W, steps=0,
                            seed=30 + K, max_draft=K, draft_k=K)
        _spec_run(wl, 12, list(range(5)), {"r32": ("replay", "f32"), "e32": ("eager", "f32")},
                  {"r32": 1e-4, "e32": 1e-4})


def test_spec_verify_gdn():
    wl = I.Workload("gdn_spec", "gdn", 6, 2, 24, 32, 2, 6, 0, 41, "f32", "f32", max_draft=3, draft_k=3)
    _spec_run(wl, 14, list(range(6)), {"r32": ("replay", "f32"), "rbf": ("replay", "bf16"),
                                       "e32": ("eager", "f32")},
              {"r32": 1e-4, "rbf": 2e-2, "e32": 1e-4})


def test_decode_and_short_verifies_on_a_deep_draft_handle():
    """A handle sized for 8 drafts serving plain decodes and verifies of fewer
    drafts (T below the handle's maximum), mixed, across folds: every output
    against the eager fp64 oracle, counters against the ring model."""
    import torch

    wl = I.TINY.replace(batch=3, nheads=4, ngroups=2, headdim=24, dstate=32, window=8, steps=0,
                        seed=61, max_draft=8, draft_k=8, input_dtype="bf16")
    seqs = list(range(wl.batch))
    layers = {n: make_layer(wl, mode="replay", state_dtype=sd)[0] for n, sd in (("f32", "f32"), ("bf16", "bf16"))}
    tols = {"f32": 1e-4, "bf16": 2e-2}
    c = I.constants(wl, seqs)
    S_ref = np.ascontiguousarray(c["S0"].copy())
    rm = RingModel(wl.batch, wl.window, wl.max_draft)
    t = 0
    rng = np.random.default_rng(5)
    for op in ["d", "d", "d", 2, "d", 5, "d", "d", 1, "d", "d", "d", "d", "d", 3, "d", 8, "d"]:
        if op == "d":
            tok = I.token(wl, t); t += 1
            ys = {n: L.decode(to_device(tok, wl, with_T=False)) for n, L in layers.items()}
            y_ref = eager.step(wl.kind, S_ref, tok, oracle_params(c))
            for n, y in ys.items():
                assert rel_err(y[:, 0].double().cpu().numpy(), y_ref) <= tols[n], (n, op)
            rm.decode()
            continue
        K = op
        toks = I.tokens(wl, t, K); t += K
        dev = to_device(toks, wl)
        ys = {n: L.verify(K, dev) for n, L in layers.items()}
        S_tmp = S_ref.copy()
        states = []
        for m in range(K):
            y_m = eager.step(wl.kind, S_tmp, {k: v[:, m] for k, v in toks.items()}, oracle_params(c))
            states.append(S_tmp.copy())
            for n, y in ys.items():
                assert rel_err(y[:, m].double().cpu().numpy(), y_m) <= tols[n], (n, op, m)
        a = rng.integers(0, K + 1, wl.batch).astype(np.int32)
        for L in layers.values():
            L.commit(torch.tensor(a, device="cuda"))
        rm.verify(K)
        rm.commit(a)
        for b in seqs:
            if a[b] > 0:
                S_ref[b] = states[a[b] - 1][b]
    for n, L in layers.items():
        sp, ck, pe, fc = L.counters()
        assert np.array_equal(sp, rm.seq_pos) and np.array_equal(ck, rm.ckpt_pos), n
        assert np.array_equal(fc, rm.flush_count), n
        assert L.status()[0] == 0
