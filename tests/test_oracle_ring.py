"""Integer ring model against hand-derived golden traces (tests/golden/ring_traces.json)."""
import json
import os

import numpy as np
import pytest

from oracle.ring import MisuseError, RingModel

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "ring_traces.json")))


def _apply(rm, op, arg):
    if op == "decode":
        return rm.decode()
    if op == "verify":
        return rm.verify(arg)
    if op == "commit":
        return rm.commit(arg)
    if op == "flush":
        return rm.flush()
    raise ValueError(op)


def _counters(rm):
    return [[int(rm.seq_pos[b]), int(rm.ckpt_pos[b]), int(rm.pending[b]), int(rm.flush_count[b])]
            for b in range(rm.batch)]


@pytest.mark.parametrize("trace", GOLD["traces"], ids=lambda t: t["name"])
def test_ring_model_matches_golden(trace):
    rm = RingModel(trace["batch"], trace["window"], trace["max_draft"])
    for st in trace["steps"]:
        out = _apply(rm, st["op"], st["arg"])
        assert _counters(rm) == st["after"], st
        if st["op"] in ("decode", "verify"):
            mask, slots = out
            assert mask.tolist() == st["flushed"]
            assert slots.tolist() == st["slots"]
        elif st["op"] == "flush":
            assert out.tolist() == st["flushed"]
        else:
            assert out.tolist() == st["bad"]


@pytest.mark.parametrize("case", GOLD["misuse"], ids=lambda c: c["why"])
def test_ring_model_rejects_misuse(case):
    rm = RingModel(1, 4, 2)
    for s in case["setup"]:
        op, *a = s.split()
        _apply(rm, op, int(a[0]) if a else None)
    op, *a = case["op"].split()
    arg = int(a[0]) if a else ([0] if op == "commit" else None)
    with pytest.raises(MisuseError):
        _apply(rm, op, arg)


def test_plain_decode_flushes_every_W_steps():
    for W in (1, 3, 16, 64):
        rm = RingModel(3, W, 1)
        for t in range(5 * W + 2):
            mask, slots = rm.decode()
            assert mask.all() == (t >= W and t % W == 0) and mask.all() == mask.any()
            assert (slots[:, 0] == t % (W + 1)).all()
        assert (rm.length <= W).all() and (rm.length >= 1).all()


def test_appended_slots_never_hit_entries_being_read():
    """Slots appended by a call never coincide with the committed entries the same
    call may fold or read (so heads sharing a group's B buffer never race)."""
    rng = np.random.default_rng(0)
    for W, K in ((4, 4), (16, 4), (2, 1), (8, 8), (1, 1)):
        rm = RingModel(4, W, K)
        for _ in range(300):
            before = [set(int(rm.slot(n)) for n in range(int(rm.ckpt_pos[b]), int(rm.seq_pos[b])))
                      for b in range(4)]
            if rng.random() < 0.5:
                k = int(rng.integers(1, min(K, W) + 1))
                _, slots = rm.verify(k)
                rm.commit(rng.integers(0, k + 1, 4))
            else:
                _, slots = rm.decode()
            for b in range(4):
                got = set(slots[b].tolist())
                assert len(got) == slots.shape[1]
                assert not (got & before[b])
                assert 0 <= rm.seq_pos[b] - rm.ckpt_pos[b] <= W


def test_eager_mode_keeps_state_current():
    rm = RingModel(2, 4, 2, mode="eager")
    for _ in range(9):
        rm.decode()
    rm.verify(2)
    rm.commit([1, 2])
    assert rm.seq_pos.tolist() == [10, 11] and rm.ckpt_pos.tolist() == [10, 11]
    assert rm.flush_count.tolist() == [0, 0]


def test_page_figures_4mib_state():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))
    s = g["layer_shape"]
    state = s["nheads"] * s["headdim"] * s["dstate"] * s["state_dtype_bytes"]
    assert state == g["state_bytes_per_seq_layer"] == 4 * 2 ** 20
    ratio = state / g["kv_entry_bytes_fp8"]
    assert ratio == 8192 and abs(ratio - g["kv_tokens_equivalent_approx"]) / 8000 < 0.03
