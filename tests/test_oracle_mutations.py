"""Planted mistakes in the oracle must fail its pins (all on the CPU).

Each test copies one oracle routine with a plausible bug (a dropped term, an
off-by-one decay index, a wrong sweep order, a transposed operand, an eager
flush rule) and checks that the same comparison the pins make rejects it.
"""
import json
import os

import numpy as np

from oracle import closed_form
from oracle.replay import ReplayOracle
from oracle.ring import RingModel
from tests.test_oracle_pins import _gdn_inputs, _m2_inputs, _rel, _tok, eager_gdn, eager_m2


def test_closed_form_off_by_one_decay_is_caught(oracle_built, monkeypatch):
    def bad(S0, A_h, D_h, x, dt, Bm, Cm, dt_scales_input=False):
        T = x.shape[0]
        a = [np.exp(dt[j] * A_h) for j in range(T)]
        ys = []
        for t in range(T):
            S_t = float(np.prod(a[: t + 1])) * S0
            for i in range(t + 1):
                S_t = S_t + float(np.prod(a[i: t + 1])) * np.outer(x[i], Bm[i])  # a_i too many
            ys.append(S_t @ Cm[t] + D_h * x[t])
        return np.array(ys), S_t

    monkeypatch.setattr(closed_form, "mamba2_one_head", bad)
    inp = _m2_inputs(np.random.default_rng(1))
    y_e, _ = eager_m2(inp)
    y_c, _ = closed_form.mamba2(inp["S0"], inp["A"], inp["D"], inp["x"], inp["dt"], inp["B"],
                                inp["C"])
    assert _rel(y_e, y_c) > 1e-3


class _NoSkip(ReplayOracle):
    def _read_seq(self, rc, e, q):
        return super()._read_seq(rc, e, q) - self.params["D"][:, None] * q["x"]


class _ForwardSweep(ReplayOracle):
    def _read_seq(self, rc, e, q):
        e = {k: v[::-1] for k, v in e.items()}  # applies the delta-rule factors in the wrong order
        return super()._read_seq(rc, e, q)


class _BdotB(ReplayOracle):
    def _read_seq(self, rc, e, q):
        q = dict(q)
        q["C"] = e["B"][-1]  # reads B where C belongs
        return super()._read_seq(rc, e, q)


def _replay_vs_eager(cls, kind, W=4, T=12):
    rng = np.random.default_rng(5)
    if kind == "mamba2":
        inp = _m2_inputs(rng, 2, T, 4, 3, 5, 2)
        y_e, _ = eager_m2(inp)
        rp = cls("mamba2", inp["S0"], W, params=dict(A=inp["A"], D=inp["D"]), ngroups=2)
    else:
        inp = _gdn_inputs(rng, 2, T, 3, 4, 5)
        y_e, _ = eager_gdn(inp)
        rp = cls("gdn", inp["S0"], W)
    return max(_rel(rp.decode(_tok(inp, t, kind)), y_e[:, t]) for t in range(T))


def test_replay_pins_catch_planted_mistakes(oracle_built):
    assert _replay_vs_eager(ReplayOracle, "mamba2") < 1e-12  # the unplanted oracle passes
    assert _replay_vs_eager(_NoSkip, "mamba2") > 1e-3
    assert _replay_vs_eager(_BdotB, "mamba2") > 1e-3
    assert _replay_vs_eager(_ForwardSweep, "gdn") > 1e-3


class _FullOnlyRing(RingModel):
    def _flush_mask(self, n_new):  # ignores how many tokens are about to be appended
        return self.length >= self.W


class _FlushWhenFilledRing(RingModel):
    def _flush_mask(self, n_new):  # folds as soon as the append would fill the buffer
        return self.length + n_new >= self.W


def test_ring_golden_catches_flush_rule_changes():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "ring_traces.json")))
    for cls in (_FullOnlyRing, _FlushWhenFilledRing):
        mismatch = False
        for tr in g["traces"]:
            rm = cls(tr["batch"], tr["window"], tr["max_draft"])
            for st in tr["steps"]:
                op, arg = st["op"], st["arg"]
                getattr(rm, op)(*([] if arg is None else [arg]))
                got = [[int(rm.seq_pos[b]), int(rm.ckpt_pos[b]), int(rm.pending[b]),
                        int(rm.flush_count[b])] for b in range(rm.batch)]
                mismatch |= got != st["after"]
        assert mismatch, cls.__name__
