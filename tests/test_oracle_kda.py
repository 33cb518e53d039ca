"""Pins of the Kimi Delta Attention oracle (per-channel gate) against facts that do
not come from the oracle itself.

- the eager recurrence (oracle/eager.c) against the brute-force unrolling with
  dense factors Diag(alpha_j) (I - beta_j k_j k_j^T) (oracle/closed_form.py);
- a gate equal on every channel reduces KDA to Gated DeltaNet (the GDN oracle is
  pinned on its own in test_oracle_pins.py);
- beta = 0: pure per-channel decay, o_t = S_0 ((prod_{j<=t} alpha_j) (.) q_t);
- alpha = 1, beta = 1 with orthonormal keys: the write replaces S k by v exactly;
- the replay formulation equals the eager recurrence at every step and window,
  and verify / commit gives the eager state after the committed tokens.
A planted mistake (the gate applied after the delta-rule correction, or a gate
per value row instead of per key channel) must fail a pin.
"""
import numpy as np
import pytest

from oracle import closed_form
from oracle.replay import ReplayOracle
from tests.test_oracle_pins import _gdn_inputs, _rel, eager_gdn


def _kda_inputs(rng, Bn=2, T=6, H=3, P=4, N=5):
    inp = _gdn_inputs(rng, Bn, T, H, P, N)
    inp["alpha"] = np.exp(-np.logaddexp(0, rng.normal(size=(Bn, T, H, N))))
    return inp


def eager_kda(inp):
    from oracle import eager
    S = inp["S0"].copy()
    os_ = []
    for t in range(inp["q"].shape[1]):
        os_.append(eager.kda_step(S, inp["q"][:, t], inp["k"][:, t], inp["v"][:, t],
                                  inp["alpha"][:, t], inp["beta"][:, t]))
    return np.stack(os_, 1), S


def _tok(inp, t):
    return {k: inp[k][:, t] for k in ("q", "k", "v", "alpha", "beta")}


def test_kda_eager_matches_closed_form(oracle_built):
    inp = _kda_inputs(np.random.default_rng(31))
    o_e, S_e = eager_kda(inp)
    o_c, S_c = closed_form.kda(inp["S0"], inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"])
    assert _rel(o_e, o_c) < 1e-12
    assert _rel(S_e, S_c) < 1e-12


def test_kda_uniform_gate_is_gdn(oracle_built):
    rng = np.random.default_rng(32)
    g = _gdn_inputs(rng, 2, 9, 3, 4, 5)
    k = dict(g)
    k["alpha"] = np.repeat(g["alpha"][..., None], 5, axis=-1)
    o_g, S_g = eager_gdn(g)
    o_k, S_k = eager_kda(k)
    assert _rel(o_k, o_g) < 1e-12
    assert _rel(S_k, S_g) < 1e-12


def test_kda_beta_zero_is_per_channel_decay(oracle_built):
    rng = np.random.default_rng(33)
    inp = _kda_inputs(rng, 1, 9, 2, 3, 4)
    inp["beta"][:] = 0.0
    o, S = eager_kda(inp)
    decay = np.cumprod(inp["alpha"][0], axis=0)  # [T,H,N]
    expect = np.einsum("hpn,thn->thp", inp["S0"][0], decay * inp["q"][0])
    assert np.max(np.abs(o[0] - expect)) < 1e-12
    assert np.max(np.abs(S[0] - inp["S0"][0] * decay[-1][:, None, :])) < 1e-12


def test_kda_orthonormal_keys_overwrite_exactly(oracle_built):
    rng = np.random.default_rng(34)
    N = P = 4
    Q, _ = np.linalg.qr(rng.normal(size=(N, N)))
    T = N
    inp = dict(S0=rng.normal(size=(1, 1, P, N)), k=Q.T[None, :, None, :], q=Q.T[None, :, None, :],
               v=rng.normal(size=(1, T, 1, P)), alpha=np.ones((1, T, 1, N)), beta=np.ones((1, T, 1)))
    o, S = eager_kda(inp)
    assert np.max(np.abs(o[0, :, 0] - inp["v"][0, :, 0])) < 1e-12
    assert np.max(np.abs(S[0, 0] - inp["v"][0, :, 0].T @ Q.T)) < 1e-12


@pytest.mark.parametrize("W", [1, 2, 4, 16, 64])
def test_kda_replay_equals_eager_every_step(oracle_built, W):
    rng = np.random.default_rng(40 + W)
    T = 40
    inp = _kda_inputs(rng, 2, T, 3, 4, 5)
    y_e, S_e = eager_kda(inp)
    rp = ReplayOracle("kda", inp["S0"], W)
    for t in range(T):
        y = rp.decode(_tok(inp, t))
        assert _rel(y, y_e[:, t]) < 1e-12, t
    assert _rel(rp.export(), S_e) < 1e-12
    assert np.all(rp.ring.flush_count == (T - 1) // W)


def test_kda_rollback_to_k_equals_eager_after_k(oracle_built):
    from oracle import eager
    rng = np.random.default_rng(41)
    K, W, rounds, Bn = 3, 8, 10, 3
    inp = _kda_inputs(rng, Bn, rounds * K, 3, 4, 5)
    rp = ReplayOracle("kda", inp["S0"], W, K)
    S_ref = inp["S0"].copy()
    for r in range(rounds):
        drafts = {k: inp[k][:, r * K:(r + 1) * K] for k in ("q", "k", "v", "alpha", "beta")}
        y = rp.verify(drafts)
        a = rng.integers(0, K + 1, Bn)
        for b in range(Bn):
            Sb = S_ref[b:b + 1].copy()
            for j in range(K):
                tok = {k: v[b:b + 1, j] for k, v in drafts.items()}
                ye = eager.kda_step(Sb, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
                assert _rel(y[b, j], ye[0]) < 1e-11
                if j + 1 == a[b]:
                    S_ref[b] = Sb[0]
        rp.commit(a)
        assert _rel(rp.export(), S_ref) < 1e-11


class _GateAfterCorrection(ReplayOracle):
    """Planted mistake: Diag(alpha) applied after the delta-rule factor in the sweep."""

    def _read_seq(self, rc, e, q):
        r = q["q"].copy()
        o = np.zeros((self.H, self.P))
        for j in range(e["k"].shape[0] - 1, -1, -1):
            r = e["alpha"][j] * r
            c = e["beta"][j] * np.sum(e["k"][j] * r, axis=1)
            r = r - c[:, None] * e["k"][j]
            o = o + c[:, None] * e["v"][j]
        return o + np.einsum("hpn,hn->hp", rc, r)


def test_kda_pins_catch_a_misplaced_gate(oracle_built):
    rng = np.random.default_rng(42)
    T, W = 12, 4
    inp = _kda_inputs(rng, 2, T, 3, 4, 5)
    y_e, _ = eager_kda(inp)
    rp = _GateAfterCorrection("kda", inp["S0"], W)
    err = max(_rel(rp.decode(_tok(inp, t)), y_e[:, t]) for t in range(T))
    assert err > 1e-3


def test_kda_closed_form_catches_a_value_row_gate(oracle_built):
    """Gating the value rows (Diag(alpha) on the left of S) instead of the key
    channels gives different numbers: the pins would see such a transposition."""
    rng = np.random.default_rng(43)
    inp = _kda_inputs(rng, 1, 5, 1, 5, 5)
    o_e, _ = eager_kda(inp)
    S = inp["S0"][0, 0].copy()
    outs = []
    for t in range(5):
        k, v, al, be = inp["k"][0, t, 0], inp["v"][0, t, 0], inp["alpha"][0, t, 0], inp["beta"][0, t, 0]
        S = np.diag(al) @ S @ (np.eye(5) - be * np.outer(k, k)) + be * np.outer(v, k)
        outs.append(S @ inp["q"][0, t, 0])
    assert _rel(np.array(outs), o_e[0, :, 0]) > 1e-3
