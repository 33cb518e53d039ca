"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each check compares two independent routes (closed-form unrolling vs the eager
recurrence, textbook special cases, library routines such as numpy.cumsum) so a
dropped term, a wrong sign or index, or a transposed operand in either fails.
"""
import numpy as np
import pytest

from oracle import closed_form, quant
from oracle.replay import ReplayOracle
from oracle.ring import RingModel

rng0 = np.random.default_rng(1234)


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _m2_inputs(rng, Bn=2, T=7, H=4, P=3, N=5, G=2):
    return dict(
        S0=rng.normal(0, 0.3, (Bn, H, P, N)),
        A=-np.exp(rng.uniform(0, 1, H)),
        D=rng.normal(size=H),
        x=rng.normal(size=(Bn, T, H, P)),
        dt=np.logaddexp(0, rng.normal(size=(Bn, T, H)) - 2),
        B=rng.normal(size=(Bn, T, G, N)),
        C=rng.normal(size=(Bn, T, G, N)),
    )


def _gdn_inputs(rng, Bn=2, T=6, H=3, P=4, N=5):
    q = rng.normal(size=(Bn, T, H, N))
    k = rng.normal(size=(Bn, T, H, N))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return dict(
        S0=rng.normal(0, 0.3, (Bn, H, P, N)), q=q, k=k,
        v=rng.normal(size=(Bn, T, H, P)),
        beta=1 / (1 + np.exp(-rng.normal(size=(Bn, T, H)))),
        alpha=np.exp(-np.logaddexp(0, rng.normal(size=(Bn, T, H)))),
    )


def eager_m2(inp, dt_scales=False):
    from oracle import eager
    S = inp["S0"].copy()
    ys = []
    for t in range(inp["x"].shape[1]):
        ys.append(eager.mamba2_step(S, inp["A"], inp["D"], inp["x"][:, t], inp["dt"][:, t],
                                    inp["B"][:, t], inp["C"][:, t], dt_scales))
    return np.stack(ys, 1), S


def eager_gdn(inp):
    from oracle import eager
    S = inp["S0"].copy()
    os_ = []
    for t in range(inp["q"].shape[1]):
        os_.append(eager.gdn_step(S, inp["q"][:, t], inp["k"][:, t], inp["v"][:, t],
                                  inp["alpha"][:, t], inp["beta"][:, t]))
    return np.stack(os_, 1), S


# ----------------------------------------------------------- eager vs closed form
@pytest.mark.parametrize("dt_scales", [False, True])
def test_mamba2_eager_matches_closed_form(oracle_built, dt_scales):
    inp = _m2_inputs(np.random.default_rng(1))
    y_e, S_e = eager_m2(inp, dt_scales)
    y_c, S_c = closed_form.mamba2(inp["S0"], inp["A"], inp["D"], inp["x"], inp["dt"], inp["B"],
                                  inp["C"], dt_scales)
    assert _rel(y_e, y_c) < 1e-12
    assert _rel(S_e, S_c) < 1e-12


def test_gdn_eager_matches_closed_form(oracle_built):
    inp = _gdn_inputs(np.random.default_rng(2))
    o_e, S_e = eager_gdn(inp)
    o_c, S_c = closed_form.gdn(inp["S0"], inp["q"], inp["k"], inp["v"], inp["alpha"],
                               inp["beta"])
    assert _rel(o_e, o_c) < 1e-12
    assert _rel(S_e, S_c) < 1e-12


# ----------------------------------------------------------- degenerate cases
def test_mamba2_unit_decay_one_hot_is_prefix_sum(oracle_built):
    """dt = 0 (a = 1), B_t = e_{n(t)}, C_t = e_m: y_t[p] = S0[p,m] + sum_{i<=t, n(i)=m} x_i[p] + D x_t[p]."""
    rng = np.random.default_rng(3)
    Bn, T, H, P, N, G = 1, 12, 2, 3, 4, 1
    inp = _m2_inputs(rng, Bn, T, H, P, N, G)
    inp["dt"][:] = 0.0
    n_of_t = rng.integers(0, N, T)
    m = 2
    inp["B"][:] = 0.0
    inp["C"][:] = 0.0
    for t in range(T):
        inp["B"][0, t, 0, n_of_t[t]] = 1.0
        inp["C"][0, t, 0, m] = 1.0
    y, _ = eager_m2(inp)
    hit = (n_of_t == m).astype(float)  # [T]
    csum = np.cumsum(hit[:, None, None] * inp["x"][0], axis=0)  # [T,H,P]
    expect = inp["S0"][0][None, :, :, m] + csum + inp["D"][None, :, None] * inp["x"][0]
    assert np.max(np.abs(y[0] - expect)) < 1e-12


def test_mamba2_scalar_geometric_series(oracle_built):
    """P = N = 1, constant a, x, B = C = 1: S_t = a^t S0 + x (1 - a^t) / (1 - a)."""
    T, a, x0, S0, D = 30, 0.8, 0.7, 1.3, 0.25
    A = np.log(a)
    inp = dict(S0=np.full((1, 1, 1, 1), S0), A=np.array([A]), D=np.array([D]),
               x=np.full((1, T, 1, 1), x0), dt=np.ones((1, T, 1)), B=np.ones((1, T, 1, 1)),
               C=np.ones((1, T, 1, 1)))
    y, S = eager_m2(inp)
    t = np.arange(1, T + 1)
    St = a ** t * S0 + x0 * (1 - a ** t) / (1 - a)
    assert np.max(np.abs(y[0, :, 0, 0] - (St + D * x0))) < 1e-12
    assert abs(S[0, 0, 0, 0] - St[-1]) < 1e-12


def test_gdn_orthonormal_keys_overwrite_exactly(oracle_built):
    """alpha = beta = 1 and orthonormal keys: writing (v, k) replaces S k by v exactly."""
    rng = np.random.default_rng(4)
    N = P = 4
    Q, _ = np.linalg.qr(rng.normal(size=(N, N)))
    T = N
    inp = dict(S0=rng.normal(size=(1, 1, P, N)), k=Q.T[None, :, None, :], q=Q.T[None, :, None, :],
               v=rng.normal(size=(1, T, 1, P)), alpha=np.ones((1, T, 1)), beta=np.ones((1, T, 1)))
    o, S = eager_gdn(inp)
    assert np.max(np.abs(o[0, :, 0] - inp["v"][0, :, 0])) < 1e-12
    # all columns rewritten: S = sum_t v_t k_t^T exactly
    assert np.max(np.abs(S[0, 0] - inp["v"][0, :, 0].T @ Q.T)) < 1e-12


def test_gdn_beta_zero_is_pure_decay(oracle_built):
    rng = np.random.default_rng(5)
    inp = _gdn_inputs(rng, 1, 9, 2, 3, 4)
    inp["beta"][:] = 0.0
    o, _ = eager_gdn(inp)
    decay = np.cumprod(inp["alpha"][0], axis=0)  # [T,H]
    expect = decay[:, :, None] * np.einsum("hpn,thn->thp", inp["S0"][0], inp["q"][0])
    assert np.max(np.abs(o[0] - expect)) < 1e-12


# ----------------------------------------------------------- replay == eager
def _tok(inp, t, kind):
    keys = ("x", "dt", "B", "C") if kind == "mamba2" else ("q", "k", "v", "alpha", "beta")
    return {k: inp[k][:, t] for k in keys}


@pytest.mark.parametrize("W", [1, 2, 4, 16, 64])
@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_replay_equals_eager_every_step(oracle_built, kind, W):
    rng = np.random.default_rng(10 + W)
    T = 40
    if kind == "mamba2":
        inp = _m2_inputs(rng, 2, T, 4, 3, 5, 2)
        y_e, S_e = eager_m2(inp)
        rp = ReplayOracle("mamba2", inp["S0"], W, params=dict(A=inp["A"], D=inp["D"]), ngroups=2)
    else:
        inp = _gdn_inputs(rng, 2, T, 3, 4, 5)
        y_e, S_e = eager_gdn(inp)
        rp = ReplayOracle("gdn", inp["S0"], W)
    for t in range(T):
        y = rp.decode(_tok(inp, t, kind))
        assert _rel(y, y_e[:, t]) < 1e-12, t
    assert _rel(rp.export(), S_e) < 1e-12
    assert np.all(rp.ring.flush_count == (T - 1) // W)


@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_rollback_to_k_equals_eager_after_k(oracle_built, kind):
    """verify K drafts, commit a: the committed state equals the eager state after the
    committed tokens, verify outputs equal eager outputs of the drafts, and a verify
    that does not flush leaves the checkpoint untouched."""
    rng = np.random.default_rng(21)
    K, W, rounds = 3, 8, 10
    T = rounds * K
    if kind == "mamba2":
        inp = _m2_inputs(rng, 3, T, 4, 3, 5, 2)
        rp = ReplayOracle("mamba2", inp["S0"], W, K, params=dict(A=inp["A"], D=inp["D"]),
                          ngroups=2)
    else:
        inp = _gdn_inputs(rng, 3, T, 3, 4, 5)
        rp = ReplayOracle("gdn", inp["S0"], W, K)
    from oracle import eager
    S_ref = inp["S0"].copy()
    for r in range(rounds):
        drafts = {k: v[:, r * K:(r + 1) * K] for k, v in inp.items() if v.ndim >= 3 and k != "S0"}
        ck_before = rp.ckpt.copy()
        len_before = rp.ring.length.copy()
        y = rp.verify(drafts)
        no_flush = len_before + K <= W
        assert np.array_equal(rp.ckpt[no_flush], ck_before[no_flush])
        a = rng.integers(0, K + 1, 3)
        for b in range(3):
            Sb = S_ref[b:b + 1].copy()
            for j in range(K):
                tok = {k: v[b:b + 1, j] for k, v in drafts.items()}
                ye = eager.step(kind, Sb, tok, dict(A=inp.get("A"), D=inp.get("D")))
                assert _rel(y[b, j], ye[0]) < 1e-11
                if j + 1 == a[b]:
                    S_ref[b] = Sb[0]
        rp.commit(a)
        assert _rel(rp.export(), S_ref) < 1e-11


def test_checkpoint_independent_of_read_copy(oracle_built):
    """The low-precision copy never feeds the fold: checkpoints are identical."""
    rng = np.random.default_rng(7)
    inp = _m2_inputs(rng, 2, 20, 4, 3, 16, 2)
    ro = {d: ReplayOracle("mamba2", inp["S0"], 4, params=dict(A=inp["A"], D=inp["D"]),
                          ngroups=2, read_dtype=d) for d in ("f64", "f32", "bf16", "fp8")}
    for t in range(20):
        for r in ro.values():
            r.decode(_tok(inp, t, "mamba2"))
    for d in ("f32", "bf16", "fp8"):
        assert np.array_equal(ro["f64"].ckpt, ro[d].ckpt)


# ----------------------------------------------------------- quantisers vs torch
def test_bf16_rne_matches_torch():
    import torch
    x = np.concatenate([rng0.normal(size=100000).astype(np.float32),
                        np.array([0, -0.0, 1, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 3.4e38, 1e-40, -1e-42],
                                 np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(quant.bf16_rne(x).view(np.uint32), ref.view(np.uint32))


def test_e4m3_rne_matches_torch():
    import torch
    grid = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32)
    grid = grid[torch.isfinite(grid)].numpy()
    mids = (np.sort(grid)[1:] + np.sort(grid)[:-1]) / 2  # exact ties
    x = np.concatenate([rng0.normal(0, 40, 200000), rng0.normal(0, 0.01, 50000), grid, mids,
                        np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = quant.e4m3_rne(x)
    assert np.array_equal(got, ref)
    assert quant.e4m3_rne(np.array([500.0, -1e9, 449.0], np.float32)).tolist() == [448, -448, 448]


def test_fp8_rows_scale_and_zero_row():
    S = np.zeros((2, 3, 8), np.float32)
    S[0, 1] = np.linspace(-3, 5, 8)
    codes, scale = quant.e4m3_rows(S)
    assert scale[0, 0] == 1.0 and np.all(codes[0, 0] == 0)
    assert np.isclose(scale[0, 1], np.float32(5.0) / np.float32(448.0))
    assert np.max(np.abs(codes[0, 1])) == 448.0
