"""Pins of the oracle's low-precision side: the read-copy quantisers
(oracle/quant.py: read_copy, e4m3_rows, dequant_e4m3_rows) and the single
low-precision-state eager comparator (oracle/replay.py: LowPrecEagerOracle).

The reports keep an fp32 checkpoint for the recurrent update and read outputs
from a low-precision copy of it, so the copy's rounding never feeds back
(irisproject.cloud, "Deux precisions pour le prix d'une"); the comparator is the
single shared low-precision state whose rounding does feed back
(blog.thibaultmonteiro.fr, "Trois ennuis nes de la meme fusion").  Neither page
fixes a format; the readings (bf16 RNE of the fp32 value; e4m3fn RNE with one
fp32 scale amax/448 per state row, value/scale and code*scale in fp32) are
pinned here against facts that do not come from the oracle:

* torch's own CPU casts (bfloat16, float8_e4m3fn) applied to the fp32-rounded
  state, including values where rounding the fp64 value directly differs;
* exact round trips for rows on the e4m3 grid with a power-of-two scale;
* the format's error bound (half an ulp of a 3-bit mantissa, half the
  subnormal step) element by element;
* the eager recurrence itself when the copy is exact, and integer prefix sums
  (a = 1, one-hot B and C) that every format holds exactly.

Each pin is also run against a planted mistake in the oracle (a dequantiser
that divides by the scale, a quantiser fed the fp64 value instead of the fp32
checkpoint, a comparator that reads its output back from the requantised
state) and must fail there.
"""
import numpy as np
import pytest

from oracle import quant
from oracle.replay import LowPrecEagerOracle

torch = pytest.importorskip("torch")


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _e4m3_grid() -> np.ndarray:
    g = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    g = g[torch.isfinite(g)].numpy()
    return np.unique(g)


def _torch_bf16(S64: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(S64, np.float64)).float().bfloat16().double().numpy()


def _torch_fp8_rows(S64: np.ndarray) -> np.ndarray:
    """Per-row scaled e4m3 copy computed with torch only: fp32 state, fp32 amax/448
    (1 for an all-zero row), torch's e4m3fn cast of value/scale, code * scale."""
    s32 = torch.from_numpy(np.asarray(S64, np.float64)).float()
    amax = s32.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / torch.tensor(448.0, dtype=torch.float32),
                        torch.ones_like(amax))
    codes = (s32 / scale[..., None]).to(torch.float8_e4m3fn).float()
    return (codes * scale[..., None]).double().numpy()


def _tricky_state(rng) -> np.ndarray:
    """fp64 state rows, some of whose values sit just off a bf16 rounding tie in
    fp64 but exactly on it once rounded to fp32 (so rounding the fp64 value
    directly gives another bf16 value), and rows of mixed magnitude with an
    all-zero row (scale 1) for the fp8 copy."""
    S = rng.normal(0, 1, (3, 4, 6, 16))
    S[0, 0, 0] = 0.0
    S[1, 2] *= 1e-3
    S[2, 3] *= 50.0
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 2 + 2 ** -7, -(1.5 + 2 ** -9)])
    S[0, 1, 0, :4] = ties + np.sign(ties) * 2 ** -30  # above the tie in fp64, the tie in fp32
    S[0, 1, 1, :4] = ties - np.sign(ties) * 2 ** -30  # below the tie in fp64, the tie in fp32
    return S


# ------------------------------------------------------------------ the pins
def check_read_copy_matches_torch():
    S = _tricky_state(np.random.default_rng(5))
    assert np.array_equal(quant.read_copy(S, "f32"), S.astype(np.float32).astype(np.float64))
    assert np.array_equal(quant.read_copy(S, "bf16"), _torch_bf16(S))
    assert np.array_equal(quant.read_copy(S, "fp8"), _torch_fp8_rows(S))


def check_fp8_round_trip_on_grid():
    rng = np.random.default_rng(6)
    grid = _e4m3_grid()
    rows = rng.choice(np.concatenate([grid, -grid]), size=(64, 32))
    rows[:, rng.integers(0, 32, 64)] = 0.0
    rows[np.arange(64), rng.integers(0, 32, 64)] = rng.choice([448.0, -448.0], 64)  # row maximum
    S = rows * np.ldexp(1.0, rng.integers(-20, 12, 64))[:, None]  # power-of-two scales
    codes, scale = quant.e4m3_rows(S.astype(np.float32))
    assert np.array_equal(quant.dequant_e4m3_rows(codes, scale), S)
    assert np.array_equal(quant.read_copy(S, "fp8"), S)


def check_fp8_error_bound():
    rng = np.random.default_rng(7)
    S = rng.standard_t(3, size=(40, 8, 128)) * np.exp(rng.uniform(-8, 8, (40, 8, 1)))
    S[0, 0] = 0.0
    s32 = S.astype(np.float32).astype(np.float64)
    codes, scale = quant.e4m3_rows(S.astype(np.float32))
    deq = quant.dequant_e4m3_rows(codes, scale)
    sc = scale.astype(np.float64)[..., None]
    # half an ulp of a 3-bit mantissa, half the subnormal step 2^-9 (in scaled
    # units), and the two fp32 roundings (value/scale and code*scale)
    bound = 2.0 ** -4 * np.abs(s32) + 2.0 ** -10 * sc + 2.0 ** -20 * np.abs(s32)
    assert np.all(np.abs(deq - s32) <= bound)
    assert np.all(np.abs(codes) <= 448.0)
    # the row maximum maps to +-448 (up to the fp32 division's rounding)
    big = np.max(np.abs(codes), axis=-1)
    assert np.all((big == 448.0) | (np.max(np.abs(s32), axis=-1) == 0))


def _m2_case(rng, Bn=2, H=4, P=3, N=8, G=2, T=12):
    return dict(
        S0=rng.normal(0, 0.3, (Bn, H, P, N)),
        A=-np.exp(rng.uniform(0, 1, H)), D=rng.normal(size=H),
        toks=[dict(x=rng.normal(size=(Bn, H, P)), dt=np.logaddexp(0, rng.normal(size=(Bn, H)) - 2),
                   B=rng.normal(size=(Bn, G, N)), C=rng.normal(size=(Bn, G, N))) for _ in range(T)],
    )


def _delta_case(rng, kind, Bn=2, H=3, P=4, N=8, T=12):
    toks = []
    for _ in range(T):
        q = rng.normal(size=(Bn, H, N))
        k = rng.normal(size=(Bn, H, N))
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        gshape = (Bn, H, N) if kind == "kda" else (Bn, H)
        toks.append(dict(q=q, k=k, v=rng.normal(size=(Bn, H, P)),
                         alpha=np.exp(-np.logaddexp(0, rng.normal(size=gshape))),
                         beta=1 / (1 + np.exp(-rng.normal(size=(Bn, H))))))
    return dict(S0=rng.normal(0, 0.3, (Bn, H, P, N)), toks=toks)


def _case(kind, seed):
    rng = np.random.default_rng(seed)
    return _m2_case(rng) if kind == "mamba2" else _delta_case(rng, kind)


def _run_eager(kind, case):
    from oracle import eager
    S = np.array(case["S0"], np.float64)
    params = dict(A=case.get("A"), D=case.get("D"))
    ys, Ss = [], []
    for tok in case["toks"]:
        ys.append(eager.step(kind, S, tok, params))
        Ss.append(S.copy())
    return ys, Ss


def _run_lowprec(kind, case, dtype):
    lp = LowPrecEagerOracle(kind, case["S0"], dtype, params=dict(A=case.get("A"), D=case.get("D")),
                            ngroups=2)
    ys, Ss = [], []
    for tok in case["toks"]:
        ys.append(lp.decode(tok))
        Ss.append(lp.S.copy())
    return ys, Ss


def check_lowprec_exact_copy_is_eager(kind):
    case = _case(kind, 11)
    ye, Se = _run_eager(kind, case)
    yl, Sl = _run_lowprec(kind, case, "f64")
    for t in range(len(ye)):
        assert _rel(yl[t], ye[t]) <= 1e-12 and _rel(Sl[t], Se[t]) <= 1e-12, t


def check_lowprec_fp32_within_rounding(kind):
    case = _case(kind, 12)
    ye, Se = _run_eager(kind, case)
    yl, Sl = _run_lowprec(kind, case, "f32")
    for t in range(len(ye)):
        assert np.array_equal(Sl[t], Sl[t].astype(np.float32).astype(np.float64)), t  # stored in fp32
        assert _rel(Sl[t], Se[t]) <= 1e-6 and _rel(yl[t], ye[t]) <= 1e-6, t
        # and it does round: the state is not the exact one
    assert max(_rel(Sl[t], Se[t]) for t in range(len(ye))) > 1e-9


def check_lowprec_output_from_unrounded_update(kind, dtype):
    """From a state already on the format's grid the first output is the exact
    eager output (the output is taken from the updated value before it is
    requantised), and the stored state is the torch rounding of the exact one."""
    case = _case(kind, 13)
    S0 = _torch_bf16(case["S0"]) if dtype == "bf16" else _torch_fp8_rows(case["S0"])
    case = dict(case, S0=S0)
    ye, Se = _run_eager(kind, case)
    yl, Sl = _run_lowprec(kind, case, dtype)
    assert _rel(yl[0], ye[0]) <= 1e-12
    ref = _torch_bf16(Se[0]) if dtype == "bf16" else _torch_fp8_rows(Se[0])
    assert np.array_equal(Sl[0], ref)
    # the rounding really is visible in this case (so the first check can fail)
    assert _rel(ref, Se[0]) > 1e-5


def check_lowprec_prefix_sums_exact(dtype):
    """Mamba-2 with a = 1 (dt = 0), one-hot B_t = e_{n(t)} and C_t = e_{m(t)}, small
    integer x: the state stays integer, y_t[p] = S_0[p, m] + sum_{i<=t, n(i)=m} x_i[p]
    + D x_t[p] (numpy cumsum), and every format holds it exactly.  For the fp8
    copy column 0 of every row holds 14 and is never written, so each row's scale
    is 14/448 = 2^-5 and the integers -14..14 are on the scaled e4m3 grid."""
    rng = np.random.default_rng(14)
    Bn, H, P, N, G, T = 2, 4, 3, 8, 2, 12
    S0 = rng.integers(-2, 3, (Bn, H, P, N)).astype(np.float64)
    S0[..., 0] = 14.0
    A = -np.exp(rng.uniform(0, 1, H))
    D = rng.integers(-2, 3, H).astype(np.float64)
    nsel = rng.integers(1, N, (T, Bn, G))
    msel = rng.integers(0, N, (T, Bn, G))
    xs = rng.integers(-1, 2, (T, Bn, H, P)).astype(np.float64)
    lp = LowPrecEagerOracle("mamba2", S0, dtype, params=dict(A=A, D=D), ngroups=G)
    hg = H // G
    for t in range(T):
        Bm = np.zeros((Bn, G, N))
        Cm = np.zeros((Bn, G, N))
        for b in range(Bn):
            for g in range(G):
                Bm[b, g, nsel[t, b, g]] = 1.0
                Cm[b, g, msel[t, b, g]] = 1.0
        y = lp.decode(dict(x=xs[t], dt=np.zeros((Bn, H)), B=Bm, C=Cm))
        for b in range(Bn):
            for h in range(H):
                g = h // hg
                m = msel[t, b, g]
                hits = np.array([nsel[i, b, g] == m for i in range(t + 1)], np.float64)
                ref = (S0[b, h, :, m] + np.cumsum(hits[:, None] * xs[: t + 1, b, h], axis=0)[-1]
                       + D[h] * xs[t, b, h])
                assert np.array_equal(y[b, h], ref), (t, b, h)


# ------------------------------------------------------------------ tests
def test_read_copy_matches_torch_casts():
    check_read_copy_matches_torch()


def test_fp8_rows_round_trip_exactly_on_grid():
    check_fp8_round_trip_on_grid()


def test_fp8_rows_error_within_format_bound():
    check_fp8_error_bound()


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_lowprec_oracle_with_exact_copy_is_eager(oracle_built, kind):
    check_lowprec_exact_copy_is_eager(kind)


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_lowprec_oracle_fp32_state_within_rounding(oracle_built, kind):
    check_lowprec_fp32_within_rounding(kind)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_lowprec_oracle_outputs_the_unrounded_update(oracle_built, kind, dtype):
    check_lowprec_output_from_unrounded_update(kind, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "fp8"])
def test_lowprec_oracle_integer_prefix_sums(oracle_built, dtype):
    check_lowprec_prefix_sums_exact(dtype)


# ------------------------------------------------------------------ planted mistakes
def _dequant_divides(codes, scale):
    return (codes.astype(np.float32) / np.asarray(scale, np.float32)[..., None]).astype(
        np.float32).astype(np.float64)


def _bf16_of_f64(v):
    """Round the fp64 value itself to 8 significant bits (no fp32 step)."""
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def _read_copy_from_f64(S, dtype):
    """read_copy that quantises the fp64 state instead of the fp32 checkpoint."""
    S = np.asarray(S, np.float64)
    if dtype == "bf16":
        return _bf16_of_f64(S)
    if dtype == "fp8":
        amax = np.max(np.abs(S), axis=-1)
        scale = np.where(amax > 0, amax / 448.0, 1.0)
        codes = quant.e4m3_rne(S / scale[..., None])
        return codes * scale[..., None]
    return np.array(S, copy=True)


def test_planted_dequant_by_reciprocal_scale_is_caught(monkeypatch, oracle_built):
    monkeypatch.setattr(quant, "dequant_e4m3_rows", _dequant_divides)
    for check in (check_read_copy_matches_torch, check_fp8_round_trip_on_grid, check_fp8_error_bound,
                  lambda: check_lowprec_prefix_sums_exact("fp8"),
                  lambda: check_lowprec_output_from_unrounded_update("gdn", "fp8")):
        with pytest.raises(AssertionError):
            check()


def test_planted_quantising_the_fp64_value_is_caught(monkeypatch, oracle_built):
    monkeypatch.setattr(quant, "read_copy", _read_copy_from_f64)
    with pytest.raises(AssertionError):
        check_read_copy_matches_torch()
    with pytest.raises(AssertionError):
        check_lowprec_output_from_unrounded_update("mamba2", "fp8")
    # the bf16 difference comes only from the values that sit off a tie in fp64
    S = _tricky_state(np.random.default_rng(5))
    assert not np.array_equal(_read_copy_from_f64(S, "bf16"), _torch_bf16(S))


def test_planted_output_from_requantised_state_is_caught(monkeypatch, oracle_built):
    from oracle import eager

    def decode_rounded_output(self, tok):
        S = np.ascontiguousarray(self.S.copy())
        eager.step(self.kind, S, tok, self.params, self.dt_scales_input)
        self.S = quant.read_copy(S, self.dtype)
        # mistake: the output read back from the requantised state
        S2 = np.ascontiguousarray(self.S.copy())
        zero = {k: (np.zeros_like(v) if k in ("x", "v", "beta") else
                    (np.ones_like(v) if k == "alpha" else v)) for k, v in tok.items()}
        if self.kind == "mamba2":
            zero["dt"] = np.zeros_like(tok["dt"])
        return eager.step(self.kind, S2, zero, self.params, self.dt_scales_input)

    monkeypatch.setattr(LowPrecEagerOracle, "decode", decode_rounded_output)
    for kind in ("mamba2", "gdn"):
        with pytest.raises(AssertionError):
            check_lowprec_output_from_unrounded_update(kind, "bf16")
    with pytest.raises(AssertionError):
        check_lowprec_output_from_unrounded_update("kda", "fp8")
