"""The chunked Mamba-2 prefill of oracle/prefill.py against the eager recurrence
(every token's output and the final state, 1e-12), for chunk lengths from 1 to
the whole prompt, with and without dt scaling the input; a planted mistake (the
state at a chunk's start read without its decay) must fail."""
import numpy as np
import pytest

from oracle import prefill
from tests.test_oracle_pins import _m2_inputs, _rel, eager_m2


@pytest.mark.parametrize("chunk", [1, 3, 8, 16, 64])
@pytest.mark.parametrize("dt_scales", [False, True])
def test_chunked_prefill_equals_eager(oracle_built, chunk, dt_scales):
    inp = _m2_inputs(np.random.default_rng(60 + chunk), 2, 40, 4, 3, 5, 2)
    y_e, S_e = eager_m2(inp, dt_scales)
    y_c, S_c = prefill.mamba2(inp["S0"], inp["A"], inp["D"], inp["x"], inp["dt"], inp["B"], inp["C"],
                              chunk, dt_scales)
    assert _rel(y_c, y_e) < 1e-12
    assert _rel(S_c, S_e) < 1e-12


def test_a_missing_start_decay_is_caught(oracle_built, monkeypatch):
    inp = _m2_inputs(np.random.default_rng(70), 1, 24, 2, 3, 4, 1)
    y_e, _ = eager_m2(inp)
    real_exp = np.exp

    def one_head(S0, A_h, D_h, x, dt, Bm, Cm, chunk, dt_scales_input=False):
        T = x.shape[0]
        S = S0.copy()
        y = np.empty((T, x.shape[1]))
        for t0 in range(0, T, chunk):
            t1 = min(T, t0 + chunk)
            lam = np.cumsum(dt[t0:t1] * A_h)
            W = np.tril(real_exp(lam[:, None] - lam[None, :]) * (Cm[t0:t1] @ Bm[t0:t1].T))
            y[t0:t1] = (Cm[t0:t1] @ S.T) + W @ x[t0:t1] + D_h * x[t0:t1]  # decay of S dropped
            S = real_exp(lam[-1]) * S + (x[t0:t1] * real_exp(lam[-1] - lam)[:, None]).T @ Bm[t0:t1]
        return y, S

    monkeypatch.setattr(prefill, "mamba2_one_head", one_head)
    y_c, _ = prefill.mamba2(inp["S0"], inp["A"], inp["D"], inp["x"], inp["dt"], inp["B"], inp["C"], 8)
    assert _rel(y_c, y_e) > 1e-3
