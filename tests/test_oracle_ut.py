"""The chunked (WY / UT) fold of oracle/ut_form.py against the sequential fold of
the replay oracle, for Gated DeltaNet and Kimi Delta Attention: two routes to the
same checkpoint, equal to 1e-12 for buffer lengths 1 .. 64; and a planted mistake
(the system matrix transposed) must break the equality."""
import numpy as np
import pytest

from oracle import ut_form
from oracle.replay import ReplayOracle


def _entries(rng, L, H, P, N, kda):
    k = rng.normal(size=(L, H, N))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a_shape = (L, H, N) if kda else (L, H)
    return dict(k=k, v=rng.normal(size=(L, H, P)),
                alpha=np.exp(-np.logaddexp(0, rng.normal(size=a_shape))),
                beta=1 / (1 + np.exp(-rng.normal(size=(L, H)))))


@pytest.mark.parametrize("kind", ["gdn", "kda"])
@pytest.mark.parametrize("L", [1, 2, 5, 16, 64])
def test_ut_fold_equals_sequential_fold(kind, L):
    rng = np.random.default_rng(100 + L + (7 if kind == "kda" else 0))
    H, P, N = 3, 6, 8
    S = rng.normal(0, 0.3, (H, P, N))
    e = _entries(rng, L, H, P, N, kind == "kda")
    seq = ReplayOracle(kind, S[None], window=64)._fold_seq(S, e)
    ut = ut_form.fold(S, e)
    assert np.max(np.abs(ut - seq)) / np.max(np.abs(seq)) < 1e-12


def test_ut_fold_of_nothing_is_identity():
    S = np.random.default_rng(1).normal(size=(2, 3, 4))
    e = dict(k=np.zeros((0, 2, 4)), v=np.zeros((0, 2, 3)), alpha=np.zeros((0, 2)), beta=np.zeros((0, 2)))
    assert np.array_equal(ut_form.fold(S, e), S)


def test_a_transposed_system_matrix_is_caught(monkeypatch):
    rng = np.random.default_rng(5)
    H, P, N, L = 2, 4, 6, 8
    S = rng.normal(size=(H, P, N))
    e = _entries(rng, L, H, P, N, True)
    seq = ReplayOracle("kda", S[None], window=64)._fold_seq(S, e)
    solve = np.linalg.solve
    monkeypatch.setattr(ut_form.np.linalg, "solve", lambda M, b: solve(M.T, b))
    bad = ut_form.fold(S, e)
    assert np.max(np.abs(bad - seq)) / np.max(np.abs(seq)) > 1e-3
