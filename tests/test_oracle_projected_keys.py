"""The algebra behind reading a Gated DeltaNet / KDA copy ahead of the backward sweep:
the swept query r is the call's query times the product of all buffered gates minus a
combination of the buffered keys, each times the gates of itself and the older entries,

    r = G_L q - sum_j c_j G_j k_j,   G_j = prod_{i <= j} Diag(alpha_i)   (GDN: scalars),

with c_j the sweep's coefficients, so S r = S (G_L q) - sum_j c_j S (G_j k_j), and
S (G_j k_j) is fixed from the moment entry j is appended until the next fold.  Checked
against the sweep as the replay oracle runs it, and against the closed form of the
recurrence (oracle/closed_form.py), on random heads."""
import numpy as np
import pytest

from oracle import closed_form


def _sweep(q, k, alpha, beta):
    """The backward sweep over entries L-1 .. 0 (newest first): coefficients and r."""
    r = q.copy()
    c = np.zeros(len(k))
    for j in range(len(k) - 1, -1, -1):
        c[j] = beta[j] * (k[j] @ r)
        r = alpha[j] * (r - c[j] * k[j])
    return c, r


@pytest.mark.parametrize("kind", ["gdn", "kda"])
@pytest.mark.parametrize("L", [1, 2, 7, 16])
def test_swept_query_is_gated_query_minus_gated_keys(kind, L):
    rng = np.random.default_rng(100 + L + (0 if kind == "gdn" else 50))
    dk, dv = 12, 9
    S = rng.standard_normal((dv, dk))
    q = rng.standard_normal(dk)
    k = rng.standard_normal((L, dk)) / np.sqrt(dk)
    beta = rng.uniform(0.1, 0.9, L)
    alpha = rng.uniform(0.6, 1.0, (L, dk)) if kind == "kda" else rng.uniform(0.6, 1.0, (L, 1)) * np.ones((1, dk))
    c, r = _sweep(q, k, alpha, beta)
    G = np.cumprod(alpha, axis=0)  # G[j] = alpha_0 * ... * alpha_j (entries j and older)
    r2 = G[-1] * q - sum(c[j] * G[j] * k[j] for j in range(L))
    assert np.allclose(r, r2, rtol=1e-12, atol=1e-12)
    # the output of the copy term, with the projected keys S (G_j k_j) formed ahead of time
    P = np.stack([S @ (G[j] * k[j]) for j in range(L)])
    out = S @ (G[-1] * q) - (c[:, None] * P).sum(axis=0)
    assert np.allclose(out, S @ r, rtol=1e-12, atol=1e-12)
    # and the whole output against the closed form of the recurrence (the last entry is the query's token)
    v = rng.standard_normal((L, dv))
    o_replay = out + (c[:, None] * v).sum(axis=0)
    qs = np.zeros((L, dk))
    qs[-1] = q
    if kind == "kda":
        o_cf, _ = closed_form.kda_one_head(S, qs, k, v, alpha, beta)
    else:
        o_cf, _ = closed_form.gdn_one_head(S, qs, k, v, alpha[:, 0], beta)
    assert np.allclose(o_replay, o_cf[-1], rtol=1e-10, atol=1e-10)


def test_a_dropped_gate_is_caught():
    """Planted mistake: the keys' gates taken from the newer entries instead of the older
    ones fail the identity."""
    rng = np.random.default_rng(7)
    L, dk = 5, 8
    q = rng.standard_normal(dk)
    k = rng.standard_normal((L, dk))
    beta = rng.uniform(0.1, 0.9, L)
    alpha = rng.uniform(0.6, 1.0, (L, dk))
    c, r = _sweep(q, k, alpha, beta)
    Gnew = np.cumprod(alpha[::-1], axis=0)[::-1]  # entries j and newer
    wrong = np.prod(alpha, axis=0) * q - sum(c[j] * Gnew[j] * k[j] for j in range(L))
    assert not np.allclose(r, wrong, rtol=1e-6, atol=1e-6)
