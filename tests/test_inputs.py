"""Seeded input generators: determinism, subsets, dtype rounding, distributions."""
import numpy as np
import torch

from checkpoint_input_replay_rssm_b200 import inputs as I


def test_subset_equals_slice_and_is_deterministic():
    wl = I.TINY.replace(batch=5)
    full = I.token(wl, 3)
    sub = I.token(wl, 3, seqs=[1, 4])
    for k in full:
        assert np.array_equal(full[k][[1, 4]], sub[k])
        assert np.array_equal(full[k], I.token(wl, 3)[k])
    c = I.constants(wl)
    assert np.array_equal(I.constants(wl, seqs=[2])["S0"][0], c["S0"][2])


def test_bf16_inputs_are_exact_bf16_values():
    wl = I.NEMOTRON.replace(batch=2)
    tok = I.token(wl, 0)
    for k in ("x", "B", "C"):
        t = torch.from_numpy(tok[k]).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(t, tok[k])
    assert np.array_equal(tok["dt"].astype(np.float32).astype(np.float64), tok["dt"])
    assert tok["x"].shape == (2, 128, 64) and tok["B"].shape == (2, 8, 128)


def test_distributions_roughly_right():
    wl = I.NEMOTRON.replace(batch=4)
    tok = I.token(wl, 1)
    assert abs(tok["x"].std() - 1) < 0.02 and abs(tok["x"].mean()) < 0.02
    assert (tok["dt"] > 0).all() and 0.05 < tok["dt"].mean() < 0.3
    c = I.constants(wl)
    assert (c["A"] < -1 + 1e-6).all() and (c["A"] > -np.e - 1e-6).all()
    assert abs(c["S0"].std() - 0.1) < 0.002
    g = I.token(I.GDN.replace(batch=2), 0)
    assert np.allclose(np.linalg.norm(g["k"], axis=-1), 1, atol=1e-2)
    assert ((g["alpha"] > 0) & (g["alpha"] < 1)).all() and ((g["beta"] > 0) & (g["beta"] < 1)).all()


def test_accept_lengths_in_range():
    a = I.accept_lengths(I.SPECVERIFY, 0)
    assert a.shape == (512,) and a.min() >= 0 and a.max() <= 4
    assert len(np.unique(a)) == 5
