"""The algorithmic-bytes model the benchmark's roofline divides by (traffic.py),
checked against hand counts and against the reports' "about half the state
traffic" (tests/golden/page_figures.json)."""
import json
import os

from checkpoint_input_replay_rssm_b200 import traffic as T

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def _m2(read="bf16"):
    return T.Shape("mamba2", 64, 128, 16, 16, read, "bf16")


def test_read_kernel_bytes_by_hand():
    """A non-folding decode call with L0 committed entries: the read kernel reads the
    copy tile, L0 buffered x rows, the call's x and C (C charged 1/16 per head), the
    coefficient row and the decay, and writes y."""
    L0 = 5
    r = T.replay_step_split(_m2(), L0, False)["read"]
    assert r["copy_read"] == 64 * 128 * 2
    assert r["buffer_read"] == L0 * 64 * 2
    assert r["inputs"] == 64 * 2 + 128 * 2 / 16
    assert r["handoff_read"] == (L0 + 1) * 4 + 4
    assert r["output"] == 64 * 4


def test_fold_bytes_by_hand():
    p = T.replay_step_split(_m2(), 16, True)["prep"]
    assert p["ckpt_read"] == p["ckpt_write"] == 64 * 128 * 4
    assert p["copy_write"] == 64 * 128 * 2


def test_state_traffic_about_half_of_eager():
    """fp32 read path (no copy): the checkpoint is read every step and rewritten once
    per window, about half of eager's read + write every step; the bf16 copy takes
    it to about a third."""
    half = GOLD["traffic_fraction_approx"]
    f32 = T.state_bytes(T.replay_decode_per_token(_m2("f32"))) / T.state_bytes(T.eager_decode_per_token(_m2(), "f32"))
    bf16 = T.state_bytes(T.replay_decode_per_token(_m2("bf16"))) / T.state_bytes(T.eager_decode_per_token(_m2(), "f32"))
    assert abs(f32 - half) < 0.12
    assert bf16 < 0.55 and bf16 < f32


def test_delta_rule_kinds():
    g = T.Shape("gdn", 128, 128, 1, 16, "bf16", "bf16")
    k = T.Shape("kda", 128, 128, 1, 16, "bf16", "bf16")
    rg, rk = T.replay_decode_per_token(g), T.replay_decode_per_token(k)
    # KDA buffers a d_k gate row per token where GDN buffers one gate
    assert T.state_bytes(rk) - T.state_bytes(rg) > 0
    # both hand the swept query (d_k fp32) to the read kernel
    h = T.replay_step_split(g, 3, False)["prep"]["handoff_write"]
    assert h == (3 + 1) * 4 + 4 + 128 * 4
    assert T.eager_decode_per_token(k)["inputs"] - T.eager_decode_per_token(g)["inputs"] == 128 * 4 - 4
