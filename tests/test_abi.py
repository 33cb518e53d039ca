"""The C-ABI library loads, exports every symbol include/rssm.h declares, and its
host-only logic (validation, workspace layout) behaves -- no GPU needed."""
import ctypes
import os
import re
import subprocess

import pytest

from checkpoint_input_replay_rssm_b200 import build, rssm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rssm.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(build.LIB):
        build.build()
    return rssm.load()


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"RSSM_API\s+[\w\s\*]+?\b(rssm_\w+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("rssm_create", "rssm_decode", "rssm_verify", "rssm_commit", "rssm_flush"):
        assert must in names
    assert set(names) == set(rssm.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (rssm_\w+)", out))
    assert set(_declared()) <= exported
    for n in _declared():
        assert getattr(lib, n) is not None


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "rssm.h"\nint main(void){rssm_config c={0};(void)c;return 0;}\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(tmp_path / "t")])


def _cfg(**kw):
    base = dict(kind="mamba2", mode="replay", state_dtype="bf16", input_dtype="bf16", batch=256,
                nheads=128, headdim=64, dstate=128, ngroups=8, window=16, max_draft=1)
    base.update(kw)
    return rssm.make_config(**base)


def test_workspace_layout_nemotron_scale(lib):
    lay = rssm.rssm_workspace_layout_of(_cfg())
    elems = 256 * 128 * 64 * 128
    assert lay.ckpt_bytes == elems * 4 == 2 ** 30          # 1 GiB fp32 checkpoint
    assert lay.rc_bytes == elems * 2 == 2 ** 29            # 512 MiB bf16 read copy
    assert lay.rc_scale_bytes == 0
    assert lay.ring == 17
    assert lay.xbuf_bytes == 256 * 128 * 17 * 64 * 2
    assert lay.bbuf_bytes == 256 * 8 * 17 * 128 * 2
    assert lay.ring_stride == 20
    assert lay.sbuf_bytes == 256 * 128 * 20 * 4
    offs = sorted((getattr(lay, f), f) for f, _ in lay._fields_ if f.endswith("_off"))
    assert all(o % 256 == 0 for o, _ in offs)
    assert rssm.rssm_workspace_bytes(_cfg()) == lay.total_bytes


def test_workspace_regions_do_not_overlap(lib):
    for kw in (dict(), dict(state_dtype="fp8"), dict(state_dtype="f32"), dict(kind="gdn", nheads=32,
               headdim=128), dict(mode="eager", max_draft=4), dict(mode="eager", state_dtype="fp8",
               max_draft=3), dict(batch=3, nheads=6, ngroups=3, headdim=40, dstate=32, window=5)):
        lay = rssm.rssm_workspace_layout_of(_cfg(**kw))
        spans = []
        for f, _ in lay._fields_:
            if f.endswith("_bytes") and f != "total_bytes" and getattr(lay, f):
                off = getattr(lay, f.replace("_bytes", "_off"))
                spans.append((off, off + getattr(lay, f)))
        spans.sort()
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 <= b0
        assert spans[-1][1] <= lay.total_bytes


def test_fp8_and_eager_layouts(lib):
    lay = rssm.rssm_workspace_layout_of(_cfg(state_dtype="fp8"))
    assert lay.rc_bytes == 256 * 128 * 64 * 128 and lay.rc_scale_bytes == 256 * 128 * 64 * 4
    e = rssm.rssm_workspace_layout_of(_cfg(mode="eager", state_dtype="f32", max_draft=4))
    assert e.ckpt_bytes == 2 ** 30 and e.rc_bytes == 0 and e.xbuf_bytes == 0
    assert e.snap_bytes == 4 * 2 ** 30
    e8 = rssm.rssm_workspace_layout_of(_cfg(mode="eager", state_dtype="fp8", max_draft=0))
    assert e8.ckpt_bytes == 0 and e8.rc_bytes == 2 ** 28 and e8.snap_bytes == 0


@pytest.mark.parametrize("bad", [
    dict(kind=5), dict(dstate=48), dict(dstate=256), dict(headdim=0), dict(headdim=257),
    dict(headdim=20), dict(headdim=7),
    dict(ngroups=3), dict(window=0), dict(window=65), dict(max_draft=9), dict(max_draft=17),
    dict(batch=0), dict(input_dtype="fp8")])
def test_invalid_configs_rejected(lib, bad):
    kw = dict(bad)
    if kw.get("kind") == 5:
        cfg = _cfg()
        cfg.kind = 5
    elif kw.get("input_dtype") == "fp8":
        cfg = _cfg()
        cfg.input_dtype = rssm.RSSM_FP8E4M3
    else:
        cfg = _cfg(**kw)
    assert rssm.rssm_workspace_bytes(cfg) == 0
    with pytest.raises(rssm.RssmError) as ei:
        rssm.rssm_workspace_layout_of(cfg)
    assert ei.value.status == rssm.RSSM_EINVAL


def test_create_validates_before_touching_cuda(lib):
    cfg = _cfg(batch=2, nheads=4, headdim=16, dstate=16, ngroups=1, window=4)
    need = rssm.rssm_workspace_bytes(cfg)
    with pytest.raises(rssm.RssmError) as ei:
        rssm.rssm_create(cfg, None, need, None)
    assert ei.value.status == rssm.RSSM_EINVAL and "NULL" in rssm.rssm_last_error(None)
    with pytest.raises(rssm.RssmError) as ei:
        rssm.rssm_create(cfg, 0x1000, need - 1, None)
    assert ei.value.status == rssm.RSSM_EINVAL and "small" in rssm.rssm_last_error(None)
    with pytest.raises(rssm.RssmError) as ei:
        rssm.rssm_create(cfg, 0x1010, need, None)
    assert "aligned" in rssm.rssm_last_error(None)


def test_null_handle_calls_are_rejected(lib):
    assert lib.rssm_decode(None, None, None) == rssm.RSSM_EINVAL
    assert lib.rssm_flush(None) == rssm.RSSM_EINVAL
    assert lib.rssm_launch_count(None) == -1


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle, and the binding has no CPU path."""
    pkg = os.path.join(ROOT, "checkpoint_input_replay_rssm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "oracle/" not in txt, f


def test_kda_layout_keeps_a_gate_row_per_buffered_token(lib):
    """Kimi Delta Attention: the gate ring holds d_k fp32 per slot ([B][H][R][N]); GDN one
    gate per slot ([B][H][ring_stride]); both keep beta and the swept-query hand-off."""
    kw = dict(nheads=32, headdim=128, dstate=128, ngroups=32)
    g = rssm.rssm_workspace_layout_of(_cfg(kind="gdn", **kw))
    k = rssm.rssm_workspace_layout_of(_cfg(kind="kda", **kw))
    R, Rs = 17, 20
    assert g.sbuf_bytes == 256 * 32 * Rs * 4
    assert k.sbuf_bytes == 256 * 32 * R * 128 * 4
    for lay in (g, k):
        assert lay.tbuf_bytes == 256 * 32 * Rs * 4
        assert lay.query_bytes == 256 * 32 * 1 * 128 * 4
        assert lay.bbuf_bytes == 256 * 32 * R * 128 * 2 and lay.xbuf_bytes == 256 * 32 * R * 128 * 2
    assert k.total_bytes - g.total_bytes >= k.sbuf_bytes - g.sbuf_bytes - 256


def test_kda_config_rules(lib):
    """KDA is validated like GDN: no dt scaling of the input; groups ignored."""
    assert rssm.rssm_workspace_bytes(_cfg(kind="kda", nheads=4, ngroups=3)) > 0
    cfg = _cfg(kind="kda")
    cfg.dt_scales_input = 1
    assert rssm.rssm_workspace_bytes(cfg) == 0
    cfg = _cfg()
    cfg.kind = 3
    assert rssm.rssm_workspace_bytes(cfg) == 0
