"""rssm_decode_static_scratch: the replay decode with its per-call scratch (the
prep kernel's hand-off to the flush and read kernels) in the library's static
device array, for callers that cannot allocate device memory on the decode
path.  Called through the C ABI.

For every layer kind, a layer decoded with rssm_decode_static_scratch must give
the outputs of an identical layer decoded with rssm_decode (within the fp32
read-path tolerance, 1e-4 x RMS; the kernels are the same, so they are expected
identical) and the same counters, call after call, two calls in a row and on
across two folds.  Two layers of different kinds and shapes take turns on the
shared array, as the layers of a model do.  Oversized layers and eager layers
are refused before anything is enqueued.  This file is collected last, so it
also runs after every other GPU test.
"""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from checkpoint_input_replay_rssm_b200 import rssm
from tests.gpu_common import make_layer, to_device

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _small(kind, **kw):
    base = dict(kind=kind, name=f"{kind}_static_scratch", batch=6, nheads=4, ngroups=2 if kind == "mamba2" else 4,
                headdim=32, dstate=64, window=4, steps=0, seed=71, input_dtype="bf16", max_draft=2, draft_k=2)
    base.update(kw)
    return I.TINY.replace(**base)


def _close(ya, yb):
    import torch

    torch.cuda.synchronize()
    rms = float(ya.double().pow(2).mean().sqrt())
    return float((ya - yb).abs().max()) <= TOL * rms


@pytest.mark.parametrize("state_dtype", ["bf16", "f32", "fp8"])
@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_static_scratch_decode_equals_decode(kind, state_dtype):
    wl = _small(kind)
    A, _ = make_layer(wl, "replay", state_dtype)
    B, _ = make_layer(wl, "replay", state_dtype)
    for t in range(2 * wl.window + 2):  # two calls in a row and more, across two folds
        dev = to_device(I.token(wl, t), wl, with_T=False)
        ya = A.decode(dev)
        yb = B.decode_static_scratch(dev)
        assert _close(ya, yb), t
        for ca, cb in zip(A.counters(), B.counters()):
            assert np.array_equal(ca, cb), t
    assert A.status()[0] == 0 and B.status()[0] == 0
    # the same handle may switch from the static entry point back to the ordinary one
    dev = to_device(I.token(wl, 99), wl, with_T=False)
    assert _close(A.decode(dev), B.decode(dev))


def test_two_layers_of_different_shapes_share_the_array():
    """Layers of different kinds, batch, heads and window (so different carve
    sizes, ring slots and fold schedules) alternate on the array; each matches its
    own twin decoded with rssm_decode, outputs and counters, across folds of all."""
    wa = _small("gdn", batch=5, nheads=6, ngroups=6, window=3, seed=81)
    wb = _small("kda", batch=9, nheads=2, ngroups=2, window=5, headdim=48, dstate=32, seed=82)
    wc = _small("mamba2", batch=7, nheads=8, ngroups=2, window=4, headdim=24, dstate=64, seed=86)
    pairs = []
    for wl in (wa, wb, wc):
        ref, _ = make_layer(wl, "replay", "bf16")
        st, _ = make_layer(wl, "replay", "bf16")
        pairs.append((wl, ref, st))
    for t in range(12):
        for wl, ref, st in pairs:
            dev = to_device(I.token(wl, t), wl, with_T=False)
            y_ref = ref.decode(dev)
            y_st = st.decode_static_scratch(dev)
            assert _close(y_ref, y_st), (wl.kind, t)
            for ca, cb in zip(ref.counters(), st.counters()):
                assert np.array_equal(ca, cb), (wl.kind, t)
    for _, ref, st in pairs:
        assert ref.status()[0] == 0 and st.status()[0] == 0


def test_static_scratch_refuses_oversized_layers_and_eager_layers():
    import torch

    # hand-off of 64 * 256 heads: 4 * (1 + 8 + 128) bytes each = 9 MB > 8 MiB
    big = _small("gdn", batch=64, nheads=256, ngroups=256, headdim=8, dstate=128, window=4, seed=84,
                 max_draft=1, draft_k=0)
    L, _ = make_layer(big, "replay", "bf16")
    n0 = L.launches()
    dev = to_device(I.token(big, 0), big, with_T=False)
    with pytest.raises(rssm.RssmError) as e:
        L.decode_static_scratch(dev)
    assert e.value.status == rssm.RSSM_EINVAL and "static array" in str(e.value)
    assert L.launches() == n0 and L.counters()[0].tolist() == [0] * big.batch
    del L
    torch.cuda.synchronize()

    small = _small("gdn", batch=2, seed=85)
    E, _ = make_layer(small, "eager", "f32")
    with pytest.raises(rssm.RssmError) as e:
        E.decode_static_scratch(to_device(I.token(small, 0), small, with_T=False))
    assert e.value.status == rssm.RSSM_EINVAL
