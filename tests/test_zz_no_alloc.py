"""rssm_decode_static_scratch: the replay decode with its per-call hand-off in
the library's static device array, called through the C ABI.

Two handles with the same configuration and state, one decoded with
rssm_decode and one with rssm_decode_static_scratch, must give the same outputs
(within the fp32 read-path tolerance; the kernels are the same, so they are
expected identical) and the same counters, call after call, across folds.
Oversized layers are refused before anything is enqueued.  This file is
collected last so that it also runs after every other GPU test in the session.
"""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from checkpoint_input_replay_rssm_b200 import rssm
from tests.gpu_common import make_layer, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("state_dtype", ["bf16", "f32", "fp8"])
def test_static_scratch_decode_equals_decode(state_dtype):
    import torch

    wl = I.TINY.replace(batch=6, nheads=8, ngroups=2, headdim=40, dstate=64, window=4, steps=0,
                        seed=71, input_dtype="bf16", max_draft=2, draft_k=2)
    A, _ = make_layer(wl, "replay", state_dtype)
    B, _ = make_layer(wl, "replay", state_dtype)
    for t in range(2 * wl.window + 2):  # two calls in a row and more, across two folds
        dev = to_device(I.token(wl, t), wl, with_T=False)
        ya = A.decode(dev)
        yb = B.decode_static_scratch(dev)
        torch.cuda.synchronize()
        rms = float(ya.double().pow(2).mean().sqrt())
        assert float((ya - yb).abs().max()) <= 1e-4 * rms, t
        for ca, cb in zip(A.counters(), B.counters()):
            assert np.array_equal(ca, cb), t
    assert A.status()[0] == 0 and B.status()[0] == 0
    # the two entry points can alternate on one handle
    dev = to_device(I.token(wl, 99), wl, with_T=False)
    ya = A.decode(dev)
    yb = B.decode(dev)
    assert float((ya - yb).abs().max()) <= 1e-4 * float(ya.double().pow(2).mean().sqrt())


def test_static_scratch_refuses_oversized_layers_and_other_kinds():
    import torch

    # hand-off: 16 * 1024 * (64 + 4) * 4 bytes > 4 MiB
    big = I.TINY.replace(batch=16, nheads=1024, ngroups=1, headdim=8, dstate=16, window=64, steps=0,
                         seed=72, input_dtype="bf16", max_draft=1, draft_k=0)
    L, _ = make_layer(big, "replay", "bf16")
    n0 = L.launches()
    dev = to_device(I.token(big, 0), big, with_T=False)
    with pytest.raises(rssm.RssmError) as e:
        L.decode_static_scratch(dev)
    assert e.value.status == rssm.RSSM_EINVAL and "static array" in str(e.value)
    assert L.launches() == n0 and L.counters()[0].tolist() == [0] * big.batch
    del L
    torch.cuda.synchronize()

    small = I.TINY.replace(batch=2, nheads=4, ngroups=2, headdim=16, dstate=16, window=4, steps=0,
                           seed=73, input_dtype="bf16")
    E, _ = make_layer(small, "eager", "f32")
    with pytest.raises(rssm.RssmError) as e:
        E.decode_static_scratch(to_device(I.token(small, 0), small, with_T=False))
    assert e.value.status == rssm.RSSM_EINVAL
