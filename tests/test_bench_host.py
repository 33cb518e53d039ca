"""The end-to-end loop's host-side input packing, on CPU: a step's inputs packed into
one byte buffer at 256-byte offsets and read back as views must be the inputs
themselves, bit for bit, in their dtypes and shapes."""
import numpy as np
import pytest


@pytest.mark.parametrize("input_dtype", ["bf16", "f32"])
def test_packed_inputs_are_the_inputs(input_dtype):
    import torch

    import bench
    from checkpoint_input_replay_rssm_b200 import inputs as I

    wl = I.TINY.replace(batch=3, nheads=6, ngroups=3, headdim=40, dstate=32, input_dtype=input_dtype)
    toks = []
    for t in range(3):
        tok = I.token(wl, t)
        toks.append({k: I.to_torch(v, wl.input_dtype if k in ("x", "B", "C") else "f32").unsqueeze(1).contiguous()
                     for k, v in tok.items()})
    packed, offs, total = bench.pack_inputs(toks, pin=False)
    assert len(packed) == 3 and all(p.numel() == total and p.dtype == torch.uint8 for p in packed)
    assert all(o % 256 == 0 for o in offs.values())
    ends = sorted((o, o + toks[0][k].numel() * toks[0][k].element_size()) for k, o in offs.items())
    assert all(a[1] <= b[0] for a, b in zip(ends, ends[1:])) and ends[-1][1] <= total  # no overlap
    for t in range(3):
        dst = torch.empty(total, dtype=torch.uint8)
        dst.copy_(packed[t])  # the one copy a step makes
        views = bench.input_views(dst, toks[0], offs)
        for k, v in toks[t].items():
            assert views[k].dtype == v.dtype and views[k].shape == v.shape and views[k].is_contiguous()
            assert np.array_equal(views[k].view(-1).view(torch.uint8).numpy(), v.view(-1).view(torch.uint8).numpy())
