"""Mamba-2 prompt prefill on the tensor cores (rssm_mamba2_prefill) against the
chunked fp64 prefill of oracle/prefill.py, itself pinned to the eager
recurrence.

Tolerance 1e-4 x RMS (the fp32 read path's): per prompt token, max over the
outputs |y - y_oracle| <= 1e-4 x RMS(y_oracle at that token), and the state after
the prompt within 1e-4 x RMS(state).  The kernel's operands are bf16 (x, B, C
exactly; the fp32 ones as a two-part split), so this checks that the split
keeps near-fp32 accuracy through every chunk.  Ragged prompts (a partial last
chunk), one-token prompts, several head sizes, dt scaling the input, a zero
initial state, the hand-off into replay decode (rssm_import_state, then decode
steps against the eager oracle), the full-size launch on sampled sequences,
and refused sizes.
"""
import numpy as np
import pytest

from checkpoint_input_replay_rssm_b200 import inputs as I
from checkpoint_input_replay_rssm_b200 import rssm
from oracle import eager, prefill as oprefill
from tests.gpu_common import make_layer, oracle_params, to_device

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _wl(**kw):
    base = dict(name="mamba2_prefill_small", batch=2, nheads=4, ngroups=2, headdim=64, dstate=128,
                window=8, steps=300, seed=91, input_dtype="bf16", read_dtype="f32")
    base.update(kw)
    return I.TINY.replace(**base)


def _dev_inputs(tok, wl):
    import torch

    d = {}
    for k, v in tok.items():
        dt = "bf16" if k in ("x", "B", "C") else "f32"
        d[k] = I.to_torch(v, dt).contiguous().cuda()
    return d


def _run(wl, S0=True, dt_scales=False, T=None):
    import torch

    T = wl.steps if T is None else T
    c = I.constants(wl)
    toks = I.tokens(wl, 0, T)
    d = _dev_inputs(toks, wl)
    A = torch.tensor(c["A"], dtype=torch.float32, device="cuda")
    D = torch.tensor(c["D"], dtype=torch.float32, device="cuda")
    S0d = torch.from_numpy(c["S0"].astype(np.float32)).cuda() if S0 else None
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    y, S = rssm.prefill(d["x"], d["dt"], d["B"], d["C"], A, D, S0d, dt_scales_input=dt_scales, err=err)
    torch.cuda.synchronize()
    assert err.tolist() == [0, 0, 0, 0]
    S0o = c["S0"] if S0 else np.zeros_like(c["S0"])
    y_ref, S_ref = oprefill.mamba2(S0o, c["A"], c["D"], toks["x"], toks["dt"], toks["B"], toks["C"], 128,
                                   dt_scales)
    return y.double().cpu().numpy(), S.double().cpu().numpy(), y_ref, S_ref, c, toks


def _check(y, S, y_ref, S_ref):
    T = y.shape[1]
    for t in range(T):
        rms = np.sqrt(np.mean(np.square(y_ref[:, t])))
        assert np.max(np.abs(y[:, t] - y_ref[:, t])) <= TOL * rms, t
    rms = np.sqrt(np.mean(np.square(S_ref)))
    assert np.max(np.abs(S - S_ref)) <= TOL * rms


@pytest.mark.parametrize("P", [32, 64, 96])
def test_prefill_ragged_prompt_matches_oracle(P):
    """300 tokens: two full chunks and a partial one."""
    y, S, y_ref, S_ref, _, _ = _run(_wl(headdim=P))
    _check(y, S, y_ref, S_ref)


@pytest.mark.parametrize("T", [1, 127, 128, 129, 256])
def test_prefill_chunk_edges(T):
    y, S, y_ref, S_ref, _, _ = _run(_wl(batch=1, nheads=2, ngroups=1), T=T)
    _check(y, S, y_ref, S_ref)


def test_prefill_dt_scaled_input_and_zero_state():
    y, S, y_ref, S_ref, _, _ = _run(_wl(seed=92), S0=False, dt_scales=True)
    _check(y, S, y_ref, S_ref)


def test_prefill_hands_its_state_to_replay_decode():
    """prefill -> rssm_import_state -> decode across a fold: every decode output
    against the eager oracle continued from the oracle's state after the prompt."""
    import torch

    wl = _wl(seed=93, window=4, steps=200)
    y, S, y_ref, S_ref, c, _ = _run(wl)
    _check(y, S, y_ref, S_ref)
    L, _ = make_layer(wl, "replay", "bf16", consts=dict(A=c["A"], D=c["D"], S0=S.astype(np.float32)))
    S_o = np.ascontiguousarray(S_ref.copy())
    for t in range(wl.steps, wl.steps + 2 * wl.window + 1):
        tok = I.token(wl, t)
        yd = L.decode(to_device(tok, wl, with_T=False))[:, 0].double().cpu().numpy()
        ye = eager.mamba2_step(S_o, c["A"], c["D"], tok["x"], tok["dt"], tok["B"], tok["C"])
        rms = np.sqrt(np.mean(np.square(ye)))
        assert np.max(np.abs(yd - ye)) <= 2e-2 * rms, t  # bf16 read copy of the imported checkpoint
    assert L.status()[0] == 0
    torch.cuda.synchronize()


def test_prefill_full_size_sampled():
    """The benchmark's launch: 256 sequences x 128 heads x 64 x 128, 512-token
    prompts.  Four sequences follow their seeded streams and are compared with
    the oracle (every token, every head, and their final states); the others
    hold seeded device-generated inputs of the same distributions."""
    import torch

    wl = I.PREFILL
    T, Bn, H, G, P, N = wl.steps, wl.batch, wl.nheads, wl.ngroups, wl.headdim, wl.dstate
    seqs = [0, 97, 128, 255]
    gen = torch.Generator(device="cuda").manual_seed(6)
    x = torch.randn((Bn, T, H, P), generator=gen, device="cuda").to(torch.bfloat16)
    dt = torch.nn.functional.softplus(torch.randn((Bn, T, H), generator=gen, device="cuda") - 2.0)
    Bm = torch.randn((Bn, T, G, N), generator=gen, device="cuda").to(torch.bfloat16)
    Cm = torch.randn((Bn, T, G, N), generator=gen, device="cuda").to(torch.bfloat16)
    S0 = 0.1 * torch.randn((Bn, H, P, N), generator=gen, device="cuda")
    c = I.constants(wl, seqs)
    toks = I.tokens(wl, 0, T, seqs)
    idx = torch.tensor(seqs, device="cuda")
    d = _dev_inputs(toks, wl)
    x[idx], dt[idx], Bm[idx], Cm[idx] = d["x"], d["dt"], d["B"], d["C"]
    S0[idx] = torch.from_numpy(c["S0"].astype(np.float32)).cuda()
    A = torch.tensor(c["A"], dtype=torch.float32, device="cuda")
    D = torch.tensor(c["D"], dtype=torch.float32, device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    y, S = rssm.prefill(x, dt, Bm, Cm, A, D, S0, err=err)
    torch.cuda.synchronize()
    assert err.tolist() == [0, 0, 0, 0]
    assert torch.isfinite(y).all() and torch.isfinite(S).all()
    y_ref, S_ref = oprefill.mamba2(c["S0"], c["A"], c["D"], toks["x"], toks["dt"], toks["B"], toks["C"], 128)
    _check(y[idx].double().cpu().numpy(), S[idx].double().cpu().numpy(), y_ref, S_ref)


def test_prefill_refuses_unsupported_sizes():
    import torch

    wl = _wl()
    for kw in (dict(dstate=64), dict(headdim=48), dict(headdim=128)):
        w2 = wl.replace(**kw)
        toks = I.tokens(w2, 0, 3)
        d = _dev_inputs(toks, w2)
        A = torch.zeros(w2.nheads, device="cuda")
        with pytest.raises(rssm.RssmError) as e:
            rssm.prefill(d["x"], d["dt"], d["B"], d["C"], A, A)
        assert e.value.status == rssm.RSSM_EINVAL
