"""Decode-throughput benchmark of one SSM layer (Mamba-2, Nemotron-scale) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one rssm_decode call: one token for each of the 256 sequences of a
Mamba-2 layer with 128 heads x headdim 64 x dstate 128 (4 MiB of fp32 state per
sequence), 8 groups, window 16, fp32 checkpoint + bf16 read copy, bf16 inputs;
the fold of a full buffer happens inside the step every 16 tokens.  Inputs are
seeded synthetic tokens already resident in HBM (cycling through up to 256
distinct steps); the 512 MiB read copy is larger than L2, so no flush is needed
between steps.  Prints one JSON line (rank 0).

N > 1 (torchrun): every rank decodes its own 256 sequences (weak scaling, no
collective on the data path); the time is the max over ranks.
--impl reference times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from checkpoint_input_replay_rssm_b200 import inputs as I  # noqa: E402
from checkpoint_input_replay_rssm_b200 import traffic  # noqa: E402

METRIC = "SSM-layer decode tokens/s and achieved HBM GB/s vs ~8 TB/s roofline (1×B200)"
WL = I.NEMOTRON
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "m2_replay_decode_b256_h128_p64_n128_w16.traffic.json")


TRAFFIC_SOURCES = ("rssm_read.cuh", "rssm_device.cuh")


def kernel_source_hash() -> str:
    """Hash of the sources of the replay-read kernel, to tell whether a stored ncu
    traffic figure was taken on the kernel as it is now."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "checkpoint_input_replay_rssm_b200", "csrc")
    for f in TRAFFIC_SOURCES:
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(p))["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls NVML (read-only) for SM clock and clock-event reasons during the timed region."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, do not guess
            self.err = str(e)
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ setup
def make_layer(wl, mode, state_dtype, consts, device, max_draft=1):
    import torch

    from checkpoint_input_replay_rssm_b200 import rssm

    cfg = rssm.make_config(kind=wl.kind, mode=mode, state_dtype=state_dtype,
                           input_dtype=wl.input_dtype, batch=wl.batch, nheads=wl.nheads,
                           headdim=wl.headdim, dstate=wl.dstate, ngroups=wl.ngroups,
                           window=wl.window, max_draft=max_draft)
    L = rssm.Layer(cfg, device=device)
    if wl.kind == "mamba2":
        L.set_params(torch.tensor(consts["A"], dtype=torch.float32, device=device),
                     torch.tensor(consts["D"], dtype=torch.float32, device=device))
    L.import_state(torch.from_numpy(consts["S0"]).to(device))
    return L


def prime(wl, mode, state_dtype, device, max_draft=1):
    """Launch every kernel a leg times once, on a 2-sequence copy of its layer, before
    the leg's own warm-up: decodes across a fold (and verify / commit rounds across a
    fold when drafts are served), so lazy module loading never lands in a timed region."""
    import torch

    small = wl.replace(batch=2)
    consts = I.constants(small, f64=False)
    L = make_layer(small, mode, state_dtype, consts, device, max_draft=max_draft)
    for t in range(small.window + 1):
        L.decode(device_tokens(small, I.token(small, t), device, False))
    if max_draft > 1:
        acc = torch.zeros(small.batch, dtype=torch.int32, device=device)
        for r in range(small.window // max_draft + 2):
            L.verify(max_draft, device_tokens(small, I.tokens(small, r * max_draft, max_draft), device, True))
            L.commit(acc)
    torch.cuda.synchronize()
    assert L.status()[0] == 0
    del L


def device_tokens(wl, tok, device, with_T):
    """One seeded token dict (numpy float64) as device tensors in storage dtypes."""
    wide = ("x", "B", "C", "q", "k", "v")
    out = {}
    for k, v in tok.items():
        t = I.to_torch(v, wl.input_dtype if k in wide else "f32")
        out[k] = (t if with_T else t.unsqueeze(1)).contiguous().to(device)
    return out


def spec_leg(rank, device, sync, dist, world, rounds, warmup):
    """Speculative verify + commit on the 512-sequence, 128-head Mamba-2 layer with K = 4
    drafts and seeded accept lengths a ~ U{0..4}: committed tokens/s, replay (bf16 copy)
    and the eager snapshot baseline (fp32 state, K snapshots per round)."""
    import torch

    wl = I.SPECVERIFY.replace(seed=I.SPECVERIFY.seed + 7919 * rank)
    K = wl.draft_k
    consts = I.constants(wl, f64=False)
    n = min(rounds + warmup, 16)
    toks = [device_tokens(wl, I.tokens(wl, r * K, K), device, True) for r in range(n)]
    acc = [torch.tensor(I.accept_lengths(wl, r), dtype=torch.int32, device=device) for r in range(n)]
    kept = [int(a.sum()) for a in acc]
    out = {}
    for name, mode, sd in (("replay", "replay", "bf16"), ("eager", "eager", "f32")):
        prime(wl, mode, sd, device, max_draft=K)
        L = make_layer(wl, mode, sd, consts, device, max_draft=K)
        y = torch.empty((wl.batch, K, wl.nheads, wl.headdim), dtype=torch.float32, device=device)
        for r in range(warmup):
            L.verify(K, toks[r % n], y=y)
            L.commit(acc[r % n])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sync()
        e0.record(L.stream)
        committed = 0
        for i in range(rounds):
            r = (warmup + i) % n
            L.verify(K, toks[r], y=y)
            L.commit(acc[r])
            committed += kept[r]
        e1.record(L.stream)
        sync()
        assert L.status()[0] == 0, "device error in the speculative leg"
        (ms,) = max_over_ranks(dist, [e0.elapsed_time(e1)], device)
        out[name] = {"value": world * committed / (ms * 1e-3), "unit": "committed tokens/s",
                     "ms_per_round": ms / rounds}
        del L
        torch.cuda.empty_cache()
    out["config"] = {"workload": wl.name, "batch_per_gpu": wl.batch, "draft_k": K, "rounds": rounds,
                     "accept": "U{0..K} per sequence and round, seeded", "read_copy": "bf16 (replay)",
                     "eager_state": "f32 with K snapshots"}
    out["speedup_vs_eager"] = out["replay"]["value"] / out["eager"]["value"]
    return out


def delta_leg(wl0, rank, device, sync, dist, world, steps, warmup, batch=None):
    """Gated DeltaNet or Kimi Delta Attention decode, 256 sequences x 32 heads x 128 x 128,
    W = 16: replay (bf16 copy) and eager (fp32) tokens/s, with the state bytes per token
    of each."""
    import torch

    wl = wl0.replace(seed=wl0.seed + 7919 * rank, batch=batch or wl0.batch)
    consts = I.constants(wl, f64=False)
    n = min(steps + warmup, 32)
    toks = [device_tokens(wl, I.token(wl, t), device, False) for t in range(n)]
    out = {}
    for name, mode, sd in (("replay", "replay", "bf16"), ("eager", "eager", "f32")):
        prime(wl, mode, sd, device)
        L = make_layer(wl, mode, sd, consts, device)
        y = torch.empty((wl.batch, 1, wl.nheads, wl.headdim), dtype=torch.float32, device=device)
        for t in range(warmup):
            L.decode(toks[t % n], y=y)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sync()
        e0.record(L.stream)
        for i in range(steps):
            L.decode(toks[(warmup + i) % n], y=y)
        e1.record(L.stream)
        sync()
        assert L.status()[0] == 0, f"device error in the {wl.kind} leg"
        (ms,) = max_over_ranks(dist, [e0.elapsed_time(e1)], device)
        out[name] = {"value": job_tokens_per_s(world, wl.batch, steps, ms), "unit": "tokens/s",
                     "ms_per_step": ms / steps}
        del L
        torch.cuda.empty_cache()
    shape = traffic.Shape(wl.kind, wl.headdim, wl.dstate, 1, wl.window, "bf16", wl.input_dtype)
    rep, eg = traffic.replay_decode_per_token(shape), traffic.eager_decode_per_token(shape, "f32")
    units = wl.batch * wl.nheads
    out["replay"]["hbm_gbs"] = traffic.total(rep) * units * steps / (out["replay"]["ms_per_step"] * steps * 1e-3) / 1e9
    out["eager"]["hbm_gbs"] = traffic.total(eg) * units * steps / (out["eager"]["ms_per_step"] * steps * 1e-3) / 1e9
    out["state_bytes_per_token_per_head"] = {"replay": traffic.state_bytes(rep), "eager": traffic.state_bytes(eg),
                                             "ratio": traffic.state_bytes(rep) / traffic.state_bytes(eg)}
    out["config"] = {"workload": wl.name, "batch_per_gpu": wl.batch, "nheads": wl.nheads, "d_k": wl.dstate,
                     "d_v": wl.headdim, "window": wl.window, "read_copy": "bf16", "inputs": wl.input_dtype}
    return out


def hybrid_leg(device, sync, dist, world, steps, warmup):
    """A synthetic hybrid decode step on the Nemotron-scale layer shapes: one block
    of five Mamba-2 layers (this library, replay with a bf16 copy or the eager
    fp32 baseline) and one attention layer (32 query / 2 key-value heads of 128,
    4096 cached tokens, bf16), each with bf16 in/out projections of a 4096-wide
    hidden state, random weights.  Whole-step tokens/s for each SSM mode, and the
    share of the step spent in the SSM layers' decode calls (a second pass with
    CUDA events around every decode call)."""
    import torch

    from checkpoint_input_replay_rssm_b200.hybrid import HybridShape, HybridStack

    shape = HybridShape()
    out = {}
    for name, mode, rd in (("replay", "replay", "bf16"), ("eager", "eager", "f32")):
        st = HybridStack(shape, ssm_mode=mode, read_dtype=rd, seed=11, device=device,
                         max_steps=warmup + 2 * steps + 2)
        g = torch.Generator(device=device).manual_seed(12)
        xs = [torch.randn((shape.batch, shape.d_model), generator=g, device=device).to(torch.bfloat16)
              for _ in range(8)]
        for i in range(warmup):
            st.step(xs[i % 8])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sync()
        e0.record()
        for i in range(steps):
            st.step(xs[i % 8])
        e1.record()
        sync()
        (ms,) = max_over_ranks(dist, [e0.elapsed_time(e1)], device)
        st.ssm_events = []
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for i in range(steps):
            st.step(xs[i % 8])
        f1.record()
        sync()
        ssm_ms = sum(a.elapsed_time(b) for a, b in st.ssm_events)
        timed_ms = f0.elapsed_time(f1)
        for L in st.ssm_layers():
            assert L.status()[0] == 0, "device error in the hybrid leg"
        out[name] = {"value": job_tokens_per_s(world, shape.batch, steps, ms), "unit": "tokens/s",
                     "ms_per_step": ms / steps, "ssm_ms_per_step": ssm_ms / steps,
                     "ssm_share": ssm_ms / timed_ms}
        del st
        torch.cuda.empty_cache()
    out["step_speedup"] = out["eager"]["ms_per_step"] / out["replay"]["ms_per_step"]
    out["ssm_speedup"] = out["eager"]["ssm_ms_per_step"] / out["replay"]["ssm_ms_per_step"]
    out["config"] = {"blocks": shape.blocks, "ssm_per_attention": shape.ssm_per_block, "batch_per_gpu": shape.batch,
                     "d_model": shape.d_model, "ssm_layer": "mamba2 128 heads x 64 x 128, 8 groups, W 16",
                     "attention": f"{shape.n_q_heads} q / {shape.n_kv_heads} kv heads x {shape.head_dim}, "
                                  f"{shape.context} cached tokens, bf16, torch SDPA (flash / memory-efficient kernels)",
                     "projections": "bf16 torch.matmul, random weights", "steps": steps}
    return out


def prefill_leg(device, sync, dist, world, reps, warmup, batch=None):
    """Prompt prefill of the Nemotron-scale layer on the tensor cores: 256 sequences x
    128 heads, 512-token prompts, seeded device-generated inputs of the decode
    workload's distributions; prompt tokens/s and the roofline of the kernel."""
    import torch

    from checkpoint_input_replay_rssm_b200 import rssm

    wl = I.PREFILL.replace(batch=batch or I.PREFILL.batch)
    Bn, T, H, G, P, N = wl.batch, wl.steps, wl.nheads, wl.ngroups, wl.headdim, wl.dstate
    g = torch.Generator(device=device).manual_seed(wl.seed)
    x = torch.randn((Bn, T, H, P), generator=g, device=device).to(torch.bfloat16)
    dt = torch.nn.functional.softplus(torch.randn((Bn, T, H), generator=g, device=device) - 2.0)
    Bm = torch.randn((Bn, T, G, N), generator=g, device=device).to(torch.bfloat16)
    Cm = torch.randn((Bn, T, G, N), generator=g, device=device).to(torch.bfloat16)
    A = -torch.exp(torch.rand(H, generator=g, device=device))
    D = torch.randn(H, generator=g, device=device)
    S0 = 0.1 * torch.randn((Bn, H, P, N), generator=g, device=device)
    y = torch.empty((Bn, T, H, P), dtype=torch.float32, device=device)
    S = torch.empty_like(S0)
    err = torch.zeros(4, dtype=torch.int32, device=device)
    for _ in range(warmup):
        rssm.prefill(x, dt, Bm, Cm, A, D, S0, y=y, S_out=S, err=err)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync()
    e0.record()
    for _ in range(reps):
        rssm.prefill(x, dt, Bm, Cm, A, D, S0, y=y, S_out=S, err=err)
    e1.record()
    sync()
    assert err.tolist() == [0, 0, 0, 0], "device error in the prefill leg"
    (ms,) = max_over_ranks(dist, [e0.elapsed_time(e1) / reps], device)
    heads = Bn * H
    bytes_per_launch = heads * (T * (P * 2 + P * 4 + 4) + P * N * 4 * 2) + Bn * T * G * N * 2 * 2
    # tensor-core work: per head and 128-token chunk, C B^T (1x), S C (2x), the
    # state update (2x) and M x (2x), the fp32 operands split in two bf16 parts
    chunks = -(-T // 128)
    flops = heads * chunks * (2 * 128 * 128 * N + 2 * 2 * 128 * P * N + 2 * 2 * N * P * 128 + 2 * 2 * 128 * P * 128)
    return {"value": world * Bn * T / (ms * 1e-3), "unit": "prompt tokens/s", "ms_per_launch": ms,
            "hbm_gbs": bytes_per_launch / (ms * 1e-3) / 1e9, "algorithmic_bytes_per_launch": bytes_per_launch,
            "tensor_tflops": flops / (ms * 1e-3) / 1e12, "mma_flops_per_launch": flops,
            "config": {"workload": wl.name, "batch_per_gpu": Bn, "prompt_tokens": T, "chunk": 128,
                       "inputs": "bf16 x, B, C; fp32 dt", "state": "fp32 in and out", "y": "fp32"}}


def host_tokens(wl, n):
    """n distinct seeded decode steps as pinned host tensors in storage dtypes."""
    import torch

    out = []
    for t in range(n):
        tok = I.token(wl, t)
        d = {}
        for k, v in tok.items():
            ht = I.to_torch(v, wl.input_dtype if k in ("x", "B", "C") else "f32").unsqueeze(1)
            d[k] = ht.contiguous().pin_memory()
        out.append(d)
    return out


def timed_loop(L, toks_dev, ys, K, W, sync, split=True):
    """W warm-up then K timed decode steps (the headline: CUDA events around the whole
    loop only, so the read kernel may overlap the prep kernel's tail); then M whole
    windows (M * window steps, each window holding exactly one folding call) timed
    the same way, the steady state; with ``split``, K more steps with CUDA events
    on the layer's stream around every call and between its prep/flush and
    replay-read kernels (an event between them keeps the two kernels apart, so
    each one's duration is its own)."""
    import torch

    from checkpoint_input_replay_rssm_b200 import rssm

    n = len(toks_dev)
    ins = [L._inputs(d) for d in toks_dev]
    yptr = [y.data_ptr() for y in ys]
    stream = L.stream
    for i in range(W):
        rssm.rssm_decode(L.h, ins[i % n], yptr[i % len(ys)])
    mk = lambda: torch.cuda.Event(enable_timing=True)
    t0, t1 = mk(), mk()
    sync()
    l0 = L.launches()
    t0.record(stream)
    for i in range(K):
        rssm.rssm_decode(L.h, ins[(W + i) % n], yptr[i % len(ys)])
    t1.record(stream)
    sync()
    launches = L.launches() - l0
    total_ms = t0.elapsed_time(t1)
    win = L.cfg.window
    M = max(1, round(K / win))
    t2, t3 = mk(), mk()
    sync()
    t2.record(stream)
    for i in range(M * win):
        rssm.rssm_decode(L.h, ins[(W + K + i) % n], yptr[i % len(ys)])
    t3.record(stream)
    sync()
    steady = (t2.elapsed_time(t3), M * win)
    W = W + M * win  # calls since the import, for the per-kernel pass below
    if not split:
        return total_ms, None, None, None, launches, steady
    starts, mids, ends = [mk() for _ in range(K)], [mk() for _ in range(K)], [mk() for _ in range(K)]
    for e in mids:  # materialise the CUDA events before handing them to the library
        e.record(stream)
    sync()
    for i in range(K):
        rssm.rssm_set_split_event(L.h, mids[i].cuda_event)
        starts[i].record(stream)
        rssm.rssm_decode(L.h, ins[(W + K + i) % n], yptr[i % len(ys)])
        ends[i].record(stream)
    sync()
    rssm.rssm_set_split_event(L.h, None)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    pre = [s.elapsed_time(m) for s, m in zip(starts, mids)]
    read = [m.elapsed_time(e) for m, e in zip(mids, ends)]
    return total_ms, per, pre, read, launches, steady


def pack_inputs(toks_host, pin):
    """Each step's input tensors packed into one byte buffer (pinned when `pin`),
    every input at a 256-byte offset, so that a step's inputs travel as one copy.
    Returns the buffers, the offsets by input name and the buffer length."""
    import torch

    keys = list(toks_host[0].keys())
    nbytes = {k: toks_host[0][k].numel() * toks_host[0][k].element_size() for k in keys}
    offs, total = {}, 0
    for k in keys:
        offs[k] = total
        total += (nbytes[k] + 255) // 256 * 256
    out = []
    for d in toks_host:
        buf = torch.zeros(total, dtype=torch.uint8)
        for k in keys:
            buf[offs[k]:offs[k] + nbytes[k]].copy_(d[k].contiguous().view(-1).view(torch.uint8))
        out.append(buf.pin_memory() if pin else buf)
    return out, offs, total


def input_views(buf, like, offs):
    """The inputs inside one packed buffer, as tensors shaped and typed like `like`."""
    return {k: buf[o:o + like[k].numel() * like[k].element_size()].view(like[k].dtype).view(like[k].shape)
            for k, o in offs.items()}


def e2e_loop(L, toks_host, K, W, sync, nbuf=4):
    """Public-API decode with host buffers: every step copies its inputs from pinned
    host memory to the device (one copy per step), decodes, and copies its output y
    back to pinned host memory, all inside the timed region.  `nbuf` sets of device
    buffers rotate so that later steps' input copies (one copy stream) and earlier
    steps' output copies (another) run while the layer's stream decodes; events
    order each buffer's reuse."""
    import torch

    n = len(toks_host)
    # A step's inputs travel as one copy: each host step packed into one pinned
    # buffer, the device inputs views of one device buffer with the same layout.
    host_packed, offs, total = pack_inputs(toks_host, pin=True)
    dev_buf = [torch.empty(total, dtype=torch.uint8, device=L.device) for _ in range(nbuf)]
    dev = [input_views(dev_buf[j], toks_host[0], offs) for j in range(nbuf)]
    y = [torch.empty((L.B, 1, L.H, L.P), dtype=torch.float32, device=L.device) for _ in range(nbuf)]
    y_host = [torch.empty_like(y[0], device="cpu").pin_memory() for _ in range(nbuf)]
    comp = torch.cuda.ExternalStream(L.stream) if not isinstance(L.stream, torch.cuda.Stream) else L.stream
    h2d_s, d2h_s = torch.cuda.Stream(L.device), torch.cuda.Stream(L.device)
    ev = lambda: torch.cuda.Event()
    in_ready, in_free = [ev() for _ in range(nbuf)], [ev() for _ in range(nbuf)]
    y_ready, y_free = [ev() for _ in range(nbuf)], [ev() for _ in range(nbuf)]
    for j in range(nbuf):  # every buffer starts free
        in_free[j].record(comp)
        y_free[j].record(d2h_s)

    def step(i):
        j = i % nbuf
        with torch.cuda.stream(h2d_s):
            h2d_s.wait_event(in_free[j])
            dev_buf[j].copy_(host_packed[i % n], non_blocking=True)
            in_ready[j].record(h2d_s)
        comp.wait_event(in_ready[j])
        comp.wait_event(y_free[j])
        L.decode(dev[j], y=y[j])
        in_free[j].record(comp)
        y_ready[j].record(comp)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(y_ready[j])
            y_host[j].copy_(y[j], non_blocking=True)
            y_free[j].record(d2h_s)

    for i in range(W):
        step(i)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync()
    t0.record(comp)
    h2d_s.wait_event(t0)
    d2h_s.wait_event(t0)
    for i in range(K):
        step(W + i)
    done = torch.cuda.Event()
    done.record(d2h_s)
    comp.wait_event(done)
    t1.record(comp)
    sync()
    return t0.elapsed_time(t1), total, y[0].numel() * y[0].element_size()


# ------------------------------------------------------------------ CPU oracle legs
def oracle_tokens_per_s(wl, seqs, max_steps, budget_s):
    """Time the fp64 eager oracle (as it stands) on `seqs` sequences for up to
    `max_steps` tokens or `budget_s` seconds of oracle time; input generation is
    outside the timed part."""
    from oracle import eager

    c = I.constants(wl, seqs=range(seqs))
    S = np.ascontiguousarray(c["S0"])
    done, t_used = 0, 0.0
    for t in range(max_steps):
        tok = I.token(wl, t, seqs=range(seqs))
        t0 = time.perf_counter()
        eager.mamba2_step(S, c["A"], c["D"], tok["x"], tok["dt"], tok["B"], tok["C"])
        t_used += time.perf_counter() - t0
        done += 1
        if t_used >= budget_s:
            break
    return seqs * done / t_used, done, t_used, eager.max_threads()


def run_reference(args, rank):
    if rank != 0:
        return
    from oracle import eager

    eager.build()
    seqs = 16
    K, W = args.steps, args.warmup
    c = I.constants(WL, seqs=range(seqs))
    n = min(K + W, 8)
    toks = [I.token(WL, t, seqs=range(seqs)) for t in range(n)]
    S = np.ascontiguousarray(c["S0"])
    for i in range(W):
        tok = toks[i % n]
        eager.mamba2_step(S, c["A"], c["D"], tok["x"], tok["dt"], tok["B"], tok["C"])
    t0 = time.perf_counter()
    for i in range(K):
        tok = toks[(W + i) % n]
        eager.mamba2_step(S, c["A"], c["D"], tok["x"], tok["dt"], tok["B"], tok["C"])
    dt = time.perf_counter() - t0
    value = seqs * K / dt
    sample = (f"fp64 eager oracle (C, OpenMP) on {seqs} of the 256 sequences x 128 heads x 64 x 128, "
              f"one token per step, inputs pre-generated")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": K, "warmup": W, "ms_per_step": dt * 1e3 / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": eager.max_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def rank_workload(rank: int, batch: int):
    """The workload one rank decodes: the same layer shapes, its own sequences
    (seeded per rank), so that N ranks run N independent batches."""
    return WL.replace(seed=WL.seed + 7919 * rank, batch=batch)


def max_over_ranks(dist, values, device):
    """Element-wise max of per-rank timings (ms) over the process group; the
    values themselves when there is no group."""
    if dist is None:
        return [float(v) for v in values]
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tokens_per_s(world: int, batch: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank decoded `batch` sequences for `steps`
    tokens, and the job took the slowest rank's time."""
    return world * batch * steps / (ms * 1e-3)


def workload_config(batch=None):
    return {"workload": WL.name, "batch_per_gpu": batch or WL.batch, "nheads": WL.nheads, "headdim": WL.headdim,
            "dstate": WL.dstate, "ngroups": WL.ngroups, "window": WL.window, "checkpoint": "f32",
            "read_copy": "bf16", "inputs": "bf16",
            "l2": "no flush: the 512 MiB read copy read every step exceeds the 126 MB L2",
            "input_steps": "seeded steps resident in HBM, cycled",
            "priming": "every timed kernel launched once on a 2-sequence copy of the layer before the warm-up"}


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-eager", action="store_true", help="skip the eager-baseline leg")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle leg")
    ap.add_argument("--no-spec", action="store_true", help="skip the speculative-verify leg")
    ap.add_argument("--no-gdn", action="store_true", help="skip the Gated DeltaNet leg")
    ap.add_argument("--no-kda", action="store_true", help="skip the Kimi Delta Attention leg")
    ap.add_argument("--no-hybrid", action="store_true", help="skip the synthetic hybrid-step leg")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill leg")
    ap.add_argument("--e2e-buffers", type=int, default=4,
                    help="device buffer sets rotating in the end-to-end loop (2 or more)")
    ap.add_argument("--batch", type=int, default=WL.batch,
                    help="sequences per GPU (default: the workload's 256; smaller for profiling; applies to "
                         "the decode, GDN, KDA and prefill legs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import datetime

    import torch

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    def sync():
        torch.cuda.synchronize(device)
        if dist is not None:
            dist.barrier()
            torch.cuda.synchronize(device)

    from checkpoint_input_replay_rssm_b200 import build, rssm

    if not os.path.exists(build.LIB):
        build.build()
    rssm.load()

    K, W = args.steps, args.warmup
    wl = rank_workload(rank, args.batch)
    consts = I.constants(wl, f64=False)
    n_distinct = min(K + W, 256)
    toks_host = host_tokens(wl, n_distinct)
    toks_dev = [{k: v.to(device) for k, v in d.items()} for d in toks_host]
    ys = [torch.empty((wl.batch, 1, wl.nheads, wl.headdim), dtype=torch.float32, device=device)
          for _ in range(2)]

    prime(wl, "replay", "bf16", device)
    if not args.no_eager:
        prime(wl, "eager", "f32", device)
    L = make_layer(wl, "replay", "bf16", consts, device)
    sampler = ClockSampler(local)
    with sampler:
        total_ms, per, flush_ms, read_ms, launches, steady = timed_loop(L, toks_dev, ys, K, W, sync)
    # calls of the per-kernel pass are W + K + M*window + i since the import: a call folds at len = window
    c0 = W + K + steady[1]
    fold = [(c0 + i) >= wl.window and (c0 + i) % wl.window == 0 for i in range(K)]
    pick = lambda xs, want: [x for x, f in zip(xs, fold) if f == want]
    clocks = sampler.summary()
    total_ms, kern_ms, steady_ms = max_over_ranks(dist, [total_ms, float(np.mean(read_ms)), steady[0]], device)
    assert L.status()[0] == 0, "device error during the benchmark"

    # e2e through the public API with host buffers (same layer, state re-imported)
    L.import_state(torch.from_numpy(consts["S0"]).to(device))
    e2e_ms, h2d, d2h = e2e_loop(L, toks_host, K, W, sync, nbuf=max(2, args.e2e_buffers))
    (e2e_ms,) = max_over_ranks(dist, [e2e_ms], device)
    assert L.status()[0] == 0, "device error in the end-to-end loop"

    shape = traffic.Shape("mamba2", wl.headdim, wl.dstate, wl.nheads // wl.ngroups, wl.window, "bf16",
                          wl.input_dtype)
    rep = traffic.replay_decode_per_token(shape)
    win = traffic.replay_decode_window(shape)
    units = wl.batch * wl.nheads
    bytes_per_launch = traffic.total(win["read"]) * units       # replay-read kernel, window mean per call
    sp_fold = traffic.replay_step_split(shape, wl.window, True)
    fold_bytes = traffic.total(sp_fold["prep"]) * units          # prep + flush kernels of a folding call
    prep_bytes = traffic.total(traffic.replay_step_split(shape, wl.window // 2, False)["prep"]) * units
    achieved = bytes_per_launch / (kern_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    tr, tr_note = None, "no ncu capture of the current kernel"
    if os.path.exists(PROFILE_TRAFFIC):
        p = json.load(open(PROFILE_TRAFFIC))
        if p.get("kernel_hash") == kernel_source_hash():
            # measured DRAM bytes per launch over its own launches, put on the
            # window-mean basis of `achieved` by the algorithmic bytes of both
            tr = p["dram_bytes_per_launch"] * bytes_per_launch / p["algorithmic_bytes_same_launches"]
            tr_note = (f"ncu dram bytes {p['dram_bytes_per_launch']:.4g} per launch over launches with "
                       f"{p['algorithmic_bytes_same_launches']:.4g} algorithmic bytes, scaled to the window mean")
    fold_call_ms = float(np.mean(pick(flush_ms, True))) if any(fold) else None
    prep_call_ms = float(np.mean(pick(flush_ms, False)))

    eager = None
    if not args.no_eager:
        del L
        torch.cuda.empty_cache()
        E = make_layer(wl, "eager", "f32", consts, device)
        e_total, _, _, _, _, _ = timed_loop(E, toks_dev, ys, K, W, sync, split=False)
        (e_total,) = max_over_ranks(dist, [e_total], device)
        e_kern = e_total / K  # one kernel per eager call
        eg = traffic.eager_decode_per_token(shape, "f32")
        eager = {"value": job_tokens_per_s(world, wl.batch, K, e_total), "unit": "tokens/s",
                 "ms_per_step": e_total / K,
                 "hbm_gbs": traffic.total(eg) * units / (e_kern * 1e-3) / 1e9,
                 "bytes_per_token_per_head": traffic.total(eg)}
        del E

    spec = None if args.no_spec else spec_leg(rank, device, sync, dist, world, min(K, 64), W)
    small = args.batch if args.batch != WL.batch else None  # a smaller batch for profiling applies to every leg
    gdn = None if args.no_gdn else delta_leg(I.GDN, rank, device, sync, dist, world, min(K, 128), W, small)
    kda = None if args.no_kda else delta_leg(I.KDA, rank, device, sync, dist, world, min(K, 128), W, small)
    hybrid = None if args.no_hybrid else hybrid_leg(device, sync, dist, world, min(K, 64), W)
    pre = None if args.no_prefill else prefill_leg(device, sync, dist, world, 5, 3, small)

    state_rep, state_eag = traffic.state_bytes(rep), traffic.state_bytes(
        traffic.eager_decode_per_token(shape, "f32"))
    line = {
        "metric": METRIC,
        "value": job_tokens_per_s(world, wl.batch, K, total_ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(wl.batch) | {"parallelism": f"dp{world} (independent sequences)"},
        "hbm_gbs": achieved,
        "steady_state": {"value": job_tokens_per_s(world, wl.batch, steady[1], steady_ms), "unit": "tokens/s",
                         "ms_per_step": steady_ms / steady[1], "steps": steady[1],
                         "note": "whole windows: every 16 consecutive calls hold exactly one folding call"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": tr, "traffic_basis": tr_note, "peak_source": peak_kind,
                     "kernel": "replay_read_kernel<128, bf16, 1>",
                     "algorithmic_bytes_per_launch": bytes_per_launch,
                     "kernel_ms_per_launch": kern_ms,
                     "read_ms_nonfold_call": float(np.mean(pick(read_ms, False))),
                     "read_gbs_nonfold_call": traffic.total(traffic.replay_step_split(shape, wl.window // 2, False)["read"])
                                              * units / (np.mean(pick(read_ms, False)) * 1e-3) / 1e9},
        "prep_kernel": {"kernel": "m2_prep_kernel<128, 1>", "ms_nonfold_call": prep_call_ms,
                        "algorithmic_bytes_nonfold_call": prep_bytes},
        "flush_kernel": {"kernel": "m2_fold_kernel<128, bf16, 1>",
                         "ms_per_fold_call": fold_call_ms, "note": "prep + flush kernels of a folding call",
                         "algorithmic_bytes_per_fold_call": fold_bytes,
                         "gbs": fold_bytes / (fold_call_ms * 1e-3) / 1e9 if fold_call_ms else None,
                         "frac": fold_bytes / (fold_call_ms * 1e-3) / 1e9 / peak if fold_call_ms else None},
        "ms_per_call": {"nonfold": float(np.mean(pick(per, False))),
                        "fold": float(np.mean(pick(per, True))) if any(fold) else None},
        "e2e": {"value": job_tokens_per_s(world, wl.batch, K, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks,
        "state_bytes_per_token_per_head": {"replay": state_rep, "eager": state_eag,
                                           "ratio": state_rep / state_eag},
        "eager": eager,
        "spec_verify": spec,
        "gdn": gdn,
        "kda": kda,
        "hybrid_step": hybrid,
        "prefill": pre,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        from oracle import eager as oracle_eager

        v, done, used, cores = oracle_tokens_per_s(wl, 64, 256, 12.0)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"fp64 eager oracle on 64 of 256 sequences x 128 heads, "
                                          f"{done} steps, {used:.1f} s"}
        all_threads = oracle_eager.max_threads()
        oracle_eager.set_threads(1)
        try:
            v1, done1, used1, _ = oracle_tokens_per_s(wl, 8, 256, 6.0)
        finally:
            oracle_eager.set_threads(all_threads)
        line["cpu_baseline_1core"] = {"value": v1, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                      "sample": f"fp64 eager oracle, one thread, on 8 of 256 sequences x 128 "
                                                f"heads, {done1} steps, {used1:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
