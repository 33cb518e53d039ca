"""A synthetic hybrid decode step: where the SSM-layer saving lands in a step.

The hybrid models the ReplaySSM reports measure interleave about five SSM
layers per attention layer (blog.thibaultmonteiro.fr, "La fiche qu'on reecrit a
chaque token"), and the reports quote the whole decode step next to the SSM
kernel alone (irisproject.cloud, "Des chiffres").  This stand-in builds such a
stack with random weights (there is no trained model here): each block is
``ssm_per_block`` Mamba-2 layers decoded by librssm (replay or the eager
baseline) and one attention layer.  Every layer projects the hidden state in
and out with plain bf16 GEMMs (torch.matmul) after an RMS normalisation of its
input (pre-norm residual blocks, as in the hybrid models); the attention layer
appends the token's key and value to a bf16 cache and attends over it with
torch.nn.functional.scaled_dot_product_attention (grouped-query: the query heads
of a key/value head stacked as its query rows; flash or memory-efficient kernel).  The Mamba-2
layer's short convolution and output gate are left out: they carry no decode
state that the method changes.

Only the SSM layers' state handling differs between the two modes, so the step
time difference is the SSM saving as it shows in a step.  Nothing here is on
the SSM decode path itself, which runs entirely in librssm's kernels.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class HybridShape:
    batch: int = 256
    blocks: int = 1
    ssm_per_block: int = 5
    d_model: int = 4096
    nheads: int = 128     # Mamba-2 heads
    headdim: int = 64
    dstate: int = 128
    ngroups: int = 8
    window: int = 16
    n_q_heads: int = 32   # attention
    n_kv_heads: int = 2
    head_dim: int = 128
    context: int = 4096   # cached tokens per sequence before the first step

    @property
    def ssm_in(self) -> int:  # x, dt, B, C
        return self.nheads * self.headdim + self.nheads + 2 * self.ngroups * self.dstate


class HybridStack:
    """``blocks`` x (``ssm_per_block`` Mamba-2 layers + 1 attention layer) on one GPU.

    ssm_mode: "replay" (checkpoint + read copy ``read_dtype`` + buffer) or "eager"
    (fp32 state rewritten every token).  Weights, initial states and the cached
    keys/values come from a seeded torch generator.
    """

    def __init__(self, shape: HybridShape, ssm_mode: str = "replay", read_dtype: str = "bf16", seed: int = 0,
                 device="cuda", max_steps: int = 512):
        import torch

        from . import rssm

        self.s = s = shape
        self.torch = torch
        self.device = torch.device(device)
        g = torch.Generator(device=self.device).manual_seed(seed)
        bf = torch.bfloat16
        rnd = lambda *sh, scale: (torch.randn(sh, generator=g, device=self.device) * scale)
        self.layers = []
        for _blk in range(s.blocks):
            for _ in range(s.ssm_per_block):
                cfg = rssm.make_config(kind="mamba2", mode=ssm_mode,
                                       state_dtype=read_dtype if ssm_mode == "replay" else "f32",
                                       input_dtype="bf16", batch=s.batch, nheads=s.nheads, headdim=s.headdim,
                                       dstate=s.dstate, ngroups=s.ngroups, window=s.window, max_draft=1)
                L = rssm.Layer(cfg, device=self.device)
                A = -torch.exp(torch.rand(s.nheads, generator=g, device=self.device))
                D = torch.randn(s.nheads, generator=g, device=self.device)
                L.set_params(A.contiguous(), D.contiguous())
                L.import_state(rnd(s.batch, s.nheads, s.headdim, s.dstate, scale=0.1).contiguous())
                self.layers.append(("ssm", {
                    "layer": L,
                    "w_in": rnd(s.d_model, s.ssm_in, scale=s.d_model ** -0.5).to(bf),
                    "dt_bias": torch.full((s.nheads,), -2.0, device=self.device),
                    "w_out": rnd(s.nheads * s.headdim, s.d_model, scale=(s.nheads * s.headdim) ** -0.5).to(bf),
                    "y": torch.empty((s.batch, 1, s.nheads, s.headdim), dtype=torch.float32, device=self.device),
                }))
            qd, kvd = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim
            cap = s.context + max_steps
            self.layers.append(("attn", {
                "wq": rnd(s.d_model, qd, scale=s.d_model ** -0.5).to(bf),
                "wk": rnd(s.d_model, kvd, scale=s.d_model ** -0.5).to(bf),
                "wv": rnd(s.d_model, kvd, scale=s.d_model ** -0.5).to(bf),
                "wo": rnd(qd, s.d_model, scale=qd ** -0.5).to(bf),
                "k": rnd(s.batch, s.n_kv_heads, cap, s.head_dim, scale=1.0).to(bf),
                "v": rnd(s.batch, s.n_kv_heads, cap, s.head_dim, scale=1.0).to(bf),
            }))
        # torch's SDPA is held to its flash and memory-efficient kernels: its
        # default dispatch may pick a backend that builds an execution plan per
        # new sequence length, which a decode meets every step (tens of
        # milliseconds of host time per new length).
        from torch.nn.attention import SDPBackend, sdpa_kernel

        self._sdpa_backends = lambda: sdpa_kernel([SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION])
        self.pos = s.context  # next cache position
        self.cap = s.context + max_steps
        self.ssm_events = None  # a list here records CUDA events around every SSM decode call

    def _norm(self, x):
        xf = x.float()
        return (xf * self.torch.rsqrt(xf.pow(2).mean(dim=-1, keepdim=True) + 1e-6)).to(self.torch.bfloat16)

    def _ssm(self, x, p):
        torch, s = self.torch, self.s
        u = self._norm(x) @ p["w_in"]
        HP, H, GN = s.nheads * s.headdim, s.nheads, s.ngroups * s.dstate
        inputs = {
            "x": u[:, :HP].reshape(s.batch, 1, H, s.headdim).contiguous(),
            "dt": torch.nn.functional.softplus(u[:, HP:HP + H].float() + p["dt_bias"]).reshape(s.batch, 1, H)
                  .contiguous(),
            "B": u[:, HP + H:HP + H + GN].reshape(s.batch, 1, s.ngroups, s.dstate).contiguous(),
            "C": u[:, HP + H + GN:].reshape(s.batch, 1, s.ngroups, s.dstate).contiguous(),
        }
        if self.ssm_events is not None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            p["layer"].decode(inputs, y=p["y"])
            e1.record()
            self.ssm_events.append((e0, e1))
        else:
            p["layer"].decode(inputs, y=p["y"])
        return x + p["y"].reshape(s.batch, HP).to(torch.bfloat16) @ p["w_out"]

    def _attn(self, x, p):
        torch, s = self.torch, self.s
        xn = self._norm(x)
        # One decode token: the query heads that share a key/value head attend to
        # the same cache, so they are stacked as that head's query rows
        # ([batch, kv heads, query heads per kv head, head_dim]); query head j
        # uses key/value head j // (n_q_heads / n_kv_heads), as in grouped-query
        # attention, and no mask applies.
        q = (xn @ p["wq"]).reshape(s.batch, s.n_kv_heads, s.n_q_heads // s.n_kv_heads, s.head_dim)
        p["k"][:, :, self.pos] = (xn @ p["wk"]).reshape(s.batch, s.n_kv_heads, s.head_dim)
        p["v"][:, :, self.pos] = (xn @ p["wv"]).reshape(s.batch, s.n_kv_heads, s.head_dim)
        n = self.pos + 1
        with self._sdpa_backends():
            o = torch.nn.functional.scaled_dot_product_attention(q, p["k"][:, :, :n], p["v"][:, :, :n])
        return x + o.reshape(s.batch, s.n_q_heads * s.head_dim) @ p["wo"]

    def step(self, x):
        """One decode token for every sequence: hidden state x [batch, d_model] bf16 -> the next."""
        if self.pos >= self.cap:
            raise RuntimeError("the attention cache is full; build the stack with a larger max_steps")
        for kind, p in self.layers:
            x = self._ssm(x, p) if kind == "ssm" else self._attn(x, p)
        self.pos += 1
        return x

    def ssm_layers(self):
        return [p["layer"] for kind, p in self.layers if kind == "ssm"]
