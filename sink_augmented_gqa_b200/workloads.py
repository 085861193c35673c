"""Seeded synthetic workloads: the five attention configurations and their inputs.

This module holds shapes and random numbers only -- no attention arithmetic --
so that both the CUDA path (tests, bench) and the fp64 oracle can be fed the
very same bits from it.

Shapes follow the pages: gpt-oss GQA is 64 query heads, 8 KV heads, head
width 64, sm_scale 1/8, fused qkv width 5120 and a 128-token band on even
layers (GQA Attention study note, "How it works"); GPT-OSS-Lite is d_model
768, 8 heads, 4 KV heads, head width 96 (GPT-OSS-Lite visual guide,
"Architecture Specifications"); long context is YaRN-scaled to 131,072 from a
4,096 training context (MoE-Xtend README, "ROPE + SCALING"; the KV-byte
example at 24 layers and 131,072 tokens in "KV CACHE").

Value recipe (all synthetic): q/k/v bf16 ~ N(0, 1); sinks fp32 ~ N(0, std^2)
(std 1, or 0.5 for GPT-OSS-Lite); pre-filled cache rows bf16 ~ N(0, 1) taken
as already rotated. Each tensor draws from its own ``torch.Generator`` seeded
with ``seed * 1000 + stream`` so a tensor never depends on which others were
drawn before it.
"""

import math
from dataclasses import dataclass, field

import torch

YARN_DEFAULT = dict(theta=150000.0, scaling=32.0, orig_ctx=4096, alpha=1.0, beta=32.0)


@dataclass(frozen=True)
class AttnConfig:
    name: str
    B: int
    n_q: int
    n_kv: int
    d: int
    T: int                 # prefill rows of the call (0: decode-only)
    offset: int = 0        # cache rows already present before the prefill
    decode_steps: int = 0
    layers: int = 2        # layer l is windowed iff l % 2 == 0
    window: int = 128
    sm_scale: float = 0.125
    sink_std: float = 1.0
    seed: int = 0
    fused_qkv: bool = False
    yarn: dict = field(default_factory=lambda: dict(YARN_DEFAULT))

    @property
    def q_mult(self):
        return self.n_q // self.n_kv

    @property
    def max_pos(self):
        return self.offset + self.T + self.decode_steps

    @property
    def cap(self):
        return self.offset + self.T + self.decode_steps

    def layer_window(self, layer):
        return self.window if layer % 2 == 0 else 0


CONFIGS = {
    # B=1, T=64 prompt then 16 decode steps, 8/2/64, W=16 band + full pair.
    "tiny": AttnConfig("tiny", B=1, n_q=8, n_kv=2, d=64, T=64, decode_steps=16,
                       window=16, sm_scale=1.0 / 8, seed=0),
    # GPT-OSS-Lite attention shapes: B=8, T=4096, 8/4/96.
    "lite": AttnConfig("lite", B=8, n_q=8, n_kv=4, d=96, T=4096,
                       sm_scale=1.0 / math.sqrt(96.0), sink_std=0.5, seed=1),
    # gpt-oss prefill: B=1, T=8192, 64/8/64 from a fused qkv [1, 8192, 5120].
    "gptoss_prefill": AttnConfig("gptoss_prefill", B=1, n_q=64, n_kv=8, d=64, T=8192,
                                 sm_scale=1.0 / 8, seed=2, fused_qkv=True),
    # Long-context decode: cache pre-filled to 131071 rows, 24 layers, 64 steps.
    "long_decode": AttnConfig("long_decode", B=1, n_q=64, n_kv=8, d=64, T=0,
                              offset=131071, decode_steps=64, layers=24,
                              sm_scale=1.0 / 8, seed=3),
    # Prefill-to-decode handoff: B=16 at offset 65536, +512 chunk, 32 decode steps.
    "handoff": AttnConfig("handoff", B=16, n_q=64, n_kv=8, d=64, T=512,
                          offset=65536, decode_steps=32, sm_scale=1.0 / 8, seed=4),
}


def _gen(seed, stream, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + int(stream))
    return g


def randn_bf16(shape, seed, stream, device="cpu"):
    """bf16 tensor of N(0,1) draws (drawn in fp32, rounded to bf16)."""
    g = _gen(seed, stream, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def sinks(cfg, layer=0, device="cpu"):
    g = _gen(cfg.seed, 100 + layer, device)
    return (torch.randn(cfg.n_q, generator=g, device=device, dtype=torch.float32)
            * cfg.sink_std)


def qkv(cfg, T, layer=0, step=0, device="cpu"):
    """(q, k, v) for T new rows of one layer at one step.

    q [B,T,n_q,d], k/v [B,T,n_kv,d]. With ``fused_qkv`` the three are strided
    views into one [B, T, d*(n_q + 2*n_kv)] tensor, as a fused qkv projection
    would produce them.
    """
    stream = 200 + 1000 * step + layer
    B, n_q, n_kv, d = cfg.B, cfg.n_q, cfg.n_kv, cfg.d
    if cfg.fused_qkv:
        width = d * (n_q + 2 * n_kv)
        x = randn_bf16((B, T, width), cfg.seed, stream, device)
        q = x[:, :, : n_q * d].unflatten(2, (n_q, d))
        k = x[:, :, n_q * d:(n_q + n_kv) * d].unflatten(2, (n_kv, d))
        v = x[:, :, (n_q + n_kv) * d:].unflatten(2, (n_kv, d))
        return q, k, v
    q = randn_bf16((B, T, n_q, d), cfg.seed, stream, device)
    k = randn_bf16((B, T, n_kv, d), cfg.seed, stream + 1_000_000, device)
    v = randn_bf16((B, T, n_kv, d), cfg.seed, stream + 2_000_000, device)
    return q, k, v


def prefilled_cache_rows(cfg, layer=0, device="cpu", rows=None):
    """Random bf16 K/V rows [B, rows, n_kv, d] standing for an already-filled
    (already rotated) cache prefix of ``cfg.offset`` rows."""
    rows = cfg.offset if rows is None else rows
    shape = (cfg.B, rows, cfg.n_kv, cfg.d)
    k = randn_bf16(shape, cfg.seed, 50_000 + layer, device)
    v = randn_bf16(shape, cfg.seed, 60_000 + layer, device)
    return k, v


def scaled(cfg, **changes):
    """A copy of ``cfg`` with some fields replaced (smaller parity cases)."""
    d = dict(cfg.__dict__)
    d.update(changes)
    return AttnConfig(**d)
