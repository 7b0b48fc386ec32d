"""Seeded synthetic inputs for the RecSA workloads.

This module draws random numbers and places them in the library's layouts; it
holds none of the method's arithmetic.  Both the CUDA path (through the tests
and the benchmark) and the CPU oracle consume the tensors it returns.

Layouts (row-major):
  K, V  [batch, n_kv_heads, capacity, head_dim]   bf16 or fp32
  Q     [batch, n_q, n_q_heads, head_dim]          same dtype
  r     [head_dim] fp32, one pooler reference vector per layer (shared by all
        KV heads and all levels)

Distributions (the workload definitions): K, V ~ N(0, 1), times a per-channel
scale sigma[g, c] ~ LogNormal(0, 0.5) per KV head for the model-shaped layers;
Q ~ N(0, 1); r ~ N(0, 1/d).  Planted needles: q_h = 4 * k_j + N(0, 1) with k_j
the key of head h's KV head at a random position j before the window;
mixtures: q_h = 2 * (k_j1 + k_j2 + k_j3 + k_j4) + N(0, 1).
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass
class Workload:
    name: str
    length: int                 # tokens in the cache (L)
    head_dim: int
    n_q_heads: int
    n_kv_heads: int
    leaf_block: int
    branching: int
    k: int
    window: int
    dtype: torch.dtype
    channel_scale: bool         # per-channel LogNormal(0, 0.5) scale on K, V
    batch: int = 1              # sequences
    n_q: int = 1                # queries per sequence
    needle_frac: float = 0.0
    mixture_frac: float = 0.0
    rope_base: float = 1e6
    extra: dict = field(default_factory=dict)


# The five workload shapes; the prefill / decode step counts live in `extra`.
WORKLOADS = {
    "tiny-4k": Workload("tiny-4k", 4096, 64, 4, 1, 16, 16, 4, 64, torch.float32,
                        False, batch=1, n_q=256, extra=dict(n_needles=16)),
    "qwen3-4b-131k": Workload("qwen3-4b-131k", 131072, 128, 32, 8, 64, 16, 8, 512,
                              torch.bfloat16, True, batch=1, n_q=1, needle_frac=0.01,
                              extra=dict(prefill_block=128, decode_steps=1024)),
    "qwen3-4b-524k": Workload("qwen3-4b-524k", 524288, 128, 32, 8, 64, 16, 8, 512,
                              torch.bfloat16, True, batch=4, n_q=1, needle_frac=0.01,
                              extra=dict(prefill_block=128, decode_steps=512)),
    "decode-1m": Workload("decode-1m", 1048576, 128, 32, 8, 64, 32, 8, 512,
                          torch.bfloat16, True, batch=8, n_q=1, needle_frac=0.02,
                          mixture_frac=0.10, extra=dict(decode_steps=256)),
    "stress-2m": Workload("stress-2m", 2097152, 128, 32, 8, 32, 8, 16, 1024,
                          torch.bfloat16, True, batch=1, n_q=1, needle_frac=0.0,
                          extra=dict(decode_steps=128, prefill_queries=65536)),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_kv(w: Workload, capacity: int, seed: int = 0, device="cpu",
            batch: Optional[int] = None):
    """K, V [batch, H_kv, capacity, d] and the pooler vector r [d] (fp32).

    Positions beyond ``w.length`` are drawn too (they are the tokens a decode
    run appends).
    """
    batch = w.batch if batch is None else batch
    g = _gen(seed, device)
    sk = sv = None
    if w.channel_scale:
        sk = torch.exp(0.5 * torch.randn((w.n_kv_heads, w.head_dim), generator=g,
                                         device=device))
        sv = torch.exp(0.5 * torch.randn((w.n_kv_heads, w.head_dim), generator=g,
                                         device=device))
    r = torch.randn((w.head_dim,), generator=g, device=device) / (w.head_dim ** 0.5)
    shape = (batch, w.n_kv_heads, capacity, w.head_dim)
    K = torch.empty(shape, dtype=w.dtype, device=device)
    V = torch.empty(shape, dtype=w.dtype, device=device)
    # one sequence at a time in fp32, so the peak memory is one sequence's worth
    for s in range(batch):
        for dst, scale in ((K, sk), (V, sv)):
            x = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
            if scale is not None:
                x.mul_(scale[:, None, :])
            dst[s].copy_(x)
            del x
    return K, V, r.float()


def make_queries(w: Workload, K: torch.Tensor, positions: torch.Tensor, seed: int = 1,
                 n_needles: Optional[int] = None):
    """Queries [batch, n, H_q, d] for query positions ``positions`` [batch, n].

    A fraction of the queries (or exactly ``n_needles``) are planted needles
    pointing at one random earlier key outside the window; another fraction are
    mixtures of four random earlier keys.  Returns (Q, kind) where kind
    [batch, n] is 0 plain, 1 needle, 2 mixture, and needle_pos [batch, n].
    """
    device = K.device
    g = _gen(seed, device)
    batch, n = positions.shape
    G = w.n_q_heads // w.n_kv_heads
    Q = torch.randn((batch, n, w.n_q_heads, w.head_dim), generator=g, device=device)
    u = torch.rand((batch, n), generator=g, device=device)
    kind = torch.zeros((batch, n), dtype=torch.int64, device=device)
    if n_needles is not None:
        perm = torch.randperm(batch * n, generator=g, device=device)[:n_needles]
        kind.view(-1)[perm] = 1
    else:
        kind[u < w.needle_frac] = 1
        kind[(u >= w.needle_frac) & (u < w.needle_frac + w.mixture_frac)] = 2
    span = (positions + 1 - w.window).clamp(min=1)             # j in [0, t+1-W)
    draws = torch.rand((batch, n, 4), generator=g, device=device)
    js = (draws * span[..., None].to(torch.float32)).long()
    js = torch.minimum(js, span[..., None] - 1).clamp(min=0)
    needle_pos = js[..., 0]
    Kf = K.float()
    bidx = torch.arange(batch, device=device)[:, None].expand(batch, n)
    heads = torch.arange(w.n_q_heads, device=device) // G      # KV head of each q head
    # Kf[b, g, j, :] for every (b, n, h)
    sel = Kf[bidx[..., None], heads[None, None, :], needle_pos[..., None], :]
    needle = 4.0 * sel
    mix = torch.zeros_like(Q)
    for m in range(4):
        mix += Kf[bidx[..., None], heads[None, None, :], js[..., m][..., None], :]
    mix = 2.0 * mix
    noise = Q
    Q = torch.where((kind == 1)[..., None, None], needle + noise, noise)
    Q = torch.where((kind == 2)[..., None, None], mix + noise, Q)
    return Q.to(w.dtype), kind, needle_pos
