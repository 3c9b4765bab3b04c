"""Seeded synthetic inputs for one expensive SparSTAR scale.

This module only draws random tensors and describes workload shapes. It holds none of
the method's arithmetic (no pooling, scoring, selection or attention), so both the CUDA
path and the CPU oracle's tests may use it.

Workloads follow the token mixes of the SparSTAR digest ("SparSTAR的贡献：每尺度动态重建",
pchao.org), sections 这篇论文解决什么问题 (about 72,000 tokens at the 720p final scale; KV =
text ‖ reference context ‖ current-scale tokens) and 核心创新 (density schedule
0.625 / 0.1875 / 0.1875 / 0.09375), with 32 heads of width 128 per InfinityStar layer
(Figure 3 caption: 36 layers and 32 heads). The activations the pages measure on come from
the trained InfinityStar 8B model on VBench prompts; neither exists here, so these seeded
Gaussian tensors stand in for them.

Value recipe, per head, drawn in this order from one generator:
  q ~ N(0, 1)        [Nq, d]
  k ~ N(0, 1)        [Nkv, d]
  off ~ N(0, 0.5)    [ceil(Nkv/128), d]   (standard deviation 0.5)
  k[t] += off[t // 128]                    (one offset vector per 128-token KV block,
                                            text blocks and a ragged last block included)
  v ~ N(0, 1)        [Nkv, d]
Each draw is fp32, rounded to bf16 (round to nearest even). The same seed gives different
values on a CPU and a CUDA generator; parity is always checked on the bytes actually used.
"""
from __future__ import annotations

import dataclasses
from typing import Iterator, List, Optional, Tuple

import torch

TOKENS_PER_BLOCK = 128  # block edge of the pages' block partition (方法概览)


@dataclasses.dataclass(frozen=True)
class Scale:
    """Shape of one expensive scale: KV = n_text ‖ n_ctx ‖ n_cur tokens; Q = current tokens."""

    name: str
    heads: int
    head_dim: int
    n_q: int
    n_text: int
    n_ctx: int
    n_cur: int
    clip: int          # 1 = first clip (ctx is the image pyramid), >= 2 = later clip (ctx is the preceding clip's final scale)
    density: float
    layers: int = 1
    grid: Optional[Tuple[int, int, int]] = None   # (frames, height, width) of the current tokens

    @property
    def n_kv(self) -> int:
        return self.n_text + self.n_ctx + self.n_cur

    def seed(self, head: int, layer: int = 0, scale_index: int = 0, cfg_index: int = 0) -> int:
        """Per-head seed; the tiny case uses one generator for all heads (seed 0)."""
        if self.layers > 1:
            return 100000 + 1000 * layer + 100 * scale_index + head
        return 1000 * cfg_index + head


# The five workloads. Q is always the current-scale tokens.
TINY_CLIP2 = Scale("tiny_clip2_d64", heads=2, head_dim=64, n_q=1024, n_text=256, n_ctx=768,
                   n_cur=1024, clip=2, density=0.25)
MID_CLIP1 = Scale("mid_refined_clip1_18k", heads=32, head_dim=128, n_q=18432, n_text=512,
                  n_ctx=4096, n_cur=18432, clip=1, density=0.1875)
FINAL_CLIP1_RAGGED = Scale("final720p_clip1_72000_ragged", heads=32, head_dim=128, n_q=72000,
                           n_text=512, n_ctx=8192, n_cur=72000, clip=1, density=0.09375)
FINAL_CLIP2 = Scale("final720p_clip2_72192", heads=32, head_dim=128, n_q=72192, n_text=512,
                    n_ctx=72192, n_cur=72192, clip=2, density=0.09375)
# Full refined-scale schedule of one clip: 36 layers x 32 heads at four scales. The pages give
# the token counts' scale (about 72,000 at the 720p final scale) but no latent grid shapes; the
# grids here (8 latent frames, growing height x width) only lay the synthetic current tokens out
# in raster order for the cross-scale block map.
SCHEDULE_CLIP1: Tuple[Scale, ...] = tuple(
    Scale(f"schedule_clip1_s{i + 1}_{n}", heads=32, head_dim=128, n_q=n, n_text=512, n_ctx=8192,
          n_cur=n, clip=1, density=dens, layers=36, grid=grid)
    for i, (n, dens, grid) in enumerate(((8192, 0.625, (8, 32, 32)), (18432, 0.1875, (8, 48, 48)),
                                         (36864, 0.1875, (8, 64, 72)), (72192, 0.09375, (8, 94, 96))))
)

WORKLOADS = {s.name: s for s in (TINY_CLIP2, MID_CLIP1, FINAL_CLIP1_RAGGED, FINAL_CLIP2) + SCHEDULE_CLIP1}
CFG_INDEX = {TINY_CLIP2.name: 1, MID_CLIP1.name: 2, FINAL_CLIP1_RAGGED.name: 3, FINAL_CLIP2.name: 4}


def _draw_head(gen: torch.Generator, n_q: int, n_kv: int, d: int, device, offset_std: float = 0.5):
    nkb = -(-n_kv // TOKENS_PER_BLOCK)
    q = torch.randn(n_q, d, generator=gen, device=device, dtype=torch.float32)
    k = torch.randn(n_kv, d, generator=gen, device=device, dtype=torch.float32)
    off = torch.randn(nkb, d, generator=gen, device=device, dtype=torch.float32) * offset_std
    k += off.repeat_interleave(TOKENS_PER_BLOCK, dim=0)[:n_kv]
    v = torch.randn(n_kv, d, generator=gen, device=device, dtype=torch.float32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_qkv(n_q: int, n_kv: int, heads: int, d: int, seeds: List[int], device="cpu",
             one_generator: bool = False, offset_std: float = 0.5):
    """Allocate contiguous bf16 q [H,Nq,d], k [H,Nkv,d], v [H,Nkv,d] and fill them per head.

    seeds[h] seeds head h; with one_generator=True a single generator seeded seeds[0]
    draws all heads in order.
    """
    q = torch.empty(heads, n_q, d, dtype=torch.bfloat16, device=device)
    k = torch.empty(heads, n_kv, d, dtype=torch.bfloat16, device=device)
    v = torch.empty(heads, n_kv, d, dtype=torch.bfloat16, device=device)
    gen = torch.Generator(device=device)
    if one_generator:
        gen.manual_seed(int(seeds[0]))
    for h in range(heads):
        if not one_generator:
            gen.manual_seed(int(seeds[h]))
        qh, kh, vh = _draw_head(gen, n_q, n_kv, d, device, offset_std)
        q[h].copy_(qh)
        k[h].copy_(kh)
        v[h].copy_(vh)
    return q, k, v


def make_scale_inputs(scale: Scale, device="cpu", layer: int = 0, scale_index: int = 0,
                      heads: Optional[int] = None):
    """Inputs of a named workload (all heads unless `heads` limits them)."""
    H = scale.heads if heads is None else heads
    if scale.name == TINY_CLIP2.name:
        return make_qkv(scale.n_q, scale.n_kv, H, scale.head_dim, [0], device, one_generator=True)
    cfg = CFG_INDEX.get(scale.name, 0)
    seeds = [scale.seed(h, layer, scale_index, cfg) for h in range(H)]
    return make_qkv(scale.n_q, scale.n_kv, H, scale.head_dim, seeds, device)


def make_prev_clip_queries(n_q: int, heads: int, d: int, seeds: List[int], device="cpu") -> torch.Tensor:
    """Queries of the preceding clip's final scale (same shape as the current queries), for the
    reference-reuse comparison: bf16 [H, Nq, d], N(0,1) per element, one generator per head
    seeded seeds[h]. Drawn independently of the current clip's inputs (the synthetic inputs
    carry no correlation between clips)."""
    q = torch.empty(heads, n_q, d, dtype=torch.bfloat16, device=device)
    gen = torch.Generator(device=device)
    for h in range(heads):
        gen.manual_seed(int(seeds[h]))
        q[h].copy_(torch.randn(n_q, d, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16))
    return q


def random_small_cases(seed: int = 1234, count: int = 12) -> Iterator[dict]:
    """Small ragged shapes for parity sweeps: H in {1,2}, d in {64,128}, ragged Q/KV tails."""
    g = torch.Generator().manual_seed(seed)

    def pick(options):
        return options[int(torch.randint(len(options), (1,), generator=g))]

    for i in range(count):
        d = pick([64, 128])
        H = pick([1, 2])
        tail_q = pick([0, 1, 64, 127])
        tail_kv = pick([0, 1, 64, 127])
        n_q = 128 * pick([1, 2, 3, 5]) + tail_q - (128 if tail_q else 0)
        n_q = max(n_q, 1)
        n_text = pick([0, 128, 256, 200])
        n_ctx = pick([0, 128, 384, 300])
        n_cur = 128 * pick([1, 2, 4, 6]) + tail_kv
        clip = pick([1, 2])
        density = pick([0.0625, 0.25, 0.5, 0.75, 1.0])
        mode = pick([0, 1])
        yield dict(name=f"small{i}", H=H, d=d, n_q=n_q, n_text=n_text, n_ctx=n_ctx,
                   n_cur=n_cur, clip=clip, density=density, mode=mode, seed=seed + i)

