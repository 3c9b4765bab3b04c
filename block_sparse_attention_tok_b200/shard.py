"""Head-parallel sharding of one scale across GPUs (one process per GPU).

Every head has its own dynamic mask and its own attention (SparSTAR digest
"SparSTAR的贡献：每尺度动态重建", section 方法概览, bullet per-head动态掩码), so a scale splits
across ranks by heads with no exchange on the path: rank r of N takes the contiguous heads
[r*H/N, (r+1)*H/N) (the first H mod N ranks one more when H is not a multiple of N), runs
selection and attention on that slice, and nothing else crosses between ranks. Gathering O
afterwards is optional (a caller whose next layer needs every head) and is one all-gather.

Host logic only: which heads a rank owns, the rank's inputs (the same bytes the one-rank
run draws for those heads), and the optional gather. The per-head compute is the library's.
"""
from __future__ import annotations

from typing import List, Tuple

import torch

from . import synth


def head_range(rank: int, world: int, heads: int) -> Tuple[int, int]:
    """[h0, h1) of the heads rank `rank` of `world` owns: contiguous, sizes differing by at most
    one, the larger shares first. A rank may own no head when world > heads."""
    if world < 1 or not 0 <= rank < world or heads < 0:
        raise ValueError(f"bad partition: rank {rank} of {world}, {heads} heads")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def partition(world: int, heads: int) -> List[Tuple[int, int]]:
    """Every rank's head range, in rank order."""
    return [head_range(r, world, heads) for r in range(world)]


def make_shard_inputs(scale: synth.Scale, rank: int, world: int, device="cpu", layer: int = 0,
                      scale_index: int = 0):
    """q, k, v of this rank's heads of a named workload: head h gets exactly the bytes it has in
    the one-rank inputs (per-head seeds; a workload drawn from one generator is drawn whole and
    sliced)."""
    h0, h1 = head_range(rank, world, scale.heads)
    if scale.name == synth.TINY_CLIP2.name:
        q, k, v = synth.make_scale_inputs(scale, device=device, layer=layer, scale_index=scale_index)
        return q[h0:h1].contiguous(), k[h0:h1].contiguous(), v[h0:h1].contiguous()
    cfg = synth.CFG_INDEX.get(scale.name, 0)
    seeds = [scale.seed(h, layer, scale_index, cfg) for h in range(h0, h1)]
    return synth.make_qkv(scale.n_q, scale.n_kv, h1 - h0, scale.head_dim, seeds, device)


def gather_heads(local: torch.Tensor, rank: int, world: int, heads: int, group=None) -> torch.Tensor:
    """All-gather of per-rank head slices [h1 - h0, ...] into the full [heads, ...] tensor on every
    rank (one collective; slices are padded to the largest share, then trimmed). world == 1
    returns `local` itself."""
    if world == 1:
        return local
    import torch.distributed as dist
    parts = partition(world, heads)
    width = max(h1 - h0 for h0, h1 in parts)
    tail = tuple(local.shape[1:])
    padded = torch.zeros((width,) + tail, dtype=local.dtype, device=local.device)
    h0, h1 = parts[rank]
    if h1 > h0:
        padded[: h1 - h0].copy_(local)
    out = torch.empty((world * width,) + tail, dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(out, padded, group=group)
    return torch.cat([out[r * width: r * width + (b - a)] for r, (a, b) in enumerate(parts)])
