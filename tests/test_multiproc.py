"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks, no GPU.

Every rank runs its own full scale (weak scaling, no data-path collective). What the ranks
share is host-side: distinct per-rank seeds, the max-over-ranks reduction of timings, and
the whole-job aggregation. These are checked here with world_size 2 over gloo.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from block_sparse_attention_tok_b200 import synth
        sc = synth.FINAL_CLIP2
        seeds = bench.rank_seeds(sc, rank)
        times = [10.0 + rank, 2.0 - rank, 5.0]             # rank 1 is slower on the first entry
        mx = bench.max_over_ranks(times, torch.device("cpu"), world)
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        out[rank] = (mx, gathered, bench.whole_job_tflops(16.2e12, mx[0], world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_use_distinct_seeds():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        mx, gathered, value = out[rank]
        assert mx == [11.0, 2.0, 5.0]
        assert set(gathered[0]).isdisjoint(gathered[1])
        assert value == pytest.approx(2 * 16.2e12 / 11e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu"), 1) == [3.0, 4.0]
    assert bench.whole_job_tflops(1e12, 1.0, 1) == pytest.approx(1000.0)
