"""The multi-GPU plumbing of bench.py and the head sharding, on CPU: gloo ranks, no GPU.

Heads are independent (per-head masks and attention), so N GPUs split a scale's heads with no
collective on the path: rank r owns a contiguous head range, draws exactly the bytes the
one-rank run draws for those heads, and an optional all-gather assembles O. Checked here with
world_size 2 over gloo: the partition, the shard inputs, the gathered outputs (per-head
compute stood in by the CPU oracle on a tiny case), the max-over-ranks reduction of timings
and the whole-job aggregation.
"""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _worker(rank, world, port, out):
    _init(rank, world, port)
    try:
        import bench
        from block_sparse_attention_tok_b200 import synth
        sc = synth.FINAL_CLIP2
        seeds = bench.rank_seeds(sc, rank)
        times = [10.0 + rank, 2.0 - rank, 5.0]             # rank 1 is slower on the first entry
        mx = bench.max_over_ranks(times, torch.device("cpu"), world)
        total = bench.sum_over_ranks(8.0e12 + rank * 1.0e12, torch.device("cpu"), world)
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        out[rank] = (mx, gathered, bench.whole_job_tflops(total, mx[0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_sum():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        mx, gathered, value = out[rank]
        assert mx == [11.0, 2.0, 5.0]
        assert set(gathered[0]).isdisjoint(gathered[1])     # weak scaling: distinct inputs per rank
        assert value == pytest.approx(17.0e12 / 11e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu"), 1) == [3.0, 4.0]
    assert bench.sum_over_ranks(5.0, torch.device("cpu"), 1) == 5.0
    assert bench.whole_job_tflops(1e12, 1.0) == pytest.approx(1000.0)


@pytest.mark.parametrize("heads", [1, 2, 3, 7, 32, 33])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_partition_covers_every_head_once(heads, world):
    from block_sparse_attention_tok_b200 import shard
    parts = shard.partition(world, heads)
    owned = [h for h0, h1 in parts for h in range(h0, h1)]
    assert owned == list(range(heads))                          # contiguous, in rank order, no repeats
    sizes = [h1 - h0 for h0, h1 in parts]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        shard.head_range(world, world, heads)


def _tiny_heads(n_heads):
    from block_sparse_attention_tok_b200 import synth
    # the tiny Clip-2 shape with per-head seeds, and an odd head count so the split is uneven
    return dataclasses.replace(synth.TINY_CLIP2, name="tiny_clip2_per_head_seeds", heads=n_heads)


def _oracle_forward(q, k, v, sc):
    """Per-head masks and attention of every query block (the CPU oracle), fp64 [H, Nq, d]."""
    from oracle import sparstar_oracle as O

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    out = []
    for h in range(q.shape[0]):
        qf, kf, vf = (O.bf16_bits_to_f64(bits(x[h])) for x in (q, k, v))
        rows, _ = O.select_head(qf, kf, sc.n_text, sc.n_ctx, sc.clip, sc.density)
        blocks = O.block_sparse_attention(qf, kf, vf, rows, range(rows.shape[0]))
        out.append(np.concatenate([o for o, _ in blocks]))
    return np.stack(out) if out else np.zeros((0, q.shape[1], q.shape[2]))


def _shard_worker(rank, world, port, n_heads, out):
    _init(rank, world, port)
    try:
        from block_sparse_attention_tok_b200 import shard
        sc = _tiny_heads(n_heads)
        q, k, v = shard.make_shard_inputs(sc, rank, world)
        o_local = torch.from_numpy(_oracle_forward(q, k, v, sc))
        o_all = shard.gather_heads(o_local, rank, world, sc.heads)
        q_all = shard.gather_heads(q, rank, world, sc.heads)
        out[rank] = (shard.head_range(rank, world, sc.heads), o_all.numpy(), q_all.view(torch.int16).numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_heads_and_gather_equals_one_rank():
    from block_sparse_attention_tok_b200 import synth
    world, n_heads = 2, 3
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_shard_worker, args=(world, _free_port(), n_heads, out), nprocs=world, join=True)
    sc = _tiny_heads(n_heads)
    q, k, v = synth.make_scale_inputs(sc)
    ref = _oracle_forward(q, k, v, sc)
    assert [out[r][0] for r in range(world)] == [(0, 2), (2, 3)]
    for r in range(world):
        _, o_all, q_bits = out[r]
        assert np.array_equal(q_bits, q.view(torch.int16).numpy())   # shards hold the one-rank bytes
        assert np.array_equal(o_all, ref)                            # gathered heads == one-rank result


def test_bench_gpus_n_starts_its_own_ranks():
    """`bench.py --gpus 2` without a torchrun environment spawns two ranks itself; on the
    reference arm (the CPU oracle) rank 0 alone prints one JSON line and the other rank exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "0", "--workload", "tiny_clip2_d64"], cwd=root, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert "fit in the 126 MB L2" in line["config"]["l2"]
