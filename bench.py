"""Benchmark of one expensive SparSTAR scale on B200: selection + block-sparse attention.

A step is the whole per-scale path (pooling, scores, Top-K, attention over the kept tiles)
over one 720p final-scale Clip-2 input (32 heads, d 128, 72,192 query tokens, KV 512 text +
72,192 preceding-clip + 72,192 current tokens, density 0.09375), inputs resident in HBM.

With N GPUs (one process per GPU, NCCL for the barrier and the timing reduction only) the
default is strong scaling: rank r owns heads [r*H/N, (r+1)*H/N) of the one input and runs the
path on them, with no collective on the path (heads are independent). `--scaling weak`
instead gives every rank its own full scale. Without a torchrun environment, `--gpus N > 1`
starts its own N ranks.

Prints one JSON line (rank 0). Timed region: barrier + synchronize, K steps bracketed by
CUDA events on the launch stream, synchronize + barrier; the max over ranks is reported.
Inputs (q, k, v: 2.97 GB at the 720p scale) are far larger than L2 (126 MB), so no flush is
inserted; the config's `l2` key states it for the run.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--scaling strong|weak]
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import math
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_attention_tok_b200 import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HBM_SPEC_GBS = 7700.0   # HGX B200 nominal HBM3e bandwidth
L2_BYTES = 126 * 1000 * 1000
METRIC = "sparse-attn TFLOP/s on kept tiles & % of bf16 peak; select GB/s; µs per scale"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--scaling", choices=["strong", "weak"], default="strong",
                    help="strong: the ranks split the heads of one input; weak: every rank runs a full scale")
    ap.add_argument("--gather-o", action="store_true",
                    help="N > 1: also time one all-gather of O across ranks (outside the step)")
    ap.add_argument("--workload", default=synth.FINAL_CLIP2.name, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--budget-mode", type=int, default=0)
    ap.add_argument("--heads", type=int, default=0, help="limit the heads (profiling small cases); 0 = all")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-block64", action="store_true", help="skip the 64-token block variant")
    ap.add_argument("--no-reuse", action="store_true",
                    help="skip the fresh vs reused reference-selection comparison")
    ap.add_argument("--no-schedule", action="store_true",
                    help="skip the per-scale timing of the refined-scale schedule (4 scales x 36 layers)")
    return ap.parse_args()


# the attention kernel's device code and the host code that picks its launch (grid size)
ATTN_SOURCES = ("attn_sm100.cuh", "ptx.cuh", "sparstar.cu")


def kernel_source_hash(sources=ATTN_SOURCES) -> str:
    """sha256 (first 16 hex digits) of the CUDA sources a kernel is built from (by default the
    attention kernel's, which keys its DRAM traffic record)."""
    import hashlib
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "block_sparse_attention_tok_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture of this exact source, else None.

    profiles/traffic.txt lines: <source hash> <kernel> <workload> <bytes per launch> <note...>
    """
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == want and parts[1] == kernel \
                    and parts[2] == workload:
                return float(parts[3])
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every 20 ms (reads only)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: no clock record
            self._nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- accounting

def kept_tile_flops(idx: torch.Tensor, cnt: torch.Tensor, n_q: int, n_kv: int, d: int, block: int = 128) -> float:
    """4 d * sum over kept tiles of valid_query_rows * valid_kv_tokens (bookkeeping only)."""
    H, nqb, kmax = idx.shape
    col = torch.arange(kmax, device=idx.device)
    live = col[None, None, :] < cnt[:, :, None]
    nkb = -(-n_kv // block)
    vk = torch.where(idx == nkb - 1, n_kv - (nkb - 1) * block, block).to(torch.float64)
    per_row = (vk * live).sum(-1)
    vq = torch.full((nqb,), float(block), dtype=torch.float64, device=idx.device)
    vq[-1] = n_q - (nqb - 1) * block
    return float(4.0 * d * (per_row * vq[None, :]).sum().item())


# ----------------------------------------------------------------------------- ranks

def rank_seeds(sc, rank: int):
    """Seeds of one rank's heads under weak scaling: every rank works on its own full scale."""
    return [1000 * synth.CFG_INDEX.get(sc.name, 0) + h + 100000 * rank for h in range(sc.heads)]


def sum_over_ranks(value: float, device, world: int) -> float:
    """Sum of a per-rank quantity (a no-op on one rank)."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(values, device, world: int):
    """Elementwise max of per-rank timings (a no-op on one rank)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(flops_all_ranks: float, ms_max: float) -> float:
    """Aggregate throughput: the units all ranks processed over the slowest rank's time."""
    return flops_all_ranks / (ms_max * 1e-3) / 1e12


def read_bandwidth_probe(S, dev, nbytes: int = 4 << 30, reps: int = 5) -> float:
    """Best read-only streaming rate (GB/s) over a buffer far larger than L2: the library's read
    probe (the pooling kernel's 16-byte streaming loads, nothing written), CUDA events. The
    denominator for the selection, whose traffic is almost all reads, next to the copy figure
    (read + write)."""
    x = torch.zeros(nbytes // 4, dtype=torch.float32, device=dev)
    sink = S.read_probe(x)
    best = 0.0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        S.read_probe(x, sink)
        b.record()
        torch.cuda.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del x, sink
    torch.cuda.empty_cache()
    return best


# ----------------------------------------------------------------------------- CPU oracle

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(q, k, v, sc, heads, q_sample, budget_mode):
    """The oracle's whole path on a bounded sample: for each listed head, widen its bf16
    inputs, run its full selection, and run attention for q_sample evenly spaced query
    blocks. Returns (kept-tile FLOPs of the sampled blocks, seconds, prorated seconds)."""
    from oracle import sparstar_oracle as O

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    flops, t_total, t_pro = 0.0, 0.0, 0.0
    nqb = O.num_blocks(sc.n_q)
    pick = np.unique(np.linspace(0, nqb - 1, min(q_sample, nqb)).round().astype(int))
    for h in heads:
        qh, kh, vh = (x[h].cpu() for x in (q, k, v))
        t0 = time.perf_counter()
        qf, kf, vf = (O.bf16_bits_to_f64(bits(x)) for x in (qh, kh, vh))
        rows, _ = O.select_head(qf, kf, sc.n_text, sc.n_ctx, sc.clip, sc.density, budget_mode)
        t1 = time.perf_counter()
        O.block_sparse_attention(qf, kf, vf, rows, pick)
        t2 = time.perf_counter()
        for i in pick:
            s, e = O.block_token_range(int(i), sc.n_q)
            vk = sum(b - a for a, b in (O.block_token_range(int(j), sc.n_kv) for j in rows[i]))
            flops += 4.0 * sc.head_dim * (e - s) * vk
        t_total += t2 - t0
        t_pro += (t1 - t0) * len(pick) / nqb + (t2 - t1)
    return flops, t_total, t_pro


# ----------------------------------------------------------------------------- arms

def run_reference(args, rank):
    """--impl reference: the CPU oracle, as it stands, on a bounded sample per step."""
    if rank != 0:
        return 0
    sc = synth.WORKLOADS[args.workload]
    q_sample = 48
    heads_total = sc.heads
    vals, times = [], []
    for step in range(args.warmup + args.steps):
        h = step % heads_total
        seed = 1000 * synth.CFG_INDEX.get(sc.name, 0) + h
        q, k, v = synth.make_qkv(sc.n_q, sc.n_kv, 1, sc.head_dim, [seed], device="cpu")
        flops, t, t_pro = oracle_sample(q, k, v, sc, [0], q_sample, args.budget_mode)
        if step >= args.warmup:
            vals.append(flops / t_pro / 1e12)
            times.append(t)
        del q, k, v
    value = float(np.mean(vals))
    cores = _blas_threads()
    sample = (f"per step one head (cycling 0..{heads_total - 1}): bf16 widening + full selection of that head "
              f"(prorated to the sampled rows) + attention of {q_sample} evenly spaced query blocks; fp64 numpy")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": float(np.mean(times) * 1e3), "higher_is_better": True,
        "scaling": args.scaling, "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(sc, args, 1), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(sc, args, world):
    if args.scaling == "strong":
        per_gpu = f"heads [r*{sc.heads}/{world}, (r+1)*{sc.heads}/{world}) of one input per rank r, no collective on the path"
        par = f"heads/{world}"
    else:
        per_gpu = "one full scale (all heads) per rank"
        par = f"replicas x{world}"
    return {"workload": sc.name, "heads": sc.heads, "head_dim": sc.head_dim, "n_q": sc.n_q,
            "kv": {"text": sc.n_text, "ctx": sc.n_ctx, "cur": sc.n_cur}, "clip": sc.clip,
            "density": sc.density, "budget": "literal" if args.budget_mode == 0 else "candidates",
            "block": 128, "per_gpu": per_gpu, "l2": l2_note(sc, world, args.scaling), "parallelism": par}


def l2_note(sc, world, scaling):
    """How the timed steps stand to the 126 MB L2: a rank's q, k, v either exceed it (no flush
    needed between steps) or fit in it (then they are said to stay resident)."""
    heads = -(-sc.heads // world) if scaling == "strong" else sc.heads
    nbytes = heads * (sc.n_q + 2 * sc.n_kv) * sc.head_dim * 2
    if nbytes > L2_BYTES:
        return f"no flush: inputs {nbytes / 1e9:.2f} GB per rank > 126 MB L2"
    return f"inputs {nbytes / 1e6:.1f} MB per rank fit in the 126 MB L2 (not flushed)"


def run_schedule(S, dev, stream, layers: int = 36):
    """Per-scale time of the refined-scale schedule of one clip (Clip 1): for each of the four
    sparsified scales and each layer, fresh seeded inputs (untimed), then selection +
    attention timed with CUDA events on resident inputs. Both budget readings; plus one
    density-1 (dense) attention per scale through the same kernel, for context."""
    out = {"workload": "refined-scale schedule, Clip 1: 4 scales x %d layers x 32 heads, d 128" % layers,
           "modes": {}, "dense_ms_per_layer": {}}
    for mode in (0, 1):
        rows = []
        for si, sc in enumerate(synth.SCHEDULE_CLIP1):
            plan = S.make_plan(sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density, mode)
            kmax = int(plan.k_total)
            ws = S.Workspace(sc.heads, sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.head_dim, dev)
            idx = torch.empty(sc.heads, int(plan.nqb), kmax, dtype=torch.int32, device=dev)
            cnt = torch.empty(sc.heads, int(plan.nqb), dtype=torch.int32, device=dev)
            t_sel, t_att, flops = [], [], 0.0
            for layer in range(layers):
                q, k, v = synth.make_scale_inputs(sc, device=dev, layer=layer, scale_index=si)
                o, lse = torch.empty_like(q), torch.empty(sc.heads, sc.n_q, dtype=torch.float32, device=dev)
                seg = (sc.n_text, sc.n_ctx, sc.n_cur)
                if layer == 0:  # warm-up of this shape
                    S.select(q, k, *seg, sc.clip, sc.density, mode, workspace=ws, idx=idx, cnt=cnt)
                    S.attn(q, k, v, idx, cnt, o=o, lse=lse)
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                torch.cuda.synchronize()
                ev[0].record(stream)
                S.select(q, k, *seg, sc.clip, sc.density, mode, workspace=ws, idx=idx, cnt=cnt)
                ev[1].record(stream)
                S.attn(q, k, v, idx, cnt, o=o, lse=lse)
                ev[2].record(stream)
                torch.cuda.synchronize()
                t_sel.append(ev[0].elapsed_time(ev[1]))
                t_att.append(ev[1].elapsed_time(ev[2]))
                flops += kept_tile_flops(idx, cnt, sc.n_q, sc.n_kv, sc.head_dim)
                if mode == 0 and layer == 0:
                    dplan = S.make_plan(sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, 1.0)
                    didx = torch.arange(int(dplan.nkb), dtype=torch.int32, device=dev).expand(
                        sc.heads, int(dplan.nqb), int(dplan.nkb)).contiguous()
                    dcnt = torch.full((sc.heads, int(dplan.nqb)), int(dplan.nkb), dtype=torch.int32, device=dev)
                    S.attn(q, k, v, didx, dcnt, o=o, lse=lse)
                    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    d0.record(stream)
                    S.attn(q, k, v, didx, dcnt, o=o, lse=lse)
                    d1.record(stream)
                    torch.cuda.synchronize()
                    out["dense_ms_per_layer"][sc.name] = d0.elapsed_time(d1)
                    del didx, dcnt
                del q, k, v, o, lse
            ms_total = float(np.sum(t_sel) + np.sum(t_att))
            rows.append({"scale": sc.name, "n_q": sc.n_q, "n_kv": sc.n_kv, "density": sc.density,
                         "k_total": int(plan.k_total), "k_topk": int(plan.k_topk),
                         "ms_all_layers": ms_total, "us_per_layer": ms_total * 1e3 / layers,
                         "select_us_per_layer": float(np.mean(t_sel)) * 1e3,
                         "attn_us_per_layer": float(np.mean(t_att)) * 1e3,
                         "attn_tflops": flops / (float(np.sum(t_att)) * 1e-3) / 1e12,
                         "selection_share": float(np.sum(t_sel)) / ms_total})
            del ws, idx, cnt
        out["modes"]["literal" if mode == 0 else "candidates"] = {
            "scales": rows, "ms_schedule": float(sum(r["ms_all_layers"] for r in rows))}
    torch.cuda.empty_cache()
    return out


def run_cross_scale(S, dev, stream):
    """Mask reuse across scales (recompute frequency): the four sparsified scales of the Clip-1
    schedule (layer 0, 32 heads, candidates reading: under the literal reading scales 2-4 keep
    only the forced prefix, so every policy gives the same masks), under three policies:
    recompute at every scale, every second scale, or once at the first scale. Per policy and
    scale: the mean retained dense softmax mass of the mask and the selection time (fresh
    selection, or score map + Top-K)."""
    from block_sparse_attention_tok_b200 import reuse
    mode = S.BUDGET_CANDIDATES
    scales, lse_dense = [], []
    for si, sc in enumerate(synth.SCHEDULE_CLIP1):
        q, k, v = synth.make_scale_inputs(sc, device=dev, layer=0, scale_index=si)
        scales.append(dict(q=q, k=k, v=v, seg=(sc.n_text, sc.n_ctx, sc.n_cur), grid=sc.grid, clip=sc.clip,
                           density=sc.density))
        nqb, nkb = -(-sc.n_q // 128), -(-sc.n_kv // 128)
        all_idx = torch.arange(nkb, dtype=torch.int32, device=dev).expand(sc.heads, nqb, nkb).contiguous()
        all_cnt = torch.full((sc.heads, nqb), nkb, dtype=torch.int32, device=dev)
        _, lse = S.attn(q, k, v, all_idx, all_cnt)
        lse_dense.append(lse)
        del all_idx, all_cnt
    out = {"workload": "Clip-1 schedule, layer 0, 32 heads; grids (frames, height, width) " +
                       ", ".join(str(sc.grid) for sc in synth.SCHEDULE_CLIP1),
           "budget": "candidates", "policies": {}}
    reuse.cross_scale_masks(scales, "every_2", mode)   # warm-up
    for policy in reuse.POLICIES:
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        masks = reuse.cross_scale_masks(scales, policy, mode)
        b.record(stream)
        torch.cuda.synchronize()
        rows = []
        for sc, (idx, cnt), ld in zip(scales, masks, lse_dense):
            _, lse_kept = S.attn(sc["q"], sc["k"], sc["v"], idx, cnt)
            _, e = S.retained_mass(lse_kept, ld, want_tokens=False)
            rows.append(float(e.mean()))
        out["policies"][policy] = {"retained_mean_per_scale": rows, "selection_ms_all_scales": a.elapsed_time(b)}
        del masks
    del scales, lse_dense
    torch.cuda.empty_cache()
    out["note"] = ("synthetic inputs are independent across scales, so reused masks act as uninformed ones; "
                   "the pages' Figure 5 differences (1.73 / 0.79 dB) come from model activations")
    return out


def run_ours(args, rank, world, local_rank):
    from block_sparse_attention_tok_b200 import sparstar as S
    import torch.distributed as dist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    S.load()
    from block_sparse_attention_tok_b200 import shard
    sc_full = synth.WORKLOADS[args.workload]
    if args.heads:
        sc_full = dataclasses.replace(sc_full, heads=args.heads)
    if args.scaling == "strong":
        # every rank takes the same decision here, before any collective, so none is left waiting
        if world > sc_full.heads:
            raise SystemExit(f"{sc_full.heads} heads cannot be split over {world} ranks: every rank needs a head")
        # this rank's heads of the one input (the same bytes the one-rank run draws for them)
        h0, h1 = shard.head_range(rank, world, sc_full.heads)
        q, k, v = shard.make_shard_inputs(sc_full, rank, world, device=dev)
    else:
        h0, h1 = 0, sc_full.heads
        q, k, v = synth.make_qkv(sc_full.n_q, sc_full.n_kv, sc_full.heads, sc_full.head_dim,
                                 rank_seeds(sc_full, rank), device=dev)
    sc = dataclasses.replace(sc_full, heads=h1 - h0)   # what this rank computes
    plan = S.make_plan(sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density, args.budget_mode)
    kmax = int(plan.k_total)
    ws = S.Workspace(sc.heads, sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.head_dim, dev)
    idx = torch.empty(sc.heads, int(plan.nqb), kmax, dtype=torch.int32, device=dev)
    cnt = torch.empty(sc.heads, int(plan.nqb), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(sc.heads, sc.n_q, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    seg = (sc.n_text, sc.n_ctx, sc.n_cur)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        S.select(q, k, *seg, sc.clip, sc.density, args.budget_mode, workspace=ws, idx=idx, cnt=cnt)
        if ev is not None:
            ev[1].record(stream)
        S.attn(q, k, v, idx, cnt, o=o, lse=lse)
        if ev is not None:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            t = torch.zeros(1, device=dev)
            dist.all_reduce(t)
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    assert S.device_status() == S.OK
    flops = kept_tile_flops(idx, cnt, sc.n_q, sc.n_kv, sc.head_dim)
    launches_per_step = (3 if 0 < plan.k_topk < plan.n_cand else 1) + 1
    sel_bytes = 2.0 * sc.heads * sc.head_dim * (sc.n_q + sc.n_kv) + 4.0 * sc.heads * plan.nqb * (kmax + 1)
    if plan.k_topk == 0 or plan.k_topk == plan.n_cand:
        sel_bytes = 4.0 * sc.heads * plan.nqb * (kmax + 1)   # rows do not depend on the inputs

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local_rank) as clocks:
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = t_start.elapsed_time(t_end) / args.steps
    t_sel = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_att = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    status = S.device_status()
    ms, t_sel, t_att = max_over_ranks([ms, t_sel, t_att], dev, world)
    flops_all = sum_over_ranks(flops, dev, world)
    sel_bytes_all = sum_over_ranks(sel_bytes, dev, world)

    peaks, peak_src = load_peaks()
    # Per GPU: this rank's share of the work over the slowest rank's kernel time.
    attn_tflops = flops_all / world / (t_att * 1e-3) / 1e12
    sel_gbs = sel_bytes_all / world / (t_sel * 1e-3) / 1e9
    # The attention launch is a ~15 ms kernel timed on its own events, so its roofline is the
    # burst cuBLAS figure; the sustained (power-capped, seconds-long) figure is reported beside it.
    peak_t = float(peaks["bf16_tflops"])
    peak_t_sus = float(peaks.get("bf16_tflops_sustained", peak_t))
    peak_hbm = float(peaks["hbm_gbs"])
    read_gbs = read_bandwidth_probe(S, dev)
    read_peak = max(peak_hbm, read_gbs)
    traffic = recorded_traffic("attn_sparse_kernel<128>", sc_full.name if not args.heads else "")
    if traffic is not None:
        traffic *= sc.heads / sc_full.heads   # the record is per launch over all heads
    result = {
        "metric": METRIC,
        "value": whole_job_tflops(flops_all, ms),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(sc_full, args, world),
        "gpu_launches": launches_per_step * args.steps,
        "attn": {"ms": t_att, "tflops": attn_tflops, "frac_of_peak": attn_tflops / peak_t,
                 "frac_of_sustained_peak": attn_tflops / peak_t_sus,
                 "kept_tile_tflop": flops_all / 1e12, "kept_blocks_per_row": kmax},
        "select": {"us": t_sel * 1e3, "gbs": sel_gbs, "frac_of_hbm": sel_gbs / peak_hbm,
                   "read_probe_gbs": read_gbs, "frac_of_read_peak": sel_gbs / read_peak,
                   "frac_of_spec": sel_gbs / HBM_SPEC_GBS, "bytes": sel_bytes_all,
                   "share_of_step": t_sel / (t_sel + t_att),
                   "note": "frac_of_hbm divides by the measured copy rate (read + write); "
                           "frac_of_read_peak by the higher of that and the library's read-only streaming "
                           "probe timed in this run; frac_of_spec by the 7.7 TB/s HGX B200 figure"},
        "us_per_scale": ms * 1e3,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak_t, "traffic": traffic,
                     "kernel": "attn_sparse_kernel<128>",
                     "peak_source": f"{peak_src} bf16 burst (the kernel is timed alone, one ~15 ms launch)",
                     "sustained_peak": peak_t_sus, "frac_of_sustained": attn_tflops / peak_t_sus},
        "device_status": int(status),
    }
    clocks_summary = clocks.summary()
    result["clocks"] = clocks_summary
    if world > 1 and args.gather_o:
        # Optional: one all-gather of O across ranks (a caller whose next layer needs every
        # head); not part of the step, which has no collective.
        shard.gather_heads(o, rank, world, sc_full.heads)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        g0.record(stream)
        full_o = shard.gather_heads(o, rank, world, sc_full.heads)
        g1.record(stream)
        torch.cuda.synchronize()
        gms, = max_over_ranks([g0.elapsed_time(g1)], dev, world)
        result["allgather_o"] = {"ms": gms, "bytes_per_rank_out": int(o.numel() * 2),
                                 "gbs_per_rank": full_o.numel() * 2 * (world - 1) / world / (gms * 1e-3) / 1e9}
        del full_o

    # The 64-token block variant on the same input (the pages' block-size ablation): same path,
    # block = 64 for the partition, the scores, the Top-K and the attention tiles.
    if not args.no_block64 and not args.heads:
        plan64 = S.make_plan(sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density, args.budget_mode, block=64)
        ws64 = S.Workspace(sc.heads, sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.head_dim, dev, block=64)
        idx64 = torch.empty(sc.heads, int(plan64.nqb), int(plan64.k_total), dtype=torch.int32, device=dev)
        cnt64 = torch.empty(sc.heads, int(plan64.nqb), dtype=torch.int32, device=dev)
        o64 = torch.empty_like(q)

        def step64(ev):
            ev[0].record(stream)
            S.select(q, k, *seg, sc.clip, sc.density, args.budget_mode, workspace=ws64, idx=idx64, cnt=cnt64, block=64)
            ev[1].record(stream)
            S.attn(q, k, v, idx64, cnt64, o=o64, want_lse=False, block=64)
            ev[2].record(stream)

        n64 = max(3, min(args.steps, 5))
        ev64 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n64 + 2)]
        for e in ev64:
            step64(e)
        torch.cuda.synchronize()
        t_sel64 = float(np.median([e[0].elapsed_time(e[1]) for e in ev64[2:]]))
        t_att64 = float(np.median([e[1].elapsed_time(e[2]) for e in ev64[2:]]))
        flops64 = kept_tile_flops(idx64, cnt64, sc.n_q, sc.n_kv, sc.head_dim, block=64)
        sel_bytes64 = 2.0 * sc.heads * sc.head_dim * (sc.n_q + sc.n_kv) + 4.0 * sc.heads * plan64.nqb * (plan64.k_total + 1)
        result["block64"] = {
            "nqb": int(plan64.nqb), "nkb": int(plan64.nkb), "k_total": int(plan64.k_total),
            "k_topk": int(plan64.k_topk), "n_cand": int(plan64.n_cand),
            "attn_ms": t_att64, "attn_tflops": flops64 / (t_att64 * 1e-3) / 1e12,
            "kept_tile_tflop": flops64 / 1e12, "select_us": t_sel64 * 1e3,
            "select_gbs": sel_bytes64 / (t_sel64 * 1e-3) / 1e9, "step_ms": t_sel64 + t_att64,
            "note": "64-row query blocks run as half of a 128-row MMA tile (pairs of kept 64-token KV "
                    "blocks form one 128-token tile), so per kept FLOP the tensor cores do about 2x the "
                    "work of block 128"}
        del ws64, idx64, cnt64, o64
        torch.cuda.empty_cache()

    # dense run of the same shape: the same kernel with every block kept
    if not args.no_dense:
        dplan = S.make_plan(sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, 1.0)
        didx = torch.arange(int(dplan.nkb), dtype=torch.int32, device=dev).expand(
            sc.heads, int(dplan.nqb), int(dplan.nkb)).contiguous()
        dcnt = torch.full((sc.heads, int(dplan.nqb)), int(dplan.nkb), dtype=torch.int32, device=dev)
        dlse = torch.empty_like(lse)   # lse keeps the sparse step's LSE for the mass analysis
        S.attn(q, k, v, didx, dcnt, o=o, lse=dlse)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        S.attn(q, k, v, didx, dcnt, o=o, lse=dlse)
        e1.record(stream)
        torch.cuda.synchronize()
        dms = e0.elapsed_time(e1)
        dflops = kept_tile_flops(didx, dcnt, sc.n_q, sc.n_kv, sc.head_dim)
        result["dense"] = {"ms": dms, "tflops": dflops / (dms * 1e-3) / 1e12,
                           "speedup_of_sparse_step": dms / ms}
        del didx, dcnt
        # Retained dense softmax mass of the selected mask and the token-wise upper bound
        # with the same per-row token budget (the pages' Figure 3 quantities).
        S.token_bound(q, k, idx, cnt, dlse, want_tokens=False)   # warm-up
        m0, m1, m2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        m0.record(stream)
        _, e_block = S.retained_mass(lse, dlse, want_tokens=False)
        m1.record(stream)
        _, u_block = S.token_bound(q, k, idx, cnt, dlse, want_tokens=False)
        m2.record(stream)
        torch.cuda.synchronize()
        bms = m1.elapsed_time(m2)
        qk_flops = 4 * 2.0 * sc.head_dim * sc.n_q * sc.n_kv * sc.heads   # four dense Q K^T passes
        result["mass"] = {
            "retained_mean": float(e_block.mean()), "retained_min": float(e_block.min()),
            "bound_mean": float(u_block.mean()), "gap_mean": float((u_block - e_block).mean()),
            "retained_ms": m0.elapsed_time(m1), "bound_ms": bms,
            "bound_qk_tflops": qk_flops / (bms * 1e-3) / 1e12,
            "note": "per query block means over valid rows; synthetic inputs, so the pages' values "
                    "(model activations) are context only"}
        del dlse, e_block, u_block

    # Fresh against reused selection over the reference context (the digest's cross-clip
    # comparison, Figure 4): the preceding clip's queries (seeded, independent of the current
    # clip's: the synthetic inputs carry no correlation between clips) pick the reused pattern.
    if not args.no_reuse and not args.heads and sc.clip >= 2 and sc.n_text % 128 == 0 and sc.n_ctx % 128 == 0:
        from block_sparse_attention_tok_b200 import reuse
        q_prev = synth.make_prev_clip_queries(sc.n_q, sc.heads, sc.head_dim,
                                              [500000 + h0 + h + (1000 * rank if args.scaling == "weak" else 0)
                                               for h in range(sc.heads)], device=dev)
        reuse.reference_reuse(q, q_prev, k, v, *seg, 0.15, workspace=ws)   # warm-up
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        res = reuse.reference_reuse(q, q_prev, k, v, *seg, 0.15, workspace=ws)
        r1.record(stream)
        torch.cuda.synchronize()
        result["reuse"] = {
            "reference_budget": 0.15, "k_ref": res["k_ref"], "n_ref_blocks": sc.n_ctx // 128,
            "fresh_mean": float(res["e_fresh"].mean()), "reused_mean": float(res["e_reused"].mean()),
            "ms": r0.elapsed_time(r1),
            "note": "retained share of the softmax mass over the reference context; the preceding clip's "
                    "queries are synthetic and independent of the current ones, so the reused pattern acts "
                    "as an uninformed one here (the pages' 85% vs 56% come from model activations)"}
        del q_prev, res
        torch.cuda.empty_cache()

    # End to end through the public API with host buffers: every step copies its q/k/v from
    # pinned host memory, runs the forward and reads o back. Heads are independent, so the
    # step is issued in head chunks on three streams: the H2D copy of chunk c+1 (and of the
    # next step) overlaps the forward of chunk c and the D2H copy of chunk c-1. The serial
    # form (copy all, forward, read back) is reported next to it.
    if not args.no_e2e:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        n_e2e = max(2, min(args.steps, 5))

        def e2e_serial_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            S.forward(q, k, v, *seg, sc.clip, sc.density, args.budget_mode, workspace=ws, idx=idx, cnt=cnt,
                      o=o, lse=lse)
            ho.copy_(o, non_blocking=True)

        e2e_serial_step()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_serial_step()
        b.record(stream)
        torch.cuda.synchronize()
        serial_ms = a.elapsed_time(b) / n_e2e

        n_chunks = min(4, sc.heads)
        bounds = [(sc.heads * c // n_chunks, sc.heads * (c + 1) // n_chunks) for c in range(n_chunks)]
        ws_c = S.Workspace(max(h1 - h0 for h0, h1 in bounds), sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.head_dim, dev)
        s_h2d, s_cmp, s_d2h = (torch.cuda.Stream(device=dev) for _ in range(3))
        done_cmp = [None] * n_chunks   # forward of chunk c finished (its inputs may be overwritten)
        done_d2h = [None] * n_chunks   # o of chunk c read back (it may be overwritten)

        def e2e_pipelined_step():
            for c, (h0, h1) in enumerate(bounds):
                with torch.cuda.stream(s_h2d):
                    if done_cmp[c] is not None:
                        s_h2d.wait_event(done_cmp[c])
                    q[h0:h1].copy_(hq[h0:h1], non_blocking=True)
                    k[h0:h1].copy_(hk[h0:h1], non_blocking=True)
                    v[h0:h1].copy_(hv[h0:h1], non_blocking=True)
                    ev_in = torch.cuda.Event()
                    ev_in.record(s_h2d)
                s_cmp.wait_event(ev_in)
                if done_d2h[c] is not None:
                    s_cmp.wait_event(done_d2h[c])
                S.forward(q[h0:h1], k[h0:h1], v[h0:h1], *seg, sc.clip, sc.density, args.budget_mode, workspace=ws_c,
                          idx=idx[h0:h1], cnt=cnt[h0:h1], o=o[h0:h1], lse=lse[h0:h1], stream=s_cmp)
                ev_c = torch.cuda.Event()
                ev_c.record(s_cmp)
                done_cmp[c] = ev_c
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(ev_c)
                    ho[h0:h1].copy_(o[h0:h1], non_blocking=True)
                    ev_o = torch.cuda.Event()
                    ev_o.record(s_d2h)
                done_d2h[c] = ev_o

        e2e_pipelined_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_h2d)
        for _ in range(n_e2e):
            e2e_pipelined_step()
        for st in (s_h2d, s_cmp, s_d2h):
            stream.wait_stream(st)
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems, serial_ms = max_over_ranks([a.elapsed_time(b) / n_e2e, serial_ms], dev, world)
        result["e2e"] = {"value": whole_job_tflops(flops_all, ems), "unit": "TFLOP/s",
                         "h2d_bytes_per_step": int(hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2),
                         "d2h_bytes_per_step": int(ho.numel() * 2), "ms_per_step": ems, "steps": n_e2e,
                         "pipelined": f"{n_chunks} head chunks per step on three streams (H2D / forward / D2H)",
                         "serial_value": whole_job_tflops(flops_all, serial_ms), "serial_ms_per_step": serial_ms}
        del hq, hk, hv, ho, ws_c

    if world == 1 and not args.no_schedule and not args.heads:
        del o, lse
        torch.cuda.empty_cache()
        result["schedule"] = run_schedule(S, dev, stream)
        result["cross_scale"] = run_cross_scale(S, dev, stream)

    if rank == 0 and not args.no_cpu_baseline:
        n_h = min(4, q.shape[0])
        qc, kc, vc = (x[:n_h].cpu() for x in (q, k, v))
        fl, t, t_pro = oracle_sample(qc, kc, vc, sc, list(range(n_h)), 160, args.budget_mode)
        result["cpu_baseline"] = {
            "value": fl / t_pro / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"heads 0-{n_h - 1} of the same input: bf16 widening + full selection (prorated to the "
                      "sampled rows) + attention of 160 evenly spaced query blocks per head, fp64 numpy; "
                      f"{t:.1f} s of CPU time"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spawned_rank(local_rank: int, world: int, port: int, argv):
    """Entry of a rank started by launch_ranks: the torchrun environment, then main()."""
    os.environ.update(RANK=str(local_rank), LOCAL_RANK=str(local_rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.argv = [sys.argv[0]] + list(argv)
    rc = main()
    if rc:
        raise SystemExit(rc)


def launch_ranks(n: int) -> int:
    """`--gpus N` without a torchrun environment: start N ranks (one process per GPU, spawned)."""
    import torch.multiprocessing as mp
    mp.start_processes(_spawned_rank, args=(n, _free_port(), sys.argv[1:]), nprocs=n, join=True,
                       start_method="spawn")
    return 0


def main():
    args = parse()
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return launch_ranks(args.gpus)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
