"""Comparison rules between the CUDA path and the CPU oracle, and the shared GPU-vs-oracle
harness of the parity tests.

Masks: a row whose gap between the K_topk-th and (K_topk+1)-th candidate score (fp64,
oracle) exceeds 1e-3 must be bit-identical. Otherwise the row passes when it has K_total
distinct ascending entries, holds the forced prefix, every chosen candidate scores at least
s_K - 1e-3 and every unchosen candidate at most s_K + 1e-3 (the K-th/(K+1)-th gap rule
that fixes how the fp32 kernel and the fp64 oracle may differ on near-ties).
Outputs: max |o - o_ref| <= 2e-2 and mean |o - o_ref| <= 2e-3 (bf16 inputs, fp32
accumulation), plus an internal relative-L2 guard of 1e-2 that catches wrong tiles and an
LSE guard of 1e-3. The oracle's attention runs on the GPU's own kept list of the row (which
the mask rule has validated), so a query block whose mask legitimately differs from the
oracle's on a near-tie is still compared, not skipped.
Scores: the kernel's block scores (tensor cores, block means split into bf16 hi + lo,
hi.hi + hi.lo + lo.hi in fp32) against the fp64 definition within SCORE_REL * sum_c |qbar_c
kbar_c| / sqrt(d). Derivation: hi = bf16(m) and lo = bf16(m - hi) leave e = m - hi - lo with
|e| <= 2^-16 |m|, |lo| <= 2^-8 |m|; the three dropped terms hi_q e_k, e_q k, lo_q lo_k (plus
lo_q e_k) are each at most about 2^-16 |q_c k_c|, and fp32 accumulation of 3 d products adds
well under 2^-17 of the same sum: below 2^-14 in all.
"""
import math

import numpy as np
import torch

GAP = 1e-3
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
REL_L2 = 1e-2
LSE_ABS = 1e-3
SCORE_REL = 2.0 ** -14

# One line per checked configuration (mask rows compared, rows identical, near-tie rows,
# query blocks whose output was compared); printed at the end of the session.
LOG = []


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_masks(gpu_idx, gpu_cnt, ref_idx, ref_scores, n_forced, k_topk):
    """Apply the mask rule to every row. Returns a stats dict; raises AssertionError on failure."""
    H, nqb, k_total = ref_idx.shape
    gpu_idx = np.asarray(gpu_idx)[:, :, :k_total]
    assert (np.asarray(gpu_cnt) == k_total).all(), "cnt differs from K_total"
    same = (gpu_idx == ref_idx).all(axis=2)
    nkb = ref_scores.shape[2]
    n_cand = nkb - n_forced
    stats = {"rows": H * nqb, "identical": int(same.sum()), "wide_gap_rows": 0, "near_tie_rows": 0}
    if k_topk == 0 or k_topk == n_cand:
        assert same.all(), "rows that do not depend on scores must be identical"
        stats["wide_gap_rows"] = H * nqb
        return stats
    cand = ref_scores[:, :, n_forced:]
    part = -np.partition(-cand, (k_topk - 1, k_topk), axis=2)
    s_k, s_k1 = part[:, :, k_topk - 1], part[:, :, k_topk]
    gap = s_k - s_k1
    wide = gap > GAP
    stats["wide_gap_rows"] = int(wide.sum())
    stats["near_tie_rows"] = int((~wide).sum())
    bad = wide & ~same
    assert not bad.any(), f"{int(bad.sum())} wide-gap rows differ, first at {np.argwhere(bad)[0]}"
    for h, i in np.argwhere(~same):
        row = gpu_idx[h, i]
        assert (np.diff(row) > 0).all(), "row not strictly ascending"
        assert (row[:n_forced] == np.arange(n_forced)).all(), "forced prefix missing"
        chosen = row[n_forced:]
        assert ((chosen >= n_forced) & (chosen < nkb)).all()
        sc = ref_scores[h, i]
        mask = np.zeros(nkb, bool)
        mask[chosen] = True
        mask[:n_forced] = False
        un = ~mask
        un[:n_forced] = False
        assert (sc[mask] >= s_k[h, i] - GAP).all(), "a chosen block scores too low"
        assert (sc[un] <= s_k[h, i] + GAP).all(), "an unchosen block scores too high"
    return stats


def check_output(o_gpu: np.ndarray, o_ref: np.ndarray, what=""):
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    rel = np.linalg.norm(o_gpu.astype(np.float64) - o_ref) / max(np.linalg.norm(o_ref), 1e-30)
    assert err.max() <= MAX_ABS, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs {err.mean():.3e}"
    assert rel <= REL_L2, f"{what}: rel L2 {rel:.3e}"
    return float(err.max()), float(err.mean()), float(rel)


def run_and_check(S, O, q, k, v, n_text, n_ctx, n_cur, clip, density, mode, block=128, qblocks=None,
                  out_heads=None, label=None):
    """The whole path on the GPU (sparstar_forward, and sparstar_select with scores), against
    the oracle:
      - masks of EVERY head and query block by the mask rule;
      - every block score within the split-precision bound;
      - outputs and LSEs of the heads `out_heads` (default: all) on the query blocks
        `qblocks(nqb)` (default: all), plus every query block of those heads whose GPU mask
        differs from the oracle's, each against the oracle run on the GPU's own kept list.
    `O` is the oracle module. Appends a line to LOG and returns the mask stats."""
    H, n_q, d = q.shape
    o, lse, idx, cnt = S.forward(q, k, v, n_text, n_ctx, n_cur, clip, density, mode, block=block)
    _, _, scores = S.select(q, k, n_text, n_ctx, n_cur, clip, density, mode, want_scores=True, block=block)
    assert S.device_status() == S.OK
    plan = S.make_plan(n_q, n_text, n_ctx, n_cur, clip, density, mode, block=block)
    nqb, k_total = int(plan.nqb), int(plan.k_total)
    gidx = idx.cpu().numpy()[:, :, :k_total]
    gcnt = cnt.cpu().numpy()
    got_S = scores.cpu().numpy()
    o_np, lse_np = o.float().cpu().numpy(), lse.cpu().numpy()
    del o, lse, idx, cnt, scores
    qb, kb = bits(q), bits(k)
    out_heads = set(range(H)) if out_heads is None else set(out_heads)
    ref_idx = np.empty((H, nqb, k_total), dtype=np.int64)
    ref_S = np.empty((H, nqb, int(plan.nkb)), dtype=np.float64)
    for h in range(H):
        qf, kf = O.bf16_bits_to_f64(qb[h]), O.bf16_bits_to_f64(kb[h])
        ref_idx[h], ref_S[h] = O.select_head(qf, kf, n_text, n_ctx, clip, density, mode, block)
        qbar, kbar = O.pool_blocks(qf, block), O.pool_blocks(kf, block)
        bound = SCORE_REL * (np.abs(qbar) @ np.abs(kbar).T) / math.sqrt(d) + 1e-7
        assert (np.abs(got_S[h] - ref_S[h]) <= bound).all(), f"h{h}: score error above the split-precision bound"
    stats = check_masks(gidx, gcnt, ref_idx, ref_S, int(plan.n_forced), int(plan.k_topk))
    del ref_S, got_S
    vb = bits(v)
    n_out = 0
    for h in sorted(out_heads):
        differ = np.flatnonzero((gidx[h] != ref_idx[h]).any(axis=1)).tolist()
        chosen = range(nqb) if qblocks is None else qblocks(nqb)
        qbl = sorted(set(chosen) | set(differ))
        qf, kf, vf = (O.bf16_bits_to_f64(x[h]) for x in (qb, kb, vb))
        outs = O.block_sparse_attention(qf, kf, vf, gidx[h], qbl, block=block)
        for i, (o_ref, lse_ref) in zip(qbl, outs):
            s, e = O.block_token_range(i, n_q, block)
            check_output(o_np[h, s:e], o_ref, f"h{h} qb{i}")
            assert np.abs(lse_np[h, s:e] - lse_ref).max() <= LSE_ABS, f"h{h} qb{i}: lse"
        n_out += len(qbl)
    stats["output_blocks"] = n_out
    stats["differing_rows"] = stats["rows"] - stats["identical"]
    if label is not None:
        LOG.append(f"{label}: heads {H}, mask rows {stats['rows']} (identical {stats['identical']}, "
                   f"near-tie {stats['near_tie_rows']}), output blocks {n_out}")
    return stats
