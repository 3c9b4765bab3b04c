"""Fresh against reused selection over the reference context (the cross-clip comparison of
the digest's Figure 4) on the GPU, against the oracle's reference_reuse_report.

The kept reference blocks follow the mask rule on the reference columns of the scores (no
forced prefix); the retained reference mass of each query block is compared with the
oracle's reference_mass computed on the GPU's own kept blocks.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_tok_b200 import synth
from oracle import sparstar_oracle as O
from tests.parity import bits, check_masks, LSE_ABS

pytestmark = pytest.mark.gpu

MASS_ABS = 3e-3   # two LSEs within 1e-3 each: exp(d lse) within about 2e-3 relative of R <= 1


@pytest.fixture(scope="module")
def S(cuda_lib):
    from block_sparse_attention_tok_b200 import sparstar
    return sparstar


@pytest.mark.parametrize("d,n_text,n_ctx,n_cur,n_q,frac", [
    (128, 128, 1024, 512, 384, 0.25),
    (64, 256, 128 * 20, 640, 700, 0.15),   # ragged query tail
])
def test_reference_reuse_matches_oracle(S, d, n_text, n_ctx, n_cur, n_q, frac):
    from block_sparse_attention_tok_b200 import reuse
    H = 2
    q, k, v = synth.make_qkv(n_q, n_text + n_ctx + n_cur, H, d, [900 + h for h in range(H)], device="cuda")
    q_prev = synth.make_prev_clip_queries(n_q, H, d, [950 + h for h in range(H)], device="cuda")
    res = reuse.reference_reuse(q, q_prev, k, v, n_text, n_ctx, n_cur, frac)
    assert S.device_status() == S.OK
    nb_text, n_ref = n_text // 128, n_ctx // 128
    nqb = O.num_blocks(n_q)
    qb, qpb, kb = bits(q), bits(q_prev), bits(k)
    for key, qsrc in (("fresh", qb), ("reused", qpb)):
        g = res[key].cpu().numpy()
        ref_rows, ref_S = [], []
        for h in range(H):
            qf, kf = O.bf16_bits_to_f64(qsrc[h]), O.bf16_bits_to_f64(kb[h])
            Sfull = O.block_scores(O.pool_blocks(qf), O.pool_blocks(kf))
            Sref = Sfull[:, nb_text:nb_text + n_ref]
            ref_S.append(Sref)
            ref_rows.append(O.select_rows(Sref, 0, res["k_ref"]))
        check_masks(g - nb_text, np.full((H, nqb), res["k_ref"]), np.stack(ref_rows), np.stack(ref_S), 0, res["k_ref"])
        e = res["e_" + key].cpu().numpy()
        for h in range(H):
            qf, kf = O.bf16_bits_to_f64(qb[h]), O.bf16_bits_to_f64(kb[h])
            want = O.reference_mass(qf, kf, g[h], n_text, n_ctx, range(nqb))
            assert np.abs(e[h] - want).max() <= MASS_ABS, f"{key} head {h}: {np.abs(e[h] - want).max():.2e}"


def test_reference_reuse_identical_queries_and_full_budget(S):
    from block_sparse_attention_tok_b200 import reuse
    q, k, v = synth.make_qkv(256, 128 + 768 + 256, 1, 128, [971], device="cuda")
    res = reuse.reference_reuse(q, q.clone(), k, v, 128, 768, 256, 0.5)
    assert torch.equal(res["fresh"], res["reused"]) and torch.equal(res["e_fresh"], res["e_reused"])
    full = reuse.reference_reuse(q, q.clone(), k, v, 128, 768, 256, 1.0)
    assert torch.allclose(full["e_fresh"], torch.ones_like(full["e_fresh"]), atol=1e-5)


# ------------------------------------------------------------------ reuse across scales (Figure 5)

@pytest.mark.parametrize("seg_prev,grid_prev,seg_now,grid_now,H", [
    ((256, 512, 384), (2, 8, 24), (256, 512, 768), (2, 12, 32), 2),        # Clip 1 shape, 3 -> 6 blocks
    ((128, 1024, 117), (1, 9, 13), (128, 1024, 231), (3, 7, 11), 3),       # reference prefix, ragged blocks
    ((512, 8192, 36864), (8, 64, 72), (512, 8192, 72192), (8, 94, 96), 4),  # the schedule's last two scales
    ((512, 8192, 72192), (8, 94, 96), (512, 8192, 8192), (8, 32, 32), 1),   # shrinking
])
def test_map_scores_is_the_oracle_gather(S, seg_prev, grid_prev, seg_now, grid_now, H):
    n_prefix = (seg_prev[0] + seg_prev[1]) // 128
    nqb_prev = O.num_blocks(seg_prev[2])
    g = torch.Generator(device="cuda").manual_seed(seg_now[2])
    s_prev = torch.randn(H, nqb_prev, n_prefix + nqb_prev, device="cuda", generator=g)
    got = S.map_scores(s_prev, seg_prev, grid_prev, seg_now, grid_now)
    assert S.device_status() == S.OK
    sp = s_prev.cpu().numpy().astype(np.float64)
    for h in range(H):
        want = O.map_scores(sp[h], n_prefix, grid_prev, grid_now).astype(np.float32)
        assert np.array_equal(got[h].cpu().numpy(), want)


def _schedule_case():
    """Three Clip-1 scales of one head pair with growing grids (ragged last blocks)."""
    seg_t, seg_c = 128, 256
    grids = [(2, 8, 15), (2, 12, 23), (2, 16, 31)]
    dens = [0.5, 0.4, 0.3]
    scales = []
    for i, (grid, dn) in enumerate(zip(grids, dens)):
        n = grid[0] * grid[1] * grid[2]
        q, k, v = synth.make_qkv(n, seg_t + seg_c + n, 2, 64, [3000 + 10 * i + h for h in range(2)], device="cuda")
        scales.append(dict(q=q, k=k, v=v, seg=(seg_t, seg_c, n), grid=grid, clip=1, density=dn))
    return scales


@pytest.mark.parametrize("policy", ["per_scale", "every_2", "one_shot"])
def test_cross_scale_policies_match_oracle(S, policy):
    """Recomputed scales: the oracle's selection by the mask rule. Reused scales: bit-identical to
    the oracle's reused_rows on the GPU's own scores of the scale they reuse (the same fp32
    values ranked by the same rule). Retained mass of every scale's mask against the oracle."""
    from block_sparse_attention_tok_b200 import reuse
    scales = _schedule_case()
    mode = S.BUDGET_CANDIDATES
    masks = reuse.cross_scale_masks(scales, policy, mode)
    assert S.device_status() == S.OK
    recompute = reuse.POLICIES[policy]
    src = None
    for si, (sc, (idx, cnt)) in enumerate(zip(scales, masks)):
        seg = sc["seg"]
        plan = S.make_plan(seg[2], *seg, 1, sc["density"], mode)
        qb, kb = bits(sc["q"]), bits(sc["k"])
        g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        if recompute(si) or src is None:
            ref = [O.select_head(O.bf16_bits_to_f64(qb[h]), O.bf16_bits_to_f64(kb[h]), seg[0], seg[1], 1,
                                 sc["density"], mode) for h in range(2)]
            check_masks(g_idx, g_cnt, np.stack([r[0] for r in ref]), np.stack([r[1] for r in ref]),
                        int(plan.n_forced), int(plan.k_topk))
            _, _, s_gpu = S.select(sc["q"], sc["k"], *seg, 1, sc["density"], mode, want_scores=True)
            src = (s_gpu.cpu().numpy().astype(np.float64), sc["grid"])
        else:
            n_prefix = (seg[0] + seg[1]) // 128
            for h in range(2):
                want = O.reused_rows(src[0][h], n_prefix, src[1], sc["grid"], int(plan.n_forced), int(plan.k_topk))
                assert np.array_equal(g_idx[h], want), f"scale {si} head {h}"
            assert (g_cnt == int(plan.k_total)).all()
        e = reuse.retained_mass_of(sc["q"], sc["k"], sc["v"], idx, cnt).cpu().numpy()
        for h in range(2):
            qf, kf = O.bf16_bits_to_f64(qb[h]), O.bf16_bits_to_f64(kb[h])
            E, _, _, _ = O.mass_report(qf, kf, g_idx[h], range(g_idx.shape[1]))
            assert np.abs(e[h] - E).max() <= 2.5 * LSE_ABS * E.max(), f"scale {si} head {h}"
