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
from tests.parity import bits, check_masks

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
