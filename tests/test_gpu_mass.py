"""Retained attention mass and its token-wise upper bound on the GPU, against the oracle.

The pages' analysis quantities (digest section 关键结果与论文证据, bullet 跨尺度复用损失,
Figure 3): R_t, the dense softmax mass a block mask keeps for query token t, and U_t, the
most mass any choice of the same number of key tokens could keep. Inputs are seeded; the
oracle reads the exact bf16 bytes and the GPU's own mask rows.

Tolerances: R = exp(lse_kept - lse_dense) inherits both LSE errors (each <= LSE_ABS against
fp64), so |R - R_ref| <= 2.5 * LSE_ABS * R; U normalises the dense probabilities by the GPU's
lse_dense (same relative error) and locates the B-th value to 2^-14 in log2 (relative error
< 5e-5), so |U - U_ref| <= 2.5 * LSE_ABS * U + 1e-4.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_tok_b200 import synth
from oracle import sparstar_oracle as O
from tests.parity import bits, LSE_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S(cuda_lib):
    from block_sparse_attention_tok_b200 import sparstar
    return sparstar


def _dense_lse(S, q, k, v):
    H, n_q, _ = q.shape
    nqb, nkb = O.num_blocks(n_q), O.num_blocks(k.shape[1])
    idx = torch.arange(nkb, dtype=torch.int32, device=q.device).expand(H, nqb, nkb).contiguous()
    cnt = torch.full((H, nqb), nkb, dtype=torch.int32, device=q.device)
    _, lse = S.attn(q, k, v, idx, cnt)
    return lse


def _check_case(S, q, k, v, idx, cnt, lse_kept):
    H, n_q, d = q.shape
    lse_dense = _dense_lse(S, q, k, v)
    r, e = S.retained_mass(lse_kept, lse_dense)
    u, ub = S.token_bound(q, k, idx, cnt, lse_dense)
    assert S.device_status() == S.OK
    qb_, kb_ = bits(q), bits(k)
    nqb = O.num_blocks(n_q)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    r_np, e_np, u_np, ub_np = (x.cpu().numpy() for x in (r, e, u, ub))
    for h in range(H):
        qf, kf = O.bf16_bits_to_f64(qb_[h]), O.bf16_bits_to_f64(kb_[h])
        rows = [gidx[h, i, :gcnt[h, i]] for i in range(nqb)]
        E, U, R_rows, U_rows = O.mass_report(qf, kf, rows, range(nqb))
        tol_r = 2.5 * LSE_ABS * R_rows
        tol_u = 2.5 * LSE_ABS * U_rows + 1e-4
        assert (np.abs(r_np[h] - R_rows) <= tol_r).all(), np.abs(r_np[h] - R_rows).max()
        assert (np.abs(u_np[h] - U_rows) <= tol_u).all(), np.abs(u_np[h] - U_rows).max()
        assert np.abs(e_np[h] - E).max() <= 2.5 * LSE_ABS * E.max()
        assert np.abs(ub_np[h] - U).max() <= 2.5 * LSE_ABS * U.max() + 1e-4
        assert (u_np[h] >= r_np[h] - 2.5 * LSE_ABS).all()   # the bound dominates the mask
    return e_np, ub_np


@pytest.mark.parametrize("d,n_q,n_text,n_ctx,n_cur,density", [
    (64, 300, 128, 256, 300, 0.4),          # ragged query and KV tails
    (128, 640, 256, 1024, 640, 0.25),
    (128, 129, 128, 0, 1000, 0.125),        # one query row in the last block, Clip 1 reading of ctx = 0
])
def test_mass_and_bound_match_oracle(S, d, n_q, n_text, n_ctx, n_cur, density):
    q, k, v = synth.make_qkv(n_q, n_text + n_ctx + n_cur, 2, d, [900 + n_q, 901 + n_q], device="cuda")
    o, lse, idx, cnt = S.forward(q, k, v, n_text, n_ctx, n_cur, 2, density)
    _check_case(S, q, k, v, idx, cnt, lse)


def test_full_budget_bound_is_one(S):
    """Every block kept: the mask retains all mass and no B-subset can hold more."""
    q, k, v = synth.make_qkv(257, 1000, 2, 128, [31, 32], device="cuda")
    nqb, nkb = O.num_blocks(257), O.num_blocks(1000)
    idx = torch.arange(nkb, dtype=torch.int32, device="cuda").expand(2, nqb, nkb).contiguous()
    cnt = torch.full((2, nqb), nkb, dtype=torch.int32, device="cuda")
    _, lse = S.attn(q, k, v, idx, cnt)
    e, ub = _check_case(S, q, k, v, idx, cnt, lse)
    assert np.abs(e - 1).max() <= 1e-5 and np.abs(ub - 1).max() <= 1e-3


def test_single_kept_block_on_oracle_rows(S):
    """Hand-made masks of one block per row (budget 128 or the ragged tail's count)."""
    q, k, v = synth.make_qkv(384, 700, 2, 64, [41, 42], device="cuda")
    nqb, nkb = 3, O.num_blocks(700)
    rng = np.random.default_rng(5)
    rows = rng.integers(0, nkb, size=(2, nqb, 1)).astype(np.int32)
    rows[0, 0, 0] = nkb - 1  # the ragged last block: 60 valid tokens
    idx = torch.from_numpy(rows).cuda().contiguous()
    cnt = torch.ones((2, nqb), dtype=torch.int32, device="cuda")
    _, lse = S.attn(q, k, v, idx, cnt)
    _check_case(S, q, k, v, idx, cnt, lse)
