"""The 64-token block variant (the pages' block-size ablation) on the GPU, against the oracle
run with block = 64: masks by the same gap rule, outputs element by element.

With 64-token blocks a query block is 64 rows of the kernel's 128-row MMA tile (the other
64 rows are computed and dropped), a KV tile is two consecutive kept 64-token blocks (an odd
last one alone, its second half masked), and rows with more than 3,965 candidates go
through the radix Top-K.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_tok_b200 import synth
from oracle import sparstar_oracle as O
from tests.parity import bits, check_output, run_and_check, LSE_ABS

pytestmark = pytest.mark.gpu
B = 64


@pytest.fixture(scope="module")
def S(cuda_lib):
    from block_sparse_attention_tok_b200 import sparstar
    return sparstar


def _f64(x):
    return O.bf16_bits_to_f64(x)


def _run(S, q, k, v, n_text, n_ctx, n_cur, clip, density, mode=0, qblocks=None, out_heads=None, label=None):
    """Masks of every head by the gap rule, scores within the split-precision bound, outputs of
    `out_heads` on `qblocks` plus every block whose mask differs (oracle on the GPU's kept list)."""
    stats = run_and_check(S, O, q, k, v, n_text, n_ctx, n_cur, clip, density, mode, block=B, qblocks=qblocks,
                          out_heads=out_heads, label=label)
    return stats, S.make_plan(q.shape[1], n_text, n_ctx, n_cur, clip, density, mode, block=B)


@pytest.mark.parametrize("d,n_q,n_text,n_ctx,n_cur,clip,density", [
    (64, 300, 128, 256, 300, 2, 0.3),        # ragged query and KV tails (300 = 4*64 + 44)
    (128, 1000, 256, 1000, 1000, 2, 0.2),
    (128, 130, 64, 200, 130, 1, 0.5),        # Clip 1: text + context forced; a 2-row last block
])
def test_block64_small_cases(S, d, n_q, n_text, n_ctx, n_cur, clip, density):
    q, k, v = synth.make_qkv(n_q, n_text + n_ctx + n_cur, 2, d, [700 + n_q, 701 + n_q], device="cuda")
    stats, plan = _run(S, q, k, v, n_text, n_ctx, n_cur, clip, density)
    assert stats["rows"] == 2 * int(plan.nqb)


def test_block64_radix_topk_rows(S):
    """More than 3,965 candidates per row: the CTA-per-row radix Top-K path."""
    n_cur = 64 * 4000
    q, k, v = synth.make_qkv(200, 64 + n_cur, 1, 128, [811], device="cuda")
    stats, plan = _run(S, q, k, v, 64, 0, n_cur, 2, 0.05, qblocks=lambda n: [0, n - 1])
    assert int(plan.n_cand) > 3965 and stats["rows"] == int(plan.nqb)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n_q,n_kv", [(1, 1), (63, 65), (200, 1000)])
def test_block64_attention_on_random_masks(S, d, n_q, n_kv):
    q, k, v = synth.make_qkv(n_q, n_kv, 2, d, [17, 18], device="cuda")
    nqb, nkb = O.num_blocks(n_q, B), O.num_blocks(n_kv, B)
    rng = np.random.default_rng(n_q * 7 + n_kv)
    kk = max(1, min(nkb, int(rng.integers(1, nkb + 1))))
    rows = np.stack([np.stack([np.sort(rng.choice(nkb, kk, replace=False)) for _ in range(nqb)]) for _ in range(2)])
    idx = torch.from_numpy(rows.astype(np.int32)).cuda().contiguous()
    cnt = torch.full((2, nqb), kk, dtype=torch.int32, device="cuda")
    o, lse = S.attn(q, k, v, idx, cnt, block=B)
    assert S.device_status() == S.OK
    qb, kb, vb = bits(q), bits(k), bits(v)
    o_np, lse_np = o.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(2):
        outs = O.block_sparse_attention(_f64(qb[h]), _f64(kb[h]), _f64(vb[h]), rows[h], range(nqb), block=B)
        for i, (o_ref, lse_ref) in enumerate(outs):
            s, e = O.block_token_range(i, n_q, B)
            check_output(o_np[h, s:e], o_ref, f"h{h} qb{i}")
            assert np.abs(lse_np[h, s:e] - lse_ref).max() <= LSE_ABS


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kk", [1, 2, 3, 4, 7, 10])
def test_block64_pairs_odd_even_and_ragged(S, d, kk):
    """Kept lists of odd and even length, each ending with the ragged last KV block (17 valid
    tokens): it is then the second half of a pair (even length) or the lone last entry (odd),
    and the lists mix adjacent and distant blocks, so pairs are not contiguous in memory. The
    index rows are wider than cnt, so an odd list's missing partner is never read."""
    n_q, n_kv = 130, 64 * 9 + 17
    q, k, v = synth.make_qkv(n_q, n_kv, 2, d, [31 + kk + d, 41 + kk + d], device="cuda")
    nqb, nkb = O.num_blocks(n_q, B), O.num_blocks(n_kv, B)
    rng = np.random.default_rng(900 + kk)
    rows = np.stack([np.stack([np.sort(np.append(rng.choice(nkb - 1, kk - 1, replace=False), nkb - 1))
                               for _ in range(nqb)]) for _ in range(2)])
    # entries past cnt hold an out-of-range block: reading one would raise the bounds flag
    padded = np.full((2, nqb, kk + 3), -7, dtype=np.int32)
    padded[:, :, :kk] = rows
    idx = torch.from_numpy(padded).cuda().contiguous()
    cnt = torch.full((2, nqb), kk, dtype=torch.int32, device="cuda")
    o, lse = S.attn(q, k, v, idx, cnt, block=B)
    assert S.device_status() == S.OK
    qb, kb, vb = bits(q), bits(k), bits(v)
    o_np, lse_np = o.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(2):
        outs = O.block_sparse_attention(_f64(qb[h]), _f64(kb[h]), _f64(vb[h]), rows[h], range(nqb), block=B)
        for i, (o_ref, lse_ref) in enumerate(outs):
            s, e = O.block_token_range(i, n_q, B)
            check_output(o_np[h, s:e], o_ref, f"h{h} qb{i}")
            assert np.abs(lse_np[h, s:e] - lse_ref).max() <= LSE_ABS


@pytest.mark.slow
def test_block64_final_scale_sampled(S):
    """The 720p Clip-2 final scale with 64-token blocks: every mask row of all 32 heads, outputs
    of three heads on sampled query blocks plus every block whose mask differs."""
    sc = synth.FINAL_CLIP2
    q, k, v = synth.make_scale_inputs(sc, device="cuda")
    rng = np.random.default_rng(64)
    stats, plan = _run(S, q, k, v, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density,
                       qblocks=lambda n: sorted({0, n - 1, *rng.choice(n, 3, replace=False).tolist()}),
                       out_heads=[0, 15, 31], label=f"{sc.name} block 64")
    assert stats["rows"] == sc.heads * int(plan.nqb)
    del q, k, v
    torch.cuda.empty_cache()
