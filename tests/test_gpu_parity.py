"""CUDA path vs CPU oracle, element by element, through the C ABI.

Small cases are compared on every output; the full-size workloads (launched exactly as
bench.py launches them) are compared on every mask row and on sampled query blocks of
the attention output. Inputs are seeded (block_sparse_attention_tok_b200.synth); the
oracle always reads the exact bytes the GPU used.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_tok_b200 import synth
from oracle import sparstar_oracle as O
from tests.parity import bits, check_output, run_and_check, LSE_ABS

pytestmark = pytest.mark.gpu


def _f64(x_bits):
    return O.bf16_bits_to_f64(x_bits)


def _oracle_attention(qb, kb, vb, rows, h, qblocks, d):
    qf, kf, vf = _f64(qb[h]), _f64(kb[h]), _f64(vb[h])
    return O.block_sparse_attention(qf, kf, vf, rows, qblocks)


def _run_case(lib, q, k, v, n_text, n_ctx, n_cur, clip, density, mode, qblocks_per_head=None, out_heads=None,
              label=None):
    """Forward on the GPU; the mask rule on every row of every head; outputs on the query
    blocks (all, or qblocks_per_head(nqb)) of `out_heads` (default all), plus every query
    block whose mask differs from the oracle's, against the oracle on the GPU's kept list."""
    return run_and_check(lib, O, q, k, v, n_text, n_ctx, n_cur, clip, density, mode, qblocks=qblocks_per_head,
                         out_heads=out_heads, label=label)


def _attn_with_oracle_mask(lib, q, k, v, rows_all, qblocks=None):
    """sparstar_attn driven by the oracle's own idx rows (uploaded), compared row by row."""
    S = lib
    H, n_q, d = q.shape
    idx = torch.from_numpy(rows_all.astype(np.int32)).to(q.device).contiguous()
    cnt = torch.full(rows_all.shape[:2], rows_all.shape[2], dtype=torch.int32, device=q.device)
    o, lse = S.attn(q, k, v, idx, cnt)
    assert S.device_status() == S.OK
    qb, kb, vb = bits(q), bits(k), bits(v)
    o_np, lse_np = o.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(H):
        qbl = list(range(rows_all.shape[1])) if qblocks is None else qblocks
        for i, (o_ref, lse_ref) in zip(qbl, _oracle_attention(qb, kb, vb, rows_all[h], h, qbl, d)):
            s, e = O.block_token_range(i, n_q)
            check_output(o_np[h, s:e], o_ref, f"h{h} qb{i}")
            assert np.abs(lse_np[h, s:e] - lse_ref).max() <= LSE_ABS


@pytest.fixture(scope="module")
def S(cuda_lib):
    from block_sparse_attention_tok_b200 import sparstar
    return sparstar


def test_tiny_clip2_scale_all_rows(S):
    sc = synth.TINY_CLIP2
    q, k, v = synth.make_scale_inputs(sc, device="cuda")
    stats = _run_case(S, q, k, v, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density, 0, label=sc.name)
    assert stats["identical"] == stats["rows"]


@pytest.mark.parametrize("case", list(synth.random_small_cases(seed=4321, count=48)), ids=lambda c: c["name"])
def test_small_ragged_cases(S, case):
    c = case
    q, k, v = synth.make_qkv(c["n_q"], c["n_text"] + c["n_ctx"] + c["n_cur"], c["H"], c["d"],
                             [c["seed"] + 100 * h for h in range(c["H"])], device="cuda")
    _run_case(S, q, k, v, c["n_text"], c["n_ctx"], c["n_cur"], c["clip"], c["density"], c["mode"])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n_q,n_kv", [(1, 1), (127, 129), (384, 1000), (700, 3000)])
def test_attention_on_random_masks(S, d, n_q, n_kv):
    """Arbitrary ascending kept lists (not only Top-K ones), including a single kept block."""
    q, k, v = synth.make_qkv(n_q, n_kv, 2, d, [7, 8], device="cuda")
    nqb, nkb = O.num_blocks(n_q), O.num_blocks(n_kv)
    rng = np.random.default_rng(n_q * 31 + n_kv)
    kk = max(1, min(nkb, int(rng.integers(1, nkb + 1))))
    rows = np.stack([np.stack([np.sort(rng.choice(nkb, kk, replace=False)) for _ in range(nqb)])
                     for _ in range(2)])
    _attn_with_oracle_mask(S, q, k, v, rows)


@pytest.mark.parametrize("block", [128, 64])
@pytest.mark.parametrize("d,H,n_q,n_kv", [(64, 3, 128 * 37 + 5, 128 * 23 + 77), (128, 2, 128 * 41, 128 * 19 + 1)])
def test_attention_with_uneven_row_counts(S, block, d, H, n_q, n_kv):
    """The attention ABI takes a count per row: rows of 1 to nkb kept blocks (first, last and
    ragged blocks among them) in one launch, with kmax above every count, so the persistent
    slots carry items of very different lengths; every query block compared."""
    q, k, v = synth.make_qkv(n_q, n_kv, H, d, [800 + 3 * h + block for h in range(H)], device="cuda")
    nqb, nkb = O.num_blocks(n_q, block), O.num_blocks(n_kv, block)
    kmax = nkb + 3
    rng = np.random.default_rng(n_q + n_kv + block)
    rows = np.full((H, nqb, kmax), -1, dtype=np.int32)
    counts = rng.integers(1, nkb + 1, size=(H, nqb))
    counts[0, 0], counts[-1, -1] = 1, nkb
    for h in range(H):
        for i in range(nqb):
            rows[h, i, :counts[h, i]] = np.sort(rng.choice(nkb, counts[h, i], replace=False))
    rows[0, 1, :1] = nkb - 1   # a row holding only the ragged last block
    counts[0, 1] = 1
    idx = torch.from_numpy(rows).cuda()
    cnt = torch.from_numpy(counts.astype(np.int32)).cuda()
    o, lse = S.attn(q, k, v, idx, cnt, block=block)
    assert S.device_status() == S.OK
    qb, kb, vb = bits(q), bits(k), bits(v)
    o_np, lse_np = o.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(H):
        qf, kf, vf = _f64(qb[h]), _f64(kb[h]), _f64(vb[h])
        rows_h = np.where(np.arange(kmax)[None, :] < counts[h][:, None], rows[h], -1)
        for i, (o_ref, lse_ref) in enumerate(O.block_sparse_attention(qf, kf, vf, rows_h, range(nqb), block=block)):
            s, e = O.block_token_range(i, n_q, block)
            check_output(o_np[h, s:e], o_ref, f"h{h} qb{i}")
            assert np.abs(lse_np[h, s:e] - lse_ref).max() <= LSE_ABS


@pytest.mark.parametrize("world", [2, 3, 5])
def test_head_shards_equal_the_whole(S, world):
    """The head split of the multi-GPU path, on one GPU: each rank's slice (its own inputs,
    drawn as make_shard_inputs draws them) run through selection + attention gives exactly the
    rows, outputs and LSEs of those heads in the one-rank run (per-head masks, no exchange)."""
    from block_sparse_attention_tok_b200 import shard
    sc = synth.Scale("shard_check_clip2", heads=7, head_dim=128, n_q=128 * 9 + 40, n_text=256, n_ctx=1024,
                     n_cur=128 * 9 + 40, clip=2, density=0.3)
    q, k, v = synth.make_qkv(sc.n_q, sc.n_kv, sc.heads, sc.head_dim,
                             [sc.seed(h, 0, 0, 0) for h in range(sc.heads)], device="cuda")
    seg = (sc.n_text, sc.n_ctx, sc.n_cur)
    o, lse, idx, cnt = S.forward(q, k, v, *seg, sc.clip, sc.density)
    for rank in range(world):
        h0, h1 = shard.head_range(rank, world, sc.heads)
        if h0 == h1:
            continue
        qs, ks, vs = shard.make_shard_inputs(sc, rank, world, device="cuda")
        assert torch.equal(qs, q[h0:h1]) and torch.equal(ks, k[h0:h1]) and torch.equal(vs, v[h0:h1])
        o_r, lse_r, idx_r, cnt_r = S.forward(qs, ks, vs, *seg, sc.clip, sc.density)
        assert torch.equal(idx_r, idx[h0:h1]) and torch.equal(cnt_r, cnt[h0:h1])
        assert torch.equal(o_r, o[h0:h1]) and torch.equal(lse_r, lse[h0:h1])
    assert S.device_status() == S.OK


def test_many_items_per_slot(S):
    """More (head, query block) items than two per CTA slot: exercises the per-slot item
    sequence (Q buffer reuse, O handover between items) of the persistent kernel."""
    q, k, v = synth.make_qkv(128 * 90 + 37, 1100, 8, 128, [61 + h for h in range(8)], device="cuda")
    stats = _run_case(S, q, k, v, 128, 256, 716, 2, 0.5, 0, qblocks_per_head=lambda n: range(0, n, 7))
    assert stats["rows"] == 8 * 91


@pytest.mark.parametrize("d,heads", [(64, 10), (128, 9)])
def test_many_heads_ragged_tail(S, d, heads):
    """An odd number of heads (more than a few) with a ragged last query and KV block, every
    row and every output compared."""
    n_cur = 128 * 6 + 5
    q, k, v = synth.make_qkv(n_cur, 256 + 512 + n_cur, heads, d, [300 + h for h in range(heads)], device="cuda")
    stats = _run_case(S, q, k, v, 256, 512, n_cur, 2, 0.3, 0)
    assert stats["rows"] == heads * 7


@pytest.mark.parametrize("d", [64, 128])
def test_row_max_jump_in_some_rows_only(S, d):
    """Rows 0-15 of every query block meet a much larger logit in a late KV block, so their
    running max moves (O rescale) while the other rows of the same warp keep theirs."""
    n_q, n_kv = 128 * 6, 128 * 8
    q, k, v = synth.make_qkv(n_q, n_kv, 2, d, [71, 72], device="cuda")
    qv = q.view(2, 6, 128, d)
    qv[:, :, :16, 0] = 16.0
    k[:, 6 * 128:7 * 128, 0] = 16.0
    rows = np.tile(np.array([0, 2, 3, 6]), (2, 6, 1))
    _attn_with_oracle_mask(S, q, k, v, rows)
    # and the same through the full path with every block kept
    _run_case(S, q, k, v, 0, 0, n_kv, 2, 1.0, 0)


def test_dense_density_one_matches_oracle(S):
    q, k, v = synth.make_qkv(640, 1100, 2, 128, [11, 12], device="cuda")
    stats = _run_case(S, q, k, v, 100, 300, 700, 2, 1.0, 0)
    assert stats["identical"] == stats["rows"]


def test_forced_only_rows(S):
    # Clip 1 where the text + pyramid prefix fills the budget: K_topk = 0.
    q, k, v = synth.make_qkv(512, 128 * 12, 2, 128, [21, 22], device="cuda")
    plan = S.make_plan(512, 256, 768, 512, 1, 0.25)
    assert plan.k_topk == 0 and plan.k_total == 8
    stats = _run_case(S, q, k, v, 256, 768, 512, 1, 0.25, 0)
    assert stats["identical"] == stats["rows"]


def test_planted_ties_go_to_lower_index(S):
    # Duplicate KV blocks have bit-identical pooled means and scores on the GPU as well.
    H, d = 2, 128
    q, k, v = synth.make_qkv(256, 128 * 10, H, d, [31, 32], device="cuda")
    for src, dst in ((3, 7), (4, 8), (5, 9)):
        k[:, dst * 128:(dst + 1) * 128] = k[:, src * 128:(src + 1) * 128]
    idx, cnt, sc = S.select(q, k, 128, 0, 128 * 9, 2, 0.5, 0, want_scores=True)
    ref_idx, _ = O.select(bits(q), bits(k), 128, 0, 2, 0.5, 0)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    s = sc.cpu().numpy()
    assert np.array_equal(s[:, :, 3], s[:, :, 7]) and np.array_equal(s[:, :, 5], s[:, :, 9])


def test_zero_queries_is_noop(S):
    q = torch.empty(2, 0, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(2, 300, 64, dtype=torch.bfloat16, device="cuda")
    o, lse, idx, cnt = S.forward(q, k, k.clone(), 100, 100, 100, 2, 0.5)
    assert o.shape == (2, 0, 64) and S.device_status() == S.OK


def test_out_of_range_index_is_clamped_and_reported(S):
    q, k, v = synth.make_qkv(256, 512, 1, 64, [41], device="cuda")
    idx = torch.tensor([[[0, 1], [2, 99]]], dtype=torch.int32, device="cuda")   # 99 >= nkb = 4
    cnt = torch.tensor([[2, 2]], dtype=torch.int32, device="cuda")
    S.device_status(clear=True)
    S.attn(q, k, v, idx, cnt)
    assert S.device_status(clear=True) == S.ERR_DEVICE_BOUNDS
    cnt = torch.tensor([[2, 7]], dtype=torch.int32, device="cuda")             # 7 > kmax = 2
    idx = torch.tensor([[[0, 1], [2, 3]]], dtype=torch.int32, device="cuda")
    S.attn(q, k, v, idx, cnt)
    assert S.device_status(clear=True) == S.ERR_DEVICE_BOUNDS
    idx = torch.tensor([[[0, 1], [2, 3]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[2, 2]], dtype=torch.int32, device="cuda")
    S.attn(q, k, v, idx, cnt)
    assert S.device_status(clear=True) == S.OK


def test_bounded_wait_reports_timeout_and_context_survives(S):
    """A wait on an mbarrier that nothing completes ends at its 2 s limit with a timeout in the
    status word (no trap, no hang); afterwards the same context still computes correctly."""
    import time
    S.device_status(clear=True)
    t0 = time.perf_counter()
    S.selftest_wait_timeout()
    code = S.device_status(clear=True)
    elapsed = time.perf_counter() - t0
    assert code == S.ERR_DEVICE_TIMEOUT
    assert 1.5 < elapsed < 60.0
    assert S.device_status(clear=True) == S.OK      # the word was cleared
    q, k, v = synth.make_qkv(640, 1100, 2, 128, [61, 62], device="cuda")
    stats = _run_case(S, q, k, v, 100, 300, 700, 2, 0.5, 0)
    assert stats["rows"] == 2 * 5


def test_custom_softmax_scale(S):
    q, k, v = synth.make_qkv(300, 700, 1, 128, [51], device="cuda")
    rows = np.array([[[0, 2, 5], [1, 3, 4], [0, 1, 2]]])
    idx = torch.from_numpy(rows.astype(np.int32)).cuda()
    cnt = torch.full((1, 3), 3, dtype=torch.int32, device="cuda")
    o, lse = S.attn(q, k, v, idx, cnt, sm_scale=0.05)
    qf, kf, vf = (_f64(bits(x)[0]) for x in (q, k, v))
    outs = O.block_sparse_attention(qf, kf, vf, rows[0], [0, 1, 2], sm_scale=0.05)
    o_np = o.float().cpu().numpy()[0]
    for i, (o_ref, _) in enumerate(outs):
        s, e = O.block_token_range(i, 300)
        check_output(o_np[s:e], o_ref, f"qb{i}")


def _sampled(nqb):
    rng = np.random.default_rng(nqb)
    return sorted({0, nqb - 1, *rng.choice(nqb, 3, replace=False).tolist()})


def _sampled3(nqb):
    rng = np.random.default_rng(nqb + 1)
    return sorted({0, nqb - 1, int(rng.integers(nqb))})


# Heads whose outputs are compared at full size (masks and scores: every head).
_OUT_HEADS = [0, 1, 7, 16, 23, 31]


@pytest.mark.slow
@pytest.mark.parametrize("name", [synth.MID_CLIP1.name, synth.FINAL_CLIP1_RAGGED.name, synth.FINAL_CLIP2.name])
@pytest.mark.parametrize("mode", [0, 1])
def test_full_size_scales(S, name, mode):
    """The three large workloads, launched as bench.py launches them (all 32 heads in one call),
    in both budget readings: every mask row of every head, every block score, and the outputs
    of six heads on sampled query blocks plus every block whose mask differs from the oracle's."""
    sc = synth.WORKLOADS[name]
    q, k, v = synth.make_scale_inputs(sc, device="cuda")
    stats = _run_case(S, q, k, v, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density, mode,
                      qblocks_per_head=_sampled3, out_heads=_OUT_HEADS, label=f"{name} budget {mode}")
    assert stats["rows"] == sc.heads * -(-sc.n_q // 128)
    del q, k, v
    torch.cuda.empty_cache()


@pytest.mark.slow
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("scale_index", [0, 1, 2, 3])
@pytest.mark.parametrize("layer", [0, 35])
def test_schedule_scales(S, scale_index, layer, mode):
    """The four refined scales of the Clip-1 schedule at layers 0 and 35, both budget readings:
    every mask row of all 32 heads; outputs of two heads on sampled query blocks plus every
    block whose mask differs."""
    sc = synth.SCHEDULE_CLIP1[scale_index]
    q, k, v = synth.make_scale_inputs(sc, device="cuda", layer=layer, scale_index=scale_index)
    stats = _run_case(S, q, k, v, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density, mode,
                      qblocks_per_head=_sampled3, out_heads=[0, 31],
                      label=f"schedule s{scale_index + 1} layer {layer} budget {mode}")
    assert stats["rows"] == sc.heads * -(-sc.n_q // 128)
    del q, k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n_cand", [3965, 3966])
def test_topk_path_boundary(S, n_cand):
    """3,965 candidates is the largest row the warp Top-K takes (124 keys per lane, 3 slots kept
    for the row's alignment offset); 3,966 goes to the CTA-per-row radix Top-K. Both must give
    the oracle's masks."""
    n_text, n_q = 128, 256
    q, k, v = synth.make_qkv(n_q, n_text + 128 * n_cand, 1, 64, [4000 + n_cand], device="cuda")
    stats = _run_case(S, q, k, v, n_text, 0, 128 * n_cand, 2, 0.05, 0)
    assert stats["rows"] == 2


@pytest.mark.slow
def test_max_candidates(S):
    """16,384 candidates per row (the radix Top-K's shared-memory limit), 2.1 M KV tokens."""
    n_text, n_cand = 128, 16384
    q, k, v = synth.make_qkv(200, n_text + 128 * n_cand, 1, 64, [4321], device="cuda")
    stats = _run_case(S, q, k, v, n_text, 0, 128 * n_cand, 2, 0.01, 0)
    assert stats["rows"] == 2
    del q, k, v
    torch.cuda.empty_cache()


def test_wider_index_buffer_and_single_head(S):
    """kmax larger than K_total: only the first K_total entries of a row are written, the rest
    keep the caller's values, and attention reads only cnt entries; one head, one query row."""
    n_text, n_ctx, n_cur = 128, 256, 513
    q, k, v = synth.make_qkv(1, n_text + n_ctx + n_cur, 1, 128, [77], device="cuda")
    plan = S.make_plan(1, n_text, n_ctx, n_cur, 2, 0.4)
    kt = int(plan.k_total)
    idx = torch.full((1, 1, kt + 5), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    S.select(q, k, n_text, n_ctx, n_cur, 2, 0.4, idx=idx, cnt=cnt)
    o, lse = S.attn(q, k, v, idx, cnt)
    assert S.device_status() == S.OK
    g = idx.cpu().numpy()[0, 0]
    assert (g[kt:] == -7).all() and int(cnt.item()) == kt
    qf, kf, vf = (O.bf16_bits_to_f64(bits(x)[0]) for x in (q, k, v))
    rows, _ = O.select_head(qf, kf, n_text, n_ctx, 2, 0.4)
    assert np.array_equal(g[:kt], rows[0])
    (o_ref, lse_ref), = O.block_sparse_attention(qf, kf, vf, rows, [0])
    check_output(o.float().cpu().numpy()[0], o_ref, "single row")
    assert abs(float(lse.cpu()[0, 0]) - float(lse_ref[0])) <= LSE_ABS


@pytest.mark.parametrize("n_q,segs,H,d,clip,density,mode", [
    (1024, (256, 768, 1024), 2, 64, 2, 0.25, 0),      # the tiny Clip-2 scale
    (300, (100, 300, 333), 3, 128, 2, 0.4, 0),        # ragged tails; nkb = 6 (not a multiple of 4)
    (1, (128, 0, 129), 1, 64, 2, 0.5, 0),             # one query row, one ragged KV block
    (640, (256, 512, 700), 2, 128, 1, 0.6, 1),        # Clip 1, candidates reading
])
def test_writes_stay_inside_outputs(S, n_q, segs, H, d, clip, density, mode):
    """Every output of selection and attention sits inside a larger buffer whose guard bands
    (before and after) hold a known pattern: after the calls the bands are unchanged, so no
    kernel writes past its idx, cnt, score, workspace, o or lse range on these shapes."""
    lib = S.load()
    G = 4096                                  # guard elements on each side
    n_kv = sum(segs)
    q, k, v = synth.make_qkv(n_q, n_kv, H, d, [900 + h for h in range(H)], device="cuda")
    plan = S.make_plan(n_q, *segs, clip, density, mode)
    nqb, nkb, kt = int(plan.nqb), int(plan.nkb), int(plan.k_total)
    kmax = kt + 3
    idx_buf = torch.full((2 * G + H * nqb * kmax,), -77, dtype=torch.int32, device="cuda")
    cnt_buf = torch.full((2 * G + H * nqb,), -77, dtype=torch.int32, device="cuda")
    sc_buf = torch.full((2 * G + H * nqb * nkb,), -7.5, dtype=torch.float32, device="cuda")
    ws_bytes = S.workspace_size(H, n_q, *segs, d)
    ws_buf = torch.full((2 * G * 4 + ws_bytes,), 0xA5, dtype=torch.uint8, device="cuda")
    o_buf = torch.full((2 * G + H * n_q * d,), 3.0, dtype=torch.bfloat16, device="cuda")
    lse_buf = torch.full((2 * G + H * n_q,), 3.0, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream or None
    for scores in (False, True):
        rc = lib.sparstar_select(q.data_ptr(), k.data_ptr(), H, n_q, S.Segments(*segs), d, clip, density, mode,
                                 idx_buf[G:].data_ptr(), cnt_buf[G:].data_ptr(), kmax,
                                 sc_buf[G:].data_ptr() if scores else None, ws_buf[4 * G:].data_ptr(), ws_bytes, st)
        assert rc == S.OK
    rc = lib.sparstar_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), H, n_q, n_kv, d, idx_buf[G:].data_ptr(),
                           cnt_buf[G:].data_ptr(), kmax, 0.0, o_buf[G:].data_ptr(), lse_buf[G:].data_ptr(), st)
    assert rc == S.OK
    assert S.device_status() == S.OK

    def guards_intact(buf, n, fill, unit=1):
        b = buf.cpu()
        head, tail = b[:unit * G], b[unit * G + n:]
        return bool((head == fill).all()) and bool((tail == fill).all())

    assert guards_intact(idx_buf, H * nqb * kmax, -77)
    assert guards_intact(cnt_buf, H * nqb, -77)
    assert guards_intact(sc_buf, H * nqb * nkb, -7.5)
    assert guards_intact(ws_buf, ws_bytes, 0xA5, unit=4)
    assert guards_intact(o_buf, H * n_q * d, 3.0)
    assert guards_intact(lse_buf, H * n_q, 3.0)
    # inside idx, entries past K_total of each row keep the caller's values
    rows = idx_buf[G:G + H * nqb * kmax].view(H, nqb, kmax).cpu()
    assert bool((rows[:, :, kt:] == -77).all())
    assert bool((cnt_buf[G:G + H * nqb].cpu() == kt).all())


@pytest.mark.parametrize("n_words", [4, 4 * 1000003, 4 * (148 * 4 * 512 * 4 + 3)])
def test_read_probe_reads_every_chunk_once(S, n_words):
    """The bandwidth probe's XOR fold equals the XOR of every 32-bit word of the buffer (each
    16-byte chunk read exactly once, including a tail that is not a multiple of the grid)."""
    g = torch.Generator(device="cuda").manual_seed(n_words)
    buf = torch.randint(-2**31, 2**31 - 1, (n_words,), dtype=torch.int32, device="cuda", generator=g)
    sink = S.read_probe(buf)
    assert S.device_status() == S.OK
    want = np.bitwise_xor.reduce(buf.cpu().numpy().view(np.uint32))
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)
