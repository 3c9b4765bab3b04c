"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against one of: a hand-worked fixture under tests/golden/, a
closed form, a library routine that computes the same special case (torch avg_pool1d,
scaled_dot_product_attention, softmax), brute force over token pairs, or exhaustive
enumeration of Top-K subsets. Together they are chosen so that a dropped term, a wrong
sign, a wrong divisor, a transposed operand or a wrong tie rule fails at least one test.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import sparstar_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


# ----------------------------------------------------------------------------- widening

def test_bf16_widening_known_bit_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x7F7F, 0x0001], dtype=np.uint16)
    got = O.bf16_bits_to_f64(bits)
    want = [1.0, -2.0, 1.0 + 2.0 ** -7, 0.0, -0.0, (2 - 2.0 ** -7) * 2.0 ** 127, 2.0 ** -133]
    assert got.tolist() == want
    assert math.copysign(1.0, got[4]) == -1.0


def test_bf16_widening_matches_torch_cast():
    x = _rand_bf16((4096,), 3, 10.0)
    assert np.array_equal(O.bf16_bits_to_f64(_bits(x)), x.to(torch.float64).numpy())


# ----------------------------------------------------------------------------- budgets

@pytest.mark.parametrize("n_text,n_ctx,n_cur,clip,density,nkb,n_forced,lit,alt", [
    # tiny clip-2 scale: 256 text + 768 ref + 1024 cur
    (256, 768, 1024, 2, 0.25, 16, 2, (4, 2), (6, 4)),
    # mid refined scale, clip 1: 512 + 4096 + 18432
    (512, 4096, 18432, 1, 0.1875, 180, 36, (36, 0), (63, 27)),
    # 720p final scale, clip 1, ragged: 512 + 8192 + 72000
    (512, 8192, 72000, 1, 0.09375, 631, 68, (68, 0), (121, 53)),
    # 720p final scale, clip 2: 512 + 72192 + 72192
    (512, 72192, 72192, 2, 0.09375, 1132, 4, (107, 103), (110, 106)),
    # schedule scale 1: 512 + 8192 + 8192 at 0.625
    (512, 8192, 8192, 1, 0.625, 132, 68, (83, 15), (108, 40)),
    (512, 8192, 18432, 1, 0.1875, 212, 68, (68, 0), (95, 27)),
    (512, 8192, 36864, 1, 0.1875, 356, 68, (68, 0), (122, 54)),
    (512, 8192, 72192, 1, 0.09375, 632, 68, (68, 0), (121, 53)),
])
def test_budget_closed_form(n_text, n_ctx, n_cur, clip, density, nkb, n_forced, lit, alt):
    # Worked by hand: nkb = ceil(Nkv/128); forced = ceil(text[+ctx]/128);
    # literal K_total = max(ceil(density*nkb), forced); alt K_topk = ceil(density*cand).
    assert O.num_blocks(n_text + n_ctx + n_cur) == nkb
    assert O.forced_block_count(n_text, n_ctx, clip) == n_forced
    assert O.row_budget(nkb, n_forced, density, O.BUDGET_LITERAL) == lit
    assert O.row_budget(nkb, n_forced, density, O.BUDGET_CANDIDATES) == alt


def test_ragged_partition():
    assert O.num_blocks(72000) == 563
    assert O.block_token_range(562, 72000) == (71936, 72000)  # 64 valid tokens
    assert O.num_blocks(0) == 0 and O.num_blocks(1) == 1 and O.num_blocks(128) == 1
    assert O.forced_block_count(200, 300, 1) == 4   # 500 tokens -> 4 blocks (block 3 mixes ctx/cur)
    assert O.forced_block_count(200, 300, 2) == 2   # block 1 holds text and context tokens


# ----------------------------------------------------------------------------- pooling

@pytest.mark.parametrize("n", [1, 64, 127, 128, 129, 255, 384, 1000])
def test_pool_matches_library_avg_pool(n):
    x = _rand_bf16((n, 32), 10 + n).to(torch.float64)
    want = torch.nn.functional.avg_pool1d(x.T[None], 128, 128, ceil_mode=True)[0].T
    got = O.pool_blocks(x.numpy())
    assert got.shape == (O.num_blocks(n), 32)
    np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-14)


def test_pool_constant_blocks_closed_form():
    # K constant inside each block (ragged tail of 5 tokens) -> the mean is that constant.
    consts = np.array([[1.5, -2.0], [0.25, 3.0], [-7.0, 0.5]])
    x = np.concatenate([np.tile(consts[0], (128, 1)), np.tile(consts[1], (128, 1)), np.tile(consts[2], (5, 1))])
    assert np.array_equal(O.pool_blocks(x), consts)


# ----------------------------------------------------------------------------- scores

def test_scores_equal_mean_of_token_pair_logits_bruteforce():
    # Bilinearity: mean(q_i).mean(k_j)/sqrt(d) = mean over token pairs of q_t.k_u/sqrt(d).
    d, block = 4, 3
    q = _rand_bf16((7, d), 1).double().numpy()
    k = _rand_bf16((8, d), 2).double().numpy()
    S = O.block_scores(O.pool_blocks(q, block), O.pool_blocks(k, block))
    for i in range(O.num_blocks(7, block)):
        for j in range(O.num_blocks(8, block)):
            ts = range(*O.block_token_range(i, 7, block))
            us = range(*O.block_token_range(j, 8, block))
            acc = 0.0
            for t in ts:
                for u in us:
                    acc += sum(q[t, c] * k[u, c] for c in range(d)) / math.sqrt(d)
            assert abs(S[i, j] - acc / (len(ts) * len(us))) < 1e-12


def test_scores_onehot_query():
    d = 16
    k = _rand_bf16((300, d), 5).double().numpy()
    kbar = O.pool_blocks(k)
    for c in (0, 7, 15):
        q = np.zeros((128, d))
        q[:, c] = 1.0
        S = O.block_scores(O.pool_blocks(q), kbar)
        np.testing.assert_allclose(S[0], kbar[:, c] / 4.0, rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------- Top-K

def _exhaustive_choice(scores, n_forced, k_topk):
    """Max score sum over subsets; among equal sums the lexicographically smallest tuple."""
    cands = list(range(n_forced, len(scores)))
    best, best_key = None, None
    for sub in itertools.combinations(cands, k_topk):
        key = (-sum(scores[j] for j in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return list(range(n_forced)) + sorted(best)


@pytest.mark.parametrize("seed", range(40))
def test_topk_matches_exhaustive_enumeration(seed):
    rng = np.random.default_rng(seed)
    nkb = int(rng.integers(2, 13))
    n_forced = int(rng.integers(0, nkb))
    k_topk = int(rng.integers(0, min(4, nkb - n_forced) + 1))
    # integer-valued scores make exact ties frequent
    scores = rng.integers(-3, 4, size=nkb).astype(np.float64) if seed % 2 else rng.normal(size=nkb)
    got = O.select_row(scores, n_forced, k_topk).tolist()
    assert got == _exhaustive_choice(scores.tolist(), n_forced, k_topk)


def test_topk_signed_zero_ties_and_lower_index():
    scores = np.array([9.0, -0.0, 0.0, -0.0, -1.0])
    assert O.select_row(scores, 1, 2).tolist() == [0, 1, 2]
    assert O.select_row(scores, 1, 1).tolist() == [0, 1]
    assert O.select_row(np.array([5.0, 1.0, np.nan, 0.5]), 0, 3).tolist() == [0, 1, 3]


def _beats(a, ia, b, ib):
    """Pairwise ranking: a number beats NaN; between numbers the larger wins (-0.0 == +0.0);
    equal scores, and two NaNs, go to the lower index."""
    na, nb = math.isnan(a), math.isnan(b)
    if na != nb:
        return nb
    if not na and a != b:
        return a > b
    return ia < ib


def _dominance_choice(scores, n_forced, k_topk):
    """The unique subset of k_topk candidates each of which beats every unchosen candidate."""
    cands = list(range(n_forced, len(scores)))
    found = [sub for sub in itertools.combinations(cands, k_topk)
             if all(_beats(scores[c], c, scores[u], u) for c in sub for u in cands if u not in sub)]
    assert len(found) == 1
    return list(range(n_forced)) + list(found[0])


@pytest.mark.parametrize("seed", range(60))
def test_topk_special_values_match_pairwise_dominance(seed):
    # NaN, +-inf and +-0 mixed with small integers (frequent ties)
    rng = np.random.default_rng(1000 + seed)
    nkb = int(rng.integers(2, 11))
    n_forced = int(rng.integers(0, nkb))
    k_topk = int(rng.integers(0, nkb - n_forced + 1))
    pool = np.array([np.nan, np.inf, -np.inf, 0.0, -0.0, 1.0, -1.0, 2.0])
    scores = rng.choice(pool, size=nkb)
    got = O.select_row(scores, n_forced, k_topk).tolist()
    assert got == _dominance_choice(scores.tolist(), n_forced, k_topk)


def test_topk_nan_below_negative_infinity():
    assert O.select_row(np.array([np.nan, -np.inf]), 0, 1).tolist() == [1]
    assert O.select_row(np.array([np.nan, -np.inf, np.nan]), 0, 2).tolist() == [0, 1]


def test_forced_only_rows_ignore_values():
    rng = np.random.default_rng(7)
    for _ in range(10):
        S = rng.normal(size=(6, 20)) * 100
        rows = O.select_rows(S, 9, 0)
        assert rows.tolist() == [list(range(9))] * 6


def test_full_budget_keeps_every_block():
    S = np.random.default_rng(1).normal(size=(3, 11))
    k_total, k_topk = O.row_budget(11, 2, 1.0)
    assert (k_total, k_topk) == (11, 9)
    assert O.select_rows(S, 2, k_topk).tolist() == [list(range(11))] * 3


# ----------------------------------------------------------------------------- golden

def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_worked_example_golden_selection():
    g = _load("worked_example_block2.json")
    b, d = g["block"], g["d"]
    q, k = np.array(g["q"], float), np.array(g["k"], float)
    np.testing.assert_array_equal(O.pool_blocks(q, b), np.array(g["qbar"], float))
    np.testing.assert_array_equal(O.pool_blocks(k, b), np.array(g["kbar"], float))
    S = O.block_scores(O.pool_blocks(q, b), O.pool_blocks(k, b))
    np.testing.assert_allclose(S * math.sqrt(d), np.array(g["scores_times_sqrt2"], float), atol=1e-14)
    for case in g["cases"]:
        nkb = O.num_blocks(len(k), b)
        n_forced = O.forced_block_count(g["n_text"], g["n_ctx"], case["clip"], b)
        assert O.row_budget(nkb, n_forced, case["density"], case["mode"]) == (case["k_total"], case["k_topk"])
        rows, _ = O.select_head(q, k, g["n_text"], g["n_ctx"], case["clip"], case["density"], case["mode"], b)
        assert rows.tolist() == case["rows"], case


def test_worked_example_golden_attention_closed_form():
    g = _load("worked_example_block2.json")
    b = g["block"]
    q, k, v = (np.array(g[x], float) for x in "qkv")
    rows, _ = O.select_head(q, k, g["n_text"], g["n_ctx"], 2, 0.5, 0, b)
    (o, lse), = O.block_sparse_attention(q, k, v, rows, [0], block=b)
    a, bb = 1 / math.sqrt(2), 4 / math.sqrt(2)
    z = 2 * math.exp(a) + math.exp(bb)
    assert abs(o[0, 0] - 2 * math.exp(a) / z) < 1e-14
    assert abs(o[0, 1] - math.exp(bb) / z) < 1e-14
    assert abs(lse[0] - math.log(z)) < 1e-14


def test_tie_golden():
    g = _load("tie_example_block2.json")
    q, k = np.array(g["q"], float), np.array(g["k"], float)
    rows, _ = O.select_head(q, k, g["n_text"], g["n_ctx"], g["clip"], g["density"], 0, g["block"])
    assert rows.tolist() == g["rows"]


# ----------------------------------------------------------------------------- attention

def _sdpa_f64(q, k, v, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], scale=scale)
    return out[0, 0].numpy()


@pytest.mark.parametrize("n_q,n_kv,d", [(128, 384, 64), (200, 300, 32), (1, 129, 16), (255, 127, 128)])
def test_density_one_equals_library_attention(n_q, n_kv, d):
    q = _rand_bf16((n_q, d), 11).double().numpy()
    k = _rand_bf16((n_kv, d), 12).double().numpy()
    v = _rand_bf16((n_kv, d), 13).double().numpy()
    rows, _ = O.select_head(q, k, 0, 0, 2, 1.0)
    assert rows.shape[1] == O.num_blocks(n_kv)
    outs = O.block_sparse_attention(q, k, v, rows, range(O.num_blocks(n_q)))
    o = np.concatenate([x[0] for x in outs])
    np.testing.assert_allclose(o, _sdpa_f64(q, k, v, 1 / math.sqrt(d)), rtol=0, atol=1e-12)


def test_lse_matches_library_logsumexp():
    q = _rand_bf16((130, 64), 21).double().numpy()
    k = _rand_bf16((500, 64), 22).double().numpy()
    v = _rand_bf16((500, 64), 23).double().numpy()
    rows = np.array([[0, 2, 3], [1, 3, -1]])
    outs = O.block_sparse_attention(q, k, v, rows, [0, 1])
    for i, (o, lse) in enumerate(outs):
        toks = np.concatenate([np.arange(j * 128, min(j * 128 + 128, 500)) for j in rows[i] if j >= 0])
        s, e = O.block_token_range(i, 130)
        logits = torch.from_numpy(q[s:e] @ k[toks].T / 8.0)
        np.testing.assert_allclose(lse, torch.logsumexp(logits, 1).numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(o, _sdpa_f64(q[s:e], k[toks], v[toks], 1 / 8.0), rtol=0, atol=1e-12)


def test_retained_mass_identity_and_block_energy():
    d = 32
    q = _rand_bf16((256, d), 31).double().numpy()
    k = _rand_bf16((640, d), 32).double().numpy()
    v = _rand_bf16((640, d), 33).double().numpy()
    rows, _ = O.select_head(q, k, 128, 0, 2, 0.4)          # 5 blocks, forced 1, keep 2
    dense = O.dense_attention(q, k, v, [0, 1])
    kept = O.block_sparse_attention(q, k, v, rows, [0, 1])
    for i in range(2):
        mass = O.retained_mass(kept[i][1], dense[i][1])
        s, e = O.block_token_range(i, 256)
        P = torch.softmax(torch.from_numpy(q[s:e] @ k.T) / math.sqrt(d), dim=1).numpy()
        toks = O.kept_token_index(rows[i], 640)
        np.testing.assert_allclose(mass, P[:, toks].sum(1), rtol=0, atol=1e-12)
        assert abs(O.block_energy(q, k, i, rows[i]) - P[:, toks].sum() / (e - s)) < 1e-12
        assert 0 < mass.min() and mass.max() <= 1 + 1e-12


def test_constant_v_gives_constant_output_and_convexity():
    q = _rand_bf16((128, 64), 41).double().numpy()
    k = _rand_bf16((512, 64), 42).double().numpy()
    v = np.full((512, 64), 0.375)
    rows = np.array([[0, 3]])
    (o, _), = O.block_sparse_attention(q, k, v, rows, [0])
    np.testing.assert_allclose(o, 0.375, rtol=0, atol=1e-14)
    v = _rand_bf16((512, 64), 43).double().numpy()
    (o, _), = O.block_sparse_attention(q, k, v, rows, [0])
    toks = O.kept_token_index([0, 3], 512)
    assert np.all(o <= v[toks].max(0) + 1e-12) and np.all(o >= v[toks].min(0) - 1e-12)


def test_unkept_blocks_do_not_matter_kept_do():
    q = _rand_bf16((128, 64), 51).double().numpy()
    k = _rand_bf16((512, 64), 52).double().numpy()
    v = _rand_bf16((512, 64), 53).double().numpy()
    rows = np.array([[1, 2]])
    (o1, l1), = O.block_sparse_attention(q, k, v, rows, [0])
    k2, v2 = k.copy(), v.copy()
    k2[:128] += 5.0
    v2[384:] -= 3.0
    (o2, l2), = O.block_sparse_attention(q, k2, v2, rows, [0])
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    v2[200] += 1.0
    (o3, _), = O.block_sparse_attention(q, k2, v2, rows, [0])
    assert not np.array_equal(o1, o3)


def test_heads_are_independent():
    H, d = 3, 64
    q = _rand_bf16((H, 256, d), 61)
    k = _rand_bf16((H, 640, d), 62)
    idx, S = O.select(_bits(q), _bits(k), 128, 128, 2, 0.5)
    perm = [2, 0, 1]
    idx_p, S_p = O.select(_bits(q[perm]), _bits(k[perm]), 128, 128, 2, 0.5)
    assert np.array_equal(idx_p, idx[perm]) and np.array_equal(S_p, S[perm])


# ---------------------------------------------------------------- token-wise bound and mass

def test_token_bound_equals_best_subset_bruteforce():
    """The bound is the best mass over every key subset of the budget's size (enumerated)."""
    rng = np.random.default_rng(71)
    q = rng.normal(size=(3, 8))
    k = rng.normal(size=(10, 8)) * 1.5
    P = torch.softmax(torch.from_numpy(q @ k.T) / math.sqrt(8), dim=1).numpy()
    for budget in range(1, 11):
        best = np.array([max(P[t, list(c)].sum() for c in itertools.combinations(range(10), budget))
                         for t in range(3)])
        np.testing.assert_allclose(O.token_topk_bound(q, k, budget), best, rtol=0, atol=1e-12)


def test_token_bound_closed_forms():
    rng = np.random.default_rng(72)
    k = rng.normal(size=(37, 16))
    # equal logits (q = 0): every token holds 1/n, the bound is budget / n
    q0 = np.zeros((2, 16))
    for b in (1, 5, 37):
        np.testing.assert_allclose(O.token_topk_bound(q0, k, b), b / 37.0, rtol=0, atol=1e-14)
    # the full budget holds everything
    q = rng.normal(size=(4, 16))
    np.testing.assert_allclose(O.token_topk_bound(q, k, 37), 1.0, rtol=0, atol=1e-12)
    # one key dominating by 60 logits: a single kept token already holds (almost) all of it
    k2 = k.copy()
    k2[11] = q[0] * 60.0 * 4.0 / np.dot(q[0], q[0])
    assert O.token_topk_bound(q[:1], k2, 1)[0] >= 1 - 1e-15 > O.token_topk_bound(q[:1], k, 1)[0]


def test_token_bound_dominates_block_mask_and_is_concave():
    """Any mask with B kept tokens retains at most the bound; the bound grows with B by
    non-increasing steps (the sorted probabilities); per-row budgets are honoured."""
    d = 32
    q = _rand_bf16((256, d), 73).double().numpy()
    k = _rand_bf16((700, d), 74).double().numpy()
    v = _rand_bf16((700, d), 75).double().numpy()
    rows, _ = O.select_head(q, k, 128, 128, 2, 0.5)
    E, U, R, Ur = O.mass_report(q, k, rows, [0, 1])
    assert (Ur >= R - 1e-12).all() and (U >= E - 1e-12).all()
    # R agrees with the LSE form of the retained mass
    dense = O.dense_attention(q, k, v, [0, 1])
    kept = O.block_sparse_attention(q, k, v, rows, [0, 1])
    np.testing.assert_allclose(R, np.concatenate([O.retained_mass(kept[i][1], dense[i][1]) for i in range(2)]),
                               rtol=0, atol=1e-12)
    u = np.stack([O.token_topk_bound(q[:5], k, b) for b in range(1, 701)])
    steps = np.diff(np.vstack([np.zeros((1, 5)), u]), axis=0)
    assert (steps >= -1e-15).all() and (np.diff(steps, axis=0) <= 1e-15).all()
    per_row = O.token_topk_bound(q[:3], k, np.array([5, 50, 500]))
    np.testing.assert_allclose(per_row, [O.token_topk_bound(q[t:t + 1], k, b)[0] for t, b in zip(range(3), (5, 50, 500))],
                               rtol=0, atol=0)
    # the ragged last block contributes its valid tokens only
    assert O.kept_token_count([0, 5], 700) == 128 + 60


def test_block_size_consistency_64_vs_128():
    """The oracle is generic in the block size: a 128-token mask written as 64-token blocks
    (each kept 128-block -> its two halves) gives the same attention, and a 128-block mean is
    the mean of its two 64-block means (full blocks)."""
    d = 32
    q = _rand_bf16((256, d), 81).double().numpy()
    k = _rand_bf16((640, d), 82).double().numpy()
    v = _rand_bf16((640, d), 83).double().numpy()
    rows128 = np.array([[0, 2, 4], [1, 3, 4]])
    out128 = O.block_sparse_attention(q, k, v, rows128, [0, 1], block=128)
    rows64 = np.array([sorted({2 * j + h for j in r for h in (0, 1)}) for r in rows128])
    rows64 = np.repeat(rows64, 2, axis=0)                  # query blocks 2i, 2i+1 share row i
    out64 = O.block_sparse_attention(q, k, v, rows64, [0, 1, 2, 3], block=64)
    for i in range(2):
        np.testing.assert_allclose(np.vstack([out64[2 * i][0], out64[2 * i + 1][0]]), out128[i][0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(np.concatenate([out64[2 * i][1], out64[2 * i + 1][1]]), out128[i][1], rtol=0, atol=1e-13)
    p64, p128 = O.pool_blocks(k, 64), O.pool_blocks(k, 128)
    np.testing.assert_allclose((p64[0::2] + p64[1::2]) / 2, p128, rtol=0, atol=1e-15)
    assert O.forced_block_count(512, 8192, 1, 64) == 2 * O.forced_block_count(512, 8192, 1, 128) == 136


# ------------------------------------------------------------------ reference-context reuse

def _reuse_case(seed, n_text=128, n_ctx=512, n_cur=256, nq=384, d=16):
    rng = np.random.default_rng(seed)
    k = rng.normal(size=(n_text + n_ctx + n_cur, d))
    k += np.repeat(rng.normal(scale=0.5, size=(O.num_blocks(k.shape[0]), d)), 128, axis=0)[:k.shape[0]]
    return rng.normal(size=(nq, d)), rng.normal(size=(nq, d)), k


def test_reference_mass_matches_torch_softmax_ratio():
    q, _, k = _reuse_case(1)
    n_text, n_ctx = 128, 512
    kept = np.array([[1, 3], [2, 4], [1, 4]])
    got = O.reference_mass(q, k, kept, n_text, n_ctx, [0, 1, 2])
    logits = torch.from_numpy(q @ k.T / math.sqrt(q.shape[1]))
    p = torch.softmax(logits, dim=1).numpy()
    for i in range(3):
        rows = slice(128 * i, 128 * (i + 1))
        cols = np.concatenate([np.arange(128 * j, 128 * (j + 1)) for j in kept[i]])
        want = (p[rows][:, cols].sum(axis=1) / p[rows, n_text:n_text + n_ctx].sum(axis=1)).mean()
        assert got[i] == pytest.approx(want, rel=1e-12)


def test_reference_reuse_full_budget_and_identical_queries():
    q_now, q_prev, k = _reuse_case(2)
    fresh, reused, ef, er = O.reference_reuse_report(q_now, q_prev, k, 128, 512, 1.0, [0, 1, 2])
    assert np.allclose(ef, 1.0, atol=1e-14) and np.allclose(er, 1.0, atol=1e-14)   # every block kept
    fresh, reused, ef, er = O.reference_reuse_report(q_now, q_now, k, 128, 512, 0.5, [0, 1, 2])
    assert np.array_equal(fresh, reused) and np.array_equal(ef, er)


def test_reference_reuse_rows_follow_global_block_scores_and_grow_with_budget():
    q_now, q_prev, k = _reuse_case(3)
    fresh, reused, ef, er = O.reference_reuse_report(q_now, q_prev, k, 128, 512, 0.5, [0, 1, 2])
    # the reference blocks are global blocks 1..4 (text is one block): pooling the segment
    # alone must agree with the scores of the whole KV
    S = O.block_scores(O.pool_blocks(q_now), O.pool_blocks(k))[:, 1:5]
    want = np.sort(np.argsort(-S, axis=1, kind="stable")[:, :2], axis=1) + 1
    assert np.array_equal(fresh, want)
    assert fresh.min() >= 1 and fresh.max() <= 4 and reused.min() >= 1 and reused.max() <= 4
    _, _, ef_small, _ = O.reference_reuse_report(q_now, q_prev, k, 128, 512, 0.25, [0, 1, 2])
    assert np.all(ef >= ef_small)   # nested Top-K sets keep at least as much mass


# ------------------------------------------------------------------ mask reuse across scales

def _brute_block_map(grid_now, grid_prev, block):
    """The old block under each new block's middle token, found by scanning every old cell per
    axis with exact fractions (the old cell whose span [i/X, (i+1)/X) holds the new cell centre)."""
    from fractions import Fraction
    Tn, Hn, Wn = grid_now
    To, Ho, Wo = grid_prev
    n_now = Tn * Hn * Wn
    out = []
    for b in range(-(-n_now // block)):
        s, e = b * block, min((b + 1) * block, n_now)
        c = s + (e - s - 1) // 2
        t, h, w = c // (Hn * Wn), (c // Wn) % Hn, c % Wn
        cell = []
        for x, X_new, X_old in ((t, Tn, To), (h, Hn, Ho), (w, Wn, Wo)):
            centre = Fraction(2 * x + 1, 2 * X_new)
            hits = [i for i in range(X_old) if Fraction(i, X_old) <= centre < Fraction(i + 1, X_old)]
            assert len(hits) == 1
            cell.append(hits[0])
        out.append(((cell[0] * Ho + cell[1]) * Wo + cell[2]) // block)
    return np.array(out)


@pytest.mark.parametrize("grid_now,grid_prev,block", [
    ((8, 94, 96), (8, 64, 72), 128),     # the synthetic schedule's last two scales
    ((8, 64, 72), (8, 32, 32), 128),
    ((3, 7, 11), (5, 4, 9), 16),         # shrinking frames, odd sizes, ragged last blocks
    ((2, 9, 13), (2, 9, 13), 64),        # same grid
    ((1, 5, 7), (4, 6, 6), 8),
])
def test_raster_block_map_against_exact_cell_scan(grid_now, grid_prev, block):
    assert np.array_equal(O.raster_block_map(grid_now, grid_prev, block), _brute_block_map(grid_now, grid_prev, block))


def test_raster_block_map_closed_forms():
    # same grid: identity
    assert np.array_equal(O.raster_block_map((8, 64, 72), (8, 64, 72)), np.arange(288))
    # 2x in height and width with one old row per block: new block b (half a new row) lies in old row b // 4
    assert np.array_equal(O.raster_block_map((1, 8, 256), (1, 4, 128)), np.arange(16) // 4)
    # 2x in frames with one frame per block: new frame b lies in old frame b // 2
    assert np.array_equal(O.raster_block_map((4, 1, 128), (2, 1, 128)), np.arange(4) // 2)


def test_map_scores_gathers_rows_and_columns():
    grid_prev, grid_now, pre = (2, 8, 24), (2, 12, 32), 5          # 384 -> 768 tokens: 3 -> 6 blocks
    nb_prev = 3
    S_prev = 1000.0 * np.arange(nb_prev)[:, None] + np.arange(pre + nb_prev)[None, :]   # encodes (i, j)
    S_now = O.map_scores(S_prev, pre, grid_prev, grid_now)
    m = _brute_block_map(grid_now, grid_prev, 128)
    assert S_now.shape == (6, pre + 6)
    rows, cols = np.divmod(S_now, 1000.0)
    assert np.array_equal(rows, np.repeat(m[:, None], pre + 6, axis=1))
    assert np.array_equal(cols[:, :pre], np.tile(np.arange(pre), (6, 1)))            # prefix: same blocks
    assert np.array_equal(cols[:, pre:], np.tile(pre + m, (6, 1)))                    # current: mapped blocks


def test_reused_rows_keep_the_current_budget_and_equal_fresh_rows_on_the_same_grid():
    rng = np.random.default_rng(11)
    S_prev = rng.standard_normal((6, 4 + 6))
    same = O.reused_rows(S_prev, 4, (1, 6, 128), (1, 6, 128), 1, 3)
    assert np.array_equal(same, O.select_rows(S_prev, 1, 3))
    grown = O.reused_rows(S_prev, 4, (1, 6, 128), (1, 12, 128), 1, 5)
    assert grown.shape == (12, 6) and (np.diff(grown, axis=1) > 0).all() and (grown[:, 0] == 0).all()
    # rows of new blocks that map to the same old block are identical
    m = O.raster_block_map((1, 12, 128), (1, 6, 128))
    for a in range(12):
        for b in range(12):
            if m[a] == m[b]:
                assert np.array_equal(grown[a], grown[b])
