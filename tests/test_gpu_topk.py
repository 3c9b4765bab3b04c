"""Clip-aware retention + joint Top-K on given scores (sparstar_topk) against the oracle's
select_rows, bit for bit.

The scores are fp32 on both sides (the oracle widens them to fp64, which is exact), so the
ranking has one right answer and no tolerance applies. Rows are built to reach every branch
of the kernels: ordinary rows; heavy ties (small integers), so that equal scores straddle
the K-th place; constant rows; signed zeros; NaN, sparse and dominant (K beyond the count of
numbers); infinities; an outlier that squeezes every other score into one value bin; a
denormal-width range; a range wider than the largest float. Sizes cover every keys-per-lane
instance of the warp kernel, the 3,965-candidate boundary to the CTA-per-row kernel, and
the rows that never read scores (K_topk = 0 or every candidate kept).
"""
import numpy as np
import pytest
import torch

from oracle import sparstar_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S(cuda_lib):
    from block_sparse_attention_tok_b200 import sparstar
    return sparstar


KINDS = ["normal", "ints", "const", "zeros", "nan10", "nan90", "inf", "outlier", "cluster", "denorm", "huge"]


def _scores(kind, rng, rows, nkb):
    shape = (rows, nkb)
    if kind == "normal":
        s = rng.normal(size=shape)
    elif kind == "ints":
        s = rng.integers(-4, 5, size=shape).astype(np.float64)
    elif kind == "const":
        s = np.full(shape, 0.25)
    elif kind == "zeros":
        s = rng.choice(np.array([0.0, -0.0, 0.0, -0.0, 1.0, -1.0]), size=shape)
    elif kind == "nan10":
        s = rng.normal(size=shape)
        s[rng.random(shape) < 0.1] = np.nan
    elif kind == "nan90":
        s = rng.normal(size=shape)
        s[rng.random(shape) < 0.9] = np.nan
    elif kind == "inf":
        s = rng.normal(size=shape)
        u = rng.random(shape)
        s[u < 0.05] = np.inf
        s[(u >= 0.05) & (u < 0.1)] = -np.inf
    elif kind == "outlier":
        s = 1e-3 * rng.normal(size=shape)
        s[:, rng.integers(0, nkb)] = 1e6
    elif kind == "cluster":
        # most scores inside one narrow cluster at the top, distinct values
        s = rng.normal(size=shape)
        s[rng.random(shape) < 0.6] = 5.0 + 1e-5 * rng.random()
        s += 1e-6 * rng.random(shape)
    elif kind == "denorm":
        s = rng.integers(-20, 20, size=shape).astype(np.float64) * 1e-44
    elif kind == "huge":
        s = rng.uniform(-3.0e38, 3.0e38, size=shape)
    else:
        raise ValueError(kind)
    return s.astype(np.float32)


def _check(S_lib, s32, n_forced, k_topk, kmax=None):
    rows, nkb = s32.shape
    k_total = n_forced + k_topk
    kmax = k_total if kmax is None else kmax
    scores = torch.from_numpy(s32).cuda()
    idx = torch.full((rows, max(kmax, 1)), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    S_lib.topk(scores, n_forced, k_topk, idx=idx, cnt=cnt)
    torch.cuda.synchronize()
    assert S_lib.device_status() == S_lib.OK
    want = O.select_rows(s32.astype(np.float64), n_forced, k_topk)
    got = idx.cpu().numpy()
    assert (cnt.cpu().numpy() == k_total).all()
    bad = np.nonzero((got[:, :k_total] != want).any(axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first row {bad[0]}: got {got[bad[0], :k_total].tolist()}"
    assert (got[:, k_total:kmax] == -7).all()


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("n_cand", [2, 33, 256, 257, 700, 1128, 1153, 1600, 2045, 2046, 2256, 3100, 3965, 3966, 5000])
def test_topk_matches_oracle(S, kind, n_cand):
    rng = np.random.default_rng(100003 * KINDS.index(kind) + n_cand)
    n_forced = int(rng.integers(0, 6))
    rows = 12
    s = _scores(kind, rng, rows, n_forced + n_cand)
    for k_topk in sorted({1, max(1, n_cand // 11), n_cand // 2, n_cand - 1}):
        if 1 <= k_topk < n_cand:
            _check(S, s, n_forced, k_topk)


@pytest.mark.parametrize("kpl_edge", [253, 509, 765, 1149, 1533, 2045, 2429, 3965])
def test_topk_keys_per_lane_edges(S, kpl_edge):
    """The largest row of each warp kernel instance (32 * keys per lane, less 3 slots for the
    row's 16-byte alignment offset), and one candidate more."""
    rng = np.random.default_rng(kpl_edge)
    for n_cand in (kpl_edge, kpl_edge + 1):
        s = _scores("ints", rng, 9, 3 + n_cand)
        _check(S, s, 3, max(1, n_cand // 10))
        s = _scores("normal", rng, 9, 3 + n_cand)
        _check(S, s, 3, n_cand - 1)


def test_topk_forced_columns_are_not_read(S):
    rng = np.random.default_rng(5)
    s = _scores("normal", rng, 20, 300)
    s[:, :7] = np.nan                          # forced columns: never ranked
    _check(S, s, 7, 40)
    s[:, :7] = np.inf
    _check(S, s, 7, 40)


def test_topk_rows_that_read_no_scores(S):
    rng = np.random.default_rng(6)
    s = _scores("normal", rng, 5, 50)
    _check(S, s, 4, 0)                         # forced prefix only
    _check(S, s, 4, 46)                        # every candidate kept
    _check(S, s, 0, 50)
    _check(S, s, 50, 0)


def test_topk_wider_index_buffer_and_many_rows(S):
    rng = np.random.default_rng(8)
    s = _scores("nan10", rng, 3001, 4 + 1128)  # a row count that leaves a partial CTA
    _check(S, s, 4, 103, kmax=120)


def test_topk_nan_versus_negative_infinity(S):
    s = np.array([[np.nan, -np.inf, np.nan, -np.inf, 1.0] * 60], dtype=np.float32)
    for k in (1, 60, 61, 120, 150, 299):
        _check(S, s, 0, k)


def test_topk_random_sweep(S):
    """60 seeded launches: random candidate counts (2 to 6,000, so every keys-per-lane instance
    and the CTA-per-row kernel), forced prefixes of 0 to 40 columns, K anywhere in [1, n_cand),
    and rows of different kinds mixed in one launch."""
    rng = np.random.default_rng(977)
    for _ in range(60):
        n_cand = int(rng.integers(2, 6001))
        n_forced = int(rng.integers(0, 41))
        k_topk = int(rng.integers(1, n_cand))
        rows = int(rng.integers(1, 40))
        kinds = rng.choice(KINDS, size=rows)
        s = np.concatenate([_scores(str(kd), rng, 1, n_forced + n_cand) for kd in kinds])
        _check(S, s, n_forced, k_topk, kmax=n_forced + k_topk + int(rng.integers(0, 3)))
