"""C-ABI library checks that need no GPU: it loads, exports every symbol the header
declares, computes plans and workspace sizes, and rejects bad arguments before touching
the device (no compute calls are made here)."""
import ctypes
import os
import re

import numpy as np
import pytest

from block_sparse_attention_tok_b200 import sparstar, synth, _build
from oracle import sparstar_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sparstar.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_build.LIB_PATH):
        _build.build()
    return sparstar.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sparstar_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 8
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(sparstar.exported_symbols()) == names


def test_abi_version_and_strerror(lib):
    assert lib.sparstar_abi_version() == 2
    for code in range(7):
        assert sparstar.strerror(code)
    assert sparstar.strerror(99) == "unknown status"


@pytest.mark.parametrize("n_q,n_text,n_ctx,n_cur,clip,density", [
    (1024, 256, 768, 1024, 2, 0.25), (18432, 512, 4096, 18432, 1, 0.1875),
    (72000, 512, 8192, 72000, 1, 0.09375), (72192, 512, 72192, 72192, 2, 0.09375),
    (8192, 512, 8192, 8192, 1, 0.625), (5, 200, 300, 1, 1, 0.5), (300, 0, 0, 129, 2, 1.0),
    (128, 1000, 0, 5, 2, 0.01), (0, 10, 10, 10, 1, 0.3),
])
@pytest.mark.parametrize("mode", [0, 1])
def test_plan_matches_oracle_budget(lib, n_q, n_text, n_ctx, n_cur, clip, density, mode):
    plan = sparstar.make_plan(n_q, n_text, n_ctx, n_cur, clip, density, mode)
    nkb = O.num_blocks(n_text + n_ctx + n_cur)
    n_forced = min(O.forced_block_count(n_text, n_ctx, clip), nkb)
    assert plan.nqb == O.num_blocks(n_q) and plan.nkb == nkb
    assert plan.n_forced == n_forced and plan.n_cand == nkb - n_forced
    assert (plan.k_total, plan.k_topk) == O.row_budget(nkb, n_forced, density, mode)


def test_plan_matches_oracle_budget_on_random_shapes(lib):
    """3,000 seeded shapes: segment lengths from 0 to 10^5 tokens (ragged and block-aligned),
    both clip modes, densities drawn from the pages' values, dyadic fractions and arbitrary
    reals in (0, 1], both budget readings and both block sizes; every plan field equals the
    oracle's (integers, so exactly)."""
    rng = np.random.default_rng(20261202)
    pages = [0.625, 0.1875, 0.09375, 1.0, 0.25, 0.5]
    for _ in range(3000):
        block = int(rng.choice([128, 64]))
        lens = []
        for _k in range(3):
            r = rng.random()
            if r < 0.2:
                lens.append(0)
            elif r < 0.5:
                lens.append(int(rng.integers(1, 400)) * block)
            else:
                lens.append(int(rng.integers(1, 100000)))
        n_text, n_ctx, n_cur = lens
        if n_text + n_ctx + n_cur == 0:
            n_cur = 1
        n_q = int(rng.integers(0, 100000))
        clip = int(rng.choice([1, 2, 3]))
        r = rng.random()
        density = (float(rng.choice(pages)) if r < 0.4 else
                   int(rng.integers(1, 1025)) / 1024.0 if r < 0.7 else float(1.0 - rng.random()))
        mode = int(rng.integers(0, 2))
        plan = sparstar.make_plan(n_q, n_text, n_ctx, n_cur, clip, density, mode, block=block)
        nkb = O.num_blocks(n_text + n_ctx + n_cur, block)
        n_forced = min(O.forced_block_count(n_text, n_ctx, clip, block), nkb)
        case = (n_q, n_text, n_ctx, n_cur, clip, density, mode, block)
        assert plan.nqb == O.num_blocks(n_q, block) and plan.nkb == nkb, case
        assert plan.n_forced == n_forced and plan.n_cand == nkb - n_forced, case
        assert (plan.k_total, plan.k_topk) == O.row_budget(nkb, n_forced, density, mode), case


def test_workspace_size(lib):
    # pooled q and k as bf16 hi/lo pairs (2 x H*n_blocks*d x 2 B each) and fp32 scores
    # (H*nqb*nkb), each section 256-byte aligned
    got = sparstar.workspace_size(32, 72192, 512, 72192, 72192, 128)
    def al(x):
        return (x + 255) // 256 * 256
    assert got == 2 * al(32 * 564 * 128 * 2) + 2 * al(32 * 1132 * 128 * 2) + al(32 * 564 * 1132 * 4)


@pytest.mark.parametrize("kwargs,code", [
    (dict(density=0.0), sparstar.ERR_ARG), (dict(density=1.5), sparstar.ERR_ARG),
    (dict(density=float("nan")), sparstar.ERR_ARG), (dict(clip=0), sparstar.ERR_ARG),
    (dict(mode=7), sparstar.ERR_ARG), (dict(n_text=-1), sparstar.ERR_ARG),
    (dict(d=96), sparstar.ERR_UNSUPPORTED), (dict(heads=0), sparstar.ERR_ARG),
    (dict(kmax=1), sparstar.ERR_ARG), (dict(q=0x1008), sparstar.ERR_ARG),
    (dict(q=None), sparstar.ERR_ARG), (dict(ws=None), sparstar.ERR_WORKSPACE),
    (dict(ws_bytes=10), sparstar.ERR_WORKSPACE), (dict(ws=0x2010), sparstar.ERR_WORKSPACE),
])
def test_select_rejects_bad_arguments_before_launch(lib, kwargs, code):
    a = dict(q=0x1000, k=0x2000, heads=2, n_q=1024, n_text=256, n_ctx=768, n_cur=1024, d=64, clip=2,
             density=0.25, mode=0, idx=0x3000, cnt=0x4000, kmax=8, scores=None, ws=0x10000,
             ws_bytes=1 << 30)
    a.update(kwargs)
    rc = lib.sparstar_select(a["q"], a["k"], a["heads"], a["n_q"],
                             sparstar.Segments(a["n_text"], a["n_ctx"], a["n_cur"]), a["d"], a["clip"],
                             a["density"], a["mode"], a["idx"], a["cnt"], a["kmax"], a["scores"], a["ws"],
                             a["ws_bytes"], None)
    assert rc == code


def test_select_zero_queries_is_a_noop(lib):
    rc = lib.sparstar_select(None, None, 2, 0, sparstar.Segments(256, 768, 1024), 64, 2, 0.25, 0, None, None, 4,
                             None, None, 0, None)
    assert rc == sparstar.OK


@pytest.mark.parametrize("kwargs,code", [
    (dict(d=80), sparstar.ERR_UNSUPPORTED), (dict(n_kv=0), sparstar.ERR_ARG), (dict(heads=0), sparstar.ERR_ARG),
    (dict(v=None), sparstar.ERR_ARG), (dict(o=0x5004), sparstar.ERR_ARG), (dict(lse=0x6002), sparstar.ERR_ARG),
    (dict(kmax=0), sparstar.ERR_ARG), (dict(scale=float("inf")), sparstar.ERR_ARG),
])
def test_attn_rejects_bad_arguments_before_launch(lib, kwargs, code):
    a = dict(q=0x1000, k=0x2000, v=0x3000, heads=2, n_q=1024, n_kv=2048, d=64, idx=0x4000, cnt=0x4800, kmax=4,
             scale=0.0, o=0x5000, lse=None)
    a.update(kwargs)
    rc = lib.sparstar_attn(a["q"], a["k"], a["v"], a["heads"], a["n_q"], a["n_kv"], a["d"], a["idx"], a["cnt"],
                           a["kmax"], a["scale"], a["o"], a["lse"], None)
    assert rc == code
    assert lib.sparstar_attn(None, None, None, 1, 0, 10, 64, None, None, 1, 0.0, None, None, None) == sparstar.OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(sparstar, "_LIB", None)
    monkeypatch.setattr(_build, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        sparstar.load()


def test_block_size_plans_match_oracle_and_reject_other_sizes(lib):
    from block_sparse_attention_tok_b200 import sparstar as S
    for sc in (synth.TINY_CLIP2, synth.MID_CLIP1, synth.FINAL_CLIP1_RAGGED, synth.FINAL_CLIP2):
        for mode in (0, 1):
            p = S.make_plan(sc.n_q, sc.n_text, sc.n_ctx, sc.n_cur, sc.clip, sc.density, mode, block=64)
            nkb = O.num_blocks(sc.n_kv, 64)
            nf = min(O.forced_block_count(sc.n_text, sc.n_ctx, sc.clip, 64), nkb)
            kt, kk = O.row_budget(nkb, nf, sc.density, mode)
            assert (int(p.nqb), int(p.nkb), int(p.n_forced), int(p.k_total), int(p.k_topk)) == \
                (O.num_blocks(sc.n_q, 64), nkb, nf, kt, kk)
    with pytest.raises(S.SparstarError) as e:
        S.make_plan(1024, 256, 768, 1024, 2, 0.25, 0, block=96)
    assert e.value.code == S.ERR_UNSUPPORTED


def test_select_rejects_more_candidates_than_supported_before_launch(lib):
    """n_cand = 16,385 is one past the radix Top-K's shared-memory limit: refused before any
    device call (fake device addresses are never touched)."""
    n_kv = 128 * (1 + 16385)
    rc = lib.sparstar_select(0x1000, 0x2000, 1, 256, sparstar.Segments(128, 0, n_kv - 128), 64, 2, 0.05, 0,
                             0x3000, 0x4000, 1 << 20, None, 0x10000, 1 << 40, None)
    assert rc == sparstar.ERR_UNSUPPORTED
    rc = lib.sparstar_select_ex(0x1000, 0x2000, 1, 256, sparstar.Segments(128, 0, n_kv - 128), 64, 2, 0.05, 0, 96,
                                0x3000, 0x4000, 1 << 20, None, 0x10000, 1 << 40, None)
    assert rc == sparstar.ERR_UNSUPPORTED   # block size 96


@pytest.mark.parametrize("args,code", [
    # (rows, nkb, n_forced, k_topk, kmax)
    ((-1, 10, 2, 3, 8), sparstar.ERR_ARG),          # negative rows
    ((4, 0, 0, 0, 8), sparstar.ERR_ARG),            # no columns
    ((4, 10, 11, 0, 16), sparstar.ERR_ARG),         # more forced blocks than columns
    ((4, 10, -1, 3, 8), sparstar.ERR_ARG),
    ((4, 10, 2, 9, 16), sparstar.ERR_ARG),          # k_topk > n_cand
    ((4, 10, 2, -1, 16), sparstar.ERR_ARG),
    ((4, 10, 2, 3, 4), sparstar.ERR_ARG),           # kmax < n_forced + k_topk
    ((4, 1 + 16385, 1, 5, 8), sparstar.ERR_UNSUPPORTED),   # 16,385 candidates, scores read
    ((1 << 31, 10, 2, 3, 8), sparstar.ERR_UNSUPPORTED),    # rows beyond a grid dimension
])
def test_topk_rejects_bad_arguments_before_launch(lib, args, code):
    rows, nkb, n_forced, k_topk, kmax = args
    assert lib.sparstar_topk(0x1000, rows, nkb, n_forced, k_topk, 0x2000, 0x3000, kmax, None) == code


def test_topk_null_and_misaligned_pointers(lib):
    assert lib.sparstar_topk(None, 4, 10, 2, 3, 0x2000, 0x3000, 8, None) == sparstar.ERR_ARG      # scores read
    assert lib.sparstar_topk(0x1002, 4, 10, 2, 3, 0x2000, 0x3000, 8, None) == sparstar.ERR_ARG    # not 4-byte aligned
    assert lib.sparstar_topk(0x1000, 4, 10, 2, 3, None, 0x3000, 8, None) == sparstar.ERR_ARG
    assert lib.sparstar_topk(0x1000, 0, 10, 2, 3, None, None, 8, None) == sparstar.OK             # rows == 0: no-op


def test_read_probe_rejects_bad_arguments_before_launch(lib):
    assert lib.sparstar_read_probe(None, 64, 0x2000, None) == sparstar.ERR_ARG         # no source
    assert lib.sparstar_read_probe(0x1008, 64, 0x2000, None) == sparstar.ERR_ARG       # not 16-byte aligned
    assert lib.sparstar_read_probe(0x1000, 40, 0x2000, None) == sparstar.ERR_ARG       # not a multiple of 16
    assert lib.sparstar_read_probe(0x1000, 64, None, None) == sparstar.ERR_ARG         # no sink
    assert lib.sparstar_read_probe(0x1000, 0, None, None) == sparstar.OK               # empty: no-op


def test_map_scores_rejects_bad_arguments_before_launch(lib):
    seg = sparstar.Segments
    grid = sparstar.Grid
    ok_args = (0x1000, 2, seg(256, 512, 384), grid(2, 8, 24), seg(256, 512, 768), grid(2, 12, 32), 0x2000, None)

    def call(**over):
        names = ["sp", "H", "seg_p", "grid_p", "seg_n", "grid_n", "sn", "st"]
        a = dict(zip(names, ok_args))
        a.update(over)
        return lib.sparstar_map_scores(*(a[n] for n in names))

    assert call(H=0) == sparstar.ERR_ARG
    assert call(grid_p=grid(2, 8, 25)) == sparstar.ERR_ARG                        # product != n_cur
    assert call(grid_n=grid(0, 12, 32)) == sparstar.ERR_ARG                        # empty axis
    assert call(seg_n=seg(128, 512, 768)) == sparstar.ERR_ARG                      # text differs across scales
    assert call(seg_p=seg(200, 512, 384), seg_n=seg(200, 512, 768)) == sparstar.ERR_ARG   # prefix not whole blocks
    assert call(sp=None) == sparstar.ERR_ARG
    assert call(sn=0x2002) == sparstar.ERR_ARG                                    # not 4-byte aligned
    big = 49152 * 128
    assert call(seg_n=seg(256, 512, big), grid_n=grid(1, 128, 49152)) == sparstar.ERR_UNSUPPORTED


def test_token_bound_rejects_too_many_kv_blocks_before_launch(lib):
    ws = ctypes.c_size_t()
    assert lib.sparstar_token_bound_workspace_size(1, 128, ctypes.byref(ws)) == sparstar.OK
    n_kv = 128 * 4096                     # 4,096 KV blocks: one more than the 16-bit counts allow
    rc = lib.sparstar_token_bound(0x1000, 0x2000, 1, 128, n_kv, 128, 0x3000, 0x4000, 4, 0x5000, 0.0, None,
                                  0x6000, 0x7000, ws.value, None)
    assert rc == sparstar.ERR_UNSUPPORTED
