"""sparstar_select_noalloc: block selection for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (a host framework that owns every device byte through
its own pool, a plugin that must not allocate, code running under a memory cap). For them
the library keeps the selection's scratch in a fixed device array of its own. These tests
call that entry point through the C ABI and compare its block lists with those of the
regular sparstar_select (which takes a caller workspace): they must be identical, on two
calls in a row with different inputs, since the array keeps the previous call's contents.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_tok_b200 import sparstar, synth


def _lib():
    return sparstar.load()


def test_oversized_request_is_rejected_before_touching_the_device():
    lib = _lib()
    # 720p-like shape with 256 heads: its scratch (about 875 MB) exceeds the fixed array.
    need = sparstar.workspace_size(256, 72192, 512, 72192, 72192, 128)
    assert need > sparstar.NOALLOC_SCRATCH_BYTES
    rc = lib.sparstar_select_noalloc(0x1000, 0x2000, 256, 72192, sparstar.Segments(512, 72192, 72192), 128, 2,
                                     0.09375, 0, 0x3000, 0x4000, 107, None)
    assert rc == sparstar.ERR_UNSUPPORTED
    rc = lib.sparstar_select_noalloc(0x1000, 0x2000, 2, 1024, sparstar.Segments(256, 768, 1024), 96, 2, 0.25, 0,
                                     0x3000, 0x4000, 4, None)
    assert rc == sparstar.ERR_UNSUPPORTED


@pytest.mark.gpu
def test_rows_without_scores_need_no_scratch():
    """Forced-only rows (the Clip-1 720p scale read literally: K_topk = 0) do not depend on the
    scores, so they take no scratch: a head count whose scratch would exceed the fixed array is
    accepted and gives the regular selection's rows (q and k are not read for such rows)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _lib()
    H, n_q, segs, d = 256, 72000, (512, 8192, 72000), 128
    plan = sparstar.make_plan(n_q, *segs, 1, 0.09375, 0)
    assert int(plan.k_topk) == 0
    assert sparstar.workspace_size(H, n_q, *segs, d) > sparstar.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(64, dtype=torch.bfloat16, device="cuda")    # never read for these rows
    idx = torch.full((H, int(plan.nqb), int(plan.k_total)), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((H, int(plan.nqb)), -1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream or None
    rc = lib.sparstar_select_noalloc(dummy.data_ptr(), dummy.data_ptr(), H, n_q, sparstar.Segments(*segs), d, 1,
                                     0.09375, 0, idx.data_ptr(), cnt.data_ptr(), idx.shape[-1], stream)
    assert rc == sparstar.OK
    assert sparstar.device_status() == sparstar.OK
    want = torch.arange(int(plan.k_total), dtype=torch.int32, device="cuda").expand_as(idx)
    assert torch.equal(idx, want) and bool((cnt == int(plan.k_total)).all())


def _call_noalloc(lib, q, k, segs, clip, density, mode, idx, cnt):
    H, n_q, d = q.shape
    stream = torch.cuda.current_stream().cuda_stream or None
    return lib.sparstar_select_noalloc(q.data_ptr(), k.data_ptr(), H, n_q, sparstar.Segments(*segs), d, clip,
                                       float(density), mode, idx.data_ptr(), cnt.data_ptr(), idx.shape[-1], stream)


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [
    # (n_q, (text, ctx, cur), H, d, clip, density, mode)
    (1024, (256, 768, 1024), 2, 64, 2, 0.25, 0),
    (18432, (512, 4096, 18432), 32, 128, 1, 0.1875, 1),
    (72192, (512, 72192, 72192), 32, 128, 2, 0.09375, 0),
])
def test_noalloc_matches_workspace_select_twice(shape):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    n_q, segs, H, d, clip, density, mode = shape
    lib = _lib()
    n_kv = sum(segs)
    plan = sparstar.make_plan(n_q, *segs, clip, density, mode)
    assert sparstar.workspace_size(H, n_q, *segs, d) <= sparstar.NOALLOC_SCRATCH_BYTES
    for call in range(2):
        q, k, _ = synth.make_qkv(n_q, n_kv, H, d, [500 * call + 7 * h for h in range(H)], device="cuda")
        ref_idx, ref_cnt, _ = sparstar.select(q, k, *segs, clip, density, mode)
        idx = torch.full((H, int(plan.nqb), int(plan.k_total)), -1, dtype=torch.int32, device="cuda")
        cnt = torch.full((H, int(plan.nqb)), -1, dtype=torch.int32, device="cuda")
        assert _call_noalloc(lib, q, k, segs, clip, density, mode, idx, cnt) == sparstar.OK
        assert sparstar.device_status() == sparstar.OK
        assert torch.equal(idx, ref_idx), f"call {call}: block lists differ"
        assert torch.equal(cnt, ref_cnt), f"call {call}: counts differ"
        del q, k
    torch.cuda.empty_cache()
