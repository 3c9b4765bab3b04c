"""The GPU path is bitwise reproducible: the same inputs give the same block lists, outputs and
LSEs on every call, at both block sizes.

No kernel on the path accumulates through atomics or reorders a sum by timing: pooling
reduces in a fixed order, the score and attention kernels accumulate in the tensor cores in
the order of the kept list, and the Top-K resolves ties by index. Two calls on the same
seeded inputs must therefore agree bit for bit, including when the second call reuses the
first call's output buffers.
"""
import pytest
import torch

from block_sparse_attention_tok_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S(cuda_lib):
    from block_sparse_attention_tok_b200 import sparstar
    return sparstar


@pytest.mark.parametrize("block", [128, 64])
@pytest.mark.parametrize("d", [64, 128])
def test_forward_is_bitwise_reproducible(S, block, d):
    n_text, n_ctx, n_cur, heads = 256, 3000, 4100, 3
    q, k, v = synth.make_qkv(n_cur, n_text + n_ctx + n_cur, heads, d, [61 + d, 62 + d, 63 + d], device="cuda")
    first = S.forward(q, k, v, n_text, n_ctx, n_cur, 2, 0.15, block=block)
    assert S.device_status() == S.OK
    first = [t.clone() for t in first]
    for _ in range(2):
        again = S.forward(q, k, v, n_text, n_ctx, n_cur, 2, 0.15, block=block)
        assert S.device_status() == S.OK
        for a, b in zip(first, again):
            assert torch.equal(a, b)


def test_attention_is_bitwise_reproducible_into_the_same_buffers(S):
    n_text, n_ctx, n_cur = 512, 4096, 5000
    q, k, v = synth.make_qkv(n_cur, n_text + n_ctx + n_cur, 4, 128, [71, 72, 73, 74], device="cuda")
    idx, cnt, _ = S.select(q, k, n_text, n_ctx, n_cur, 2, 0.1)
    o, lse = S.attn(q, k, v, idx, cnt)
    o_ref, lse_ref = o.clone(), lse.clone()
    o.fill_(0)
    lse.fill_(0)
    S.attn(q, k, v, idx, cnt, o=o, lse=lse)
    assert S.device_status() == S.OK
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_attention_without_lse_gives_the_same_output(S):
    """With no LSE buffer (a null pointer through the C ABI) the kernel skips that store only."""
    n_text, n_ctx, n_cur = 128, 2048, 3000
    q, k, v = synth.make_qkv(n_cur, n_text + n_ctx + n_cur, 2, 128, [81, 82], device="cuda")
    idx, cnt, _ = S.select(q, k, n_text, n_ctx, n_cur, 2, 0.2)
    o_with, lse = S.attn(q, k, v, idx, cnt)
    o_without, none = S.attn(q, k, v, idx, cnt, want_lse=False)
    assert S.device_status() == S.OK
    assert none is None and lse is not None
    assert torch.equal(o_with, o_without)
