"""Retained attention mass over the reference context, for a fresh selection against the
preceding clip's pattern under one reference budget.

This is the cross-clip analysis of the SparSTAR digest ("SparSTAR的贡献：每尺度动态重建",
pchao.org), section 关键结果与论文证据, bullet 跨clip边界 (Figure 4). The reference context
of the current clip is the preceding clip's final scale, so its key blocks are the very
tokens that clip's final scale selected among. Per query block the budget is
ceil(budget_frac * n_ref) of the n_ref reference blocks:
  fresh:  the best of them by the current queries' block scores;
  reused: the best by the preceding clip's queries of the same query block (same position).
The measure is, per query block, the mean over its rows of the softmax mass on the kept
reference tokens divided by the mass on all reference tokens.

Every computation runs in the library's kernels: the block scores (sparstar_select_ex), the
Top-K over the reference columns (sparstar_topk, with the text blocks as the forced prefix,
so the chosen ids are global), the attention log-sum-exps over the kept and over all
reference blocks (sparstar_attn_ex) and their ratio (sparstar_retained_mass). This module
only slices columns and rows between those calls.
"""
from __future__ import annotations

import math

import torch

from . import sparstar as S

BLOCK = S.BLOCK


def reference_reuse(q_now: torch.Tensor, q_prev: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    n_text: int, n_ctx: int, n_cur: int, budget_frac: float, workspace=None) -> dict:
    """q_now, q_prev [H, Nq, d]; k, v [H, Nkv, d] with Nkv = n_text + n_ctx + n_cur (bf16, CUDA).
    n_text and n_ctx must be whole 128-token blocks. Returns the fresh and reused kept
    reference blocks ([H, nqb, K] int32, global block ids) and the per-query-block retained
    reference mass of each ([H, nqb] fp32)."""
    if n_text % BLOCK or n_ctx % BLOCK or n_ctx == 0:
        raise ValueError("text and reference segments must be whole, non-empty 128-token blocks")
    if q_prev.shape != q_now.shape:
        raise ValueError("the preceding clip's queries must have the current queries' shape")
    nb_text, n_ref = n_text // BLOCK, n_ctx // BLOCK
    k_ref = int(math.ceil(budget_frac * n_ref - 1e-9))
    if not 1 <= k_ref <= n_ref:
        raise ValueError("the budget must keep between 1 and all reference blocks")
    H, n_q, _ = q_now.shape
    nqb = -(-n_q // BLOCK)
    width = nb_text + n_ref

    def choose(q):
        # density 1: every row keeps every block, so only the scores are computed
        _, _, sc = S.select(q, k, n_text, n_ctx, n_cur, 2, 1.0, want_scores=True, workspace=workspace)
        head = sc[:, :, :width].contiguous()      # text (forced prefix) + reference columns
        idx, _ = S.topk(head, nb_text, k_ref)
        return idx[:, :, nb_text:].contiguous()   # the chosen reference blocks

    fresh, reused = choose(q_now), choose(q_prev)
    cnt = torch.full((H, nqb), k_ref, dtype=torch.int32, device=q_now.device)
    all_ref = torch.arange(nb_text, width, dtype=torch.int32, device=q_now.device).expand(H, nqb, n_ref).contiguous()
    cnt_all = torch.full((H, nqb), n_ref, dtype=torch.int32, device=q_now.device)
    o = torch.empty_like(q_now)
    _, lse_ref = S.attn(q_now, k, v, all_ref, cnt_all, o=o)
    _, lse_fresh = S.attn(q_now, k, v, fresh, cnt, o=o)
    _, lse_reused = S.attn(q_now, k, v, reused, cnt, o=o)
    _, e_fresh = S.retained_mass(lse_fresh, lse_ref, want_tokens=False)
    _, e_reused = S.retained_mass(lse_reused, lse_ref, want_tokens=False)
    return {"fresh": fresh, "reused": reused, "e_fresh": e_fresh, "e_reused": e_reused, "k_ref": k_ref}
