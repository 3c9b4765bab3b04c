"""Mask reuse analyses: across clips (reference context) and across scales (recompute
frequency).

Across clips: retained attention mass over the reference context, for a fresh selection
against the preceding clip's pattern under one reference budget.

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


# Recompute policies of the cross-scale comparison (digest, 关键结果与论文证据, bullet 重算频率,
# Figure 5): which scales of a clip's sparsified schedule compute fresh block scores.
POLICIES = {
    "per_scale": lambda s: True,            # recompute at every scale
    "every_2": lambda s: s % 2 == 0,        # recompute at scales 1, 3, ...; reuse at 2, 4, ...
    "one_shot": lambda s: s == 0,           # compute once at the first scale, transfer to the rest
}


def cross_scale_masks(scales, policy: str, budget_mode: int = S.BUDGET_LITERAL, workspaces=None):
    """Kept blocks at every scale of one clip's schedule under a recompute policy.

    `scales` lists, in schedule order, dicts with q, k (bf16 [H, N, d] CUDA), seg (n_text, n_ctx,
    n_cur), grid (frames, height, width) of the current tokens, clip and density. A scale whose
    policy says "recompute" runs the whole selection with its scores kept
    (sparstar_select_ex); any other scale takes the scores of the latest recomputed scale
    through the nearest-position block map (sparstar_map_scores) and fills its own budget by
    the clip-aware joint Top-K (sparstar_topk), so every scale keeps the same number of blocks
    under every policy. Returns a list of (idx, cnt)."""
    recompute = POLICIES[policy]
    out, last = [], None
    for si, sc in enumerate(scales):
        seg = tuple(sc["seg"])
        plan = S.make_plan(seg[2], *seg, sc["clip"], sc["density"], budget_mode)
        ws = None if workspaces is None else workspaces[si]
        if recompute(si) or last is None:
            idx, cnt, scores = S.select(sc["q"], sc["k"], *seg, sc["clip"], sc["density"], budget_mode,
                                        want_scores=True, workspace=ws)
            last = (scores, seg, tuple(sc["grid"]))
        else:
            mapped = S.map_scores(last[0], last[1], last[2], seg, tuple(sc["grid"]))
            idx, cnt = S.topk(mapped, int(plan.n_forced), int(plan.k_topk))
            del mapped
        out.append((idx, cnt))
    return out


def retained_mass_of(q, k, v, idx, cnt):
    """Per query block, the mean dense softmax mass the kept blocks hold (sparstar_attn with the
    mask and with every block, then sparstar_retained_mass). Returns fp32 [H, nqb]."""
    H, n_q, _ = q.shape
    nqb, nkb = -(-n_q // BLOCK), -(-k.shape[1] // BLOCK)
    o = torch.empty_like(q)
    _, lse_kept = S.attn(q, k, v, idx, cnt, o=o)
    all_idx = torch.arange(nkb, dtype=torch.int32, device=q.device).expand(H, nqb, nkb).contiguous()
    all_cnt = torch.full((H, nqb), nkb, dtype=torch.int32, device=q.device)
    _, lse_dense = S.attn(q, k, v, all_idx, all_cnt, o=o)
    _, e = S.retained_mass(lse_kept, lse_dense, want_tokens=False)
    return e
