"""CPU oracle for SparSTAR's per-scale dynamic block-sparse attention (fp64, numpy).

TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the benchmark's CPU
baseline may import this module. The CUDA library never calls it, and it imports nothing
from the CUDA side: it takes plain arrays (bf16 bit patterns as uint16) and works in fp64.

What it computes, per head, for one expensive scale. Source: the SparSTAR digest
"SparSTAR的贡献：每尺度动态重建" (pchao.org), section 方法概览 ("method overview"), and the
English abstract "SparSTAR: Sparse Attention for SpaceTime AutoRegressive Video Synthesis"
(newx.sg), section Abstract:
  1. split Q and the mixed KV context (text ‖ reference context ‖ current tokens) into
     128-token blocks                                    (方法概览, bullet 块划分与聚合评分);
  2. mean-pool each block (the same bullet: a block is represented by the average of its
     token vectors);
  3. score every (query block, key block) pair from the pooled vectors (same bullet);
  4. keep the clip-aware conditioning blocks dense: text always, and in Clip 1 also the
     image-pyramid blocks                                 (bullet clip感知保留策略);
  5. fill each query-block row with a joint Top-K over the remaining key blocks
     (方法概览, first paragraph: one Top-K over all blocks not kept by rule), separately for
     every head
     (bullet per-head动态掩码);
  6. run forward-only attention over the kept blocks only (bullet FastFlex执行路径).
The pages print no formulas, code or worked example for SparSTAR. Readings of the open
points (all also listed in the design notes):
  - score: S_ij = mean(q_i) . mean(k_j) / sqrt(d);
  - budget: each row holds max(ceil(density * n_kv_blocks), n_forced) blocks ("literal");
    the alternative "candidates" mode keeps ceil(density * n_candidates) Top-K blocks on
    top of the forced ones;
  - ties in the Top-K go to the lower block index;
  - a ragged last block is pooled over its valid tokens only;
  - blocks are counted globally over the concatenated KV; a block is forced when it holds
    any forced (text, or Clip-1 context) token;
  - no causal or intra-block mask; attention scale 1/sqrt(d).
The retained attention mass used by the self-checks follows the block-energy definition of
"Accelerating Text-to-Video Generation with Calibrated Sparse Attention" (papernotes.org),
section 关键设计 1, eq. (5): the softmax mass that a query block's rows put on a set of key
blocks, averaged over the rows.

Every array here is fp64 except the uint16 inputs and int64 index outputs.
"""
from __future__ import annotations

import math
from typing import Sequence, Tuple

import numpy as np

BLOCK = 128  # block edge of the partition, in tokens (方法概览)

BUDGET_LITERAL = 0      # rows hold max(ceil(density * nkb), n_forced) blocks
BUDGET_CANDIDATES = 1   # Top-K keeps ceil(density * n_candidates) non-forced blocks


# --------------------------------------------------------------------------- inputs

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) exactly to fp64: a bf16 is the top half of an fp32."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    as_f32 = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return as_f32.astype(np.float64)


# --------------------------------------------------------------------------- step 1

def num_blocks(n_tokens: int, block: int = BLOCK) -> int:
    """Number of `block`-token blocks covering n_tokens (the last one may be ragged)."""
    return -(-int(n_tokens) // block)


def block_token_range(j: int, n_tokens: int, block: int = BLOCK) -> Tuple[int, int]:
    """[start, end) token range of block j; the last block stops at n_tokens."""
    return j * block, min((j + 1) * block, n_tokens)


def forced_block_count(n_text: int, n_ctx: int, clip: int, block: int = BLOCK) -> int:
    """Blocks kept dense by the clip-aware rule (方法概览, bullet clip感知保留策略).

    The KV context is text ‖ reference context ‖ current tokens, so the forced blocks are a
    prefix of the KV blocks: the blocks holding text tokens, plus in Clip 1 the blocks
    holding image-pyramid tokens. A block holding any forced token counts as forced.
    """
    forced_tokens = n_text + (n_ctx if clip == 1 else 0)
    return num_blocks(forced_tokens, block)


def ceil_exact(x: float) -> int:
    """ceil with a 1e-9 guard so that a product such as 0.1875 * 16 = 3.0 stays 3."""
    return int(math.ceil(x - 1e-9))


def row_budget(nkb: int, n_forced: int, density: float, mode: int = BUDGET_LITERAL) -> Tuple[int, int]:
    """(K_total, K_topk): blocks kept per query-block row, and how many of them Top-K picks.

    Literal reading: fill each row to ceil(density * nkb) blocks, never fewer than the
    forced ones. Candidates reading: Top-K picks ceil(density * n_candidates) of the
    non-forced blocks. Both are clipped to what exists.
    """
    n_forced = min(n_forced, nkb)
    n_cand = nkb - n_forced
    if mode == BUDGET_LITERAL:
        k_total = min(max(ceil_exact(density * nkb), n_forced), nkb)
        k_topk = k_total - n_forced
    elif mode == BUDGET_CANDIDATES:
        k_topk = min(ceil_exact(density * n_cand), n_cand)
        k_total = n_forced + k_topk
    else:
        raise ValueError(f"unknown budget mode {mode}")
    return k_total, k_topk


# --------------------------------------------------------------------------- step 2

def pool_blocks(x: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Mean of the token vectors inside each block, [N, d] -> [nb, d] (方法概览, bullet 块划分与聚合评分:
    the block average).

    A ragged last block is averaged over its valid tokens only.
    """
    n, d = x.shape
    nb = num_blocks(n, block)
    out = np.zeros((nb, d), dtype=np.float64)
    for j in range(nb):
        s, e = block_token_range(j, n, block)
        out[j] = x[s:e].sum(axis=0) / (e - s)
    return out


# --------------------------------------------------------------------------- step 3

def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Aggregate compatibility S_ij = qbar_i . kbar_j / sqrt(d), [nqb, nkb] (方法概览)."""
    d = qbar.shape[1]
    return (qbar @ kbar.T) / math.sqrt(d)


# --------------------------------------------------------------------------- steps 4-5

def select_rows(S: np.ndarray, n_forced: int, k_topk: int) -> np.ndarray:
    """Kept KV blocks of each query-block row, ascending (方法概览: clip-aware retention + joint Top-K).

    S is [nqb, nkb]. The forced blocks 0..n_forced-1 are always kept. The K_topk
    highest-scoring remaining blocks join them; among equal scores the lower block index
    comes first; -0.0 and +0.0 are the same score; NaN (never produced from finite inputs)
    ranks below every number, -inf included. The ranking is one library sort per row on the
    key (is NaN, -score, index).
    """
    nqb, nkb = S.shape
    n_forced = min(n_forced, nkb)
    cand = S[:, n_forced:]
    is_nan = np.isnan(cand)
    value = np.where(is_nan, 0.0, cand) + 0.0             # + 0.0 turns -0.0 into +0.0
    index = np.broadcast_to(np.arange(n_forced, nkb), cand.shape)
    order = np.lexsort((index, -value, is_nan), axis=-1)  # primary key last
    chosen = np.sort(order[:, :k_topk] + n_forced, axis=1)
    forced = np.broadcast_to(np.arange(n_forced), (nqb, n_forced))
    return np.concatenate([forced, chosen], axis=1).astype(np.int64)


def select_row(scores_row: np.ndarray, n_forced: int, k_topk: int) -> np.ndarray:
    """One row of select_rows."""
    return select_rows(np.asarray(scores_row, dtype=np.float64)[None, :], n_forced, k_topk)[0]


def select_head(q: np.ndarray, k: np.ndarray, n_text: int, n_ctx: int, clip: int,
                density: float, mode: int = BUDGET_LITERAL, block: int = BLOCK):
    """One head's block mask. q [Nq,d], k [Nkv,d] fp64 -> (rows [nqb, K_total] int64, S [nqb, nkb])."""
    nkb = num_blocks(k.shape[0], block)
    n_forced = min(forced_block_count(n_text, n_ctx, clip, block), nkb)
    k_total, k_topk = row_budget(nkb, n_forced, density, mode)
    S = block_scores(pool_blocks(q, block), pool_blocks(k, block))
    return select_rows(S, n_forced, k_topk), S


def select(q_bits: np.ndarray, k_bits: np.ndarray, n_text: int, n_ctx: int, clip: int,
           density: float, mode: int = BUDGET_LITERAL, block: int = BLOCK):
    """All heads (per-head masks, bullet per-head动态掩码). Inputs are bf16 bits [H,N,d].

    Returns (idx [H, nqb, K_total] int64, scores [H, nqb, nkb] fp64).
    """
    H = q_bits.shape[0]
    idx, scores = [], []
    for h in range(H):
        rows, S = select_head(bf16_bits_to_f64(q_bits[h]), bf16_bits_to_f64(k_bits[h]),
                              n_text, n_ctx, clip, density, mode, block)
        idx.append(rows)
        scores.append(S)
    return np.stack(idx), np.stack(scores)


# --------------------------------------------------------------------------- step 6

def kept_token_index(kept_blocks: Sequence[int], n_kv: int, block: int = BLOCK) -> np.ndarray:
    """Token positions of the kept KV blocks (valid tokens only)."""
    parts = [np.arange(*block_token_range(int(j), n_kv, block)) for j in kept_blocks]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def attend_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, tokens: np.ndarray,
                sm_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of q_rows over the listed KV tokens (bullet FastFlex执行路径).

    logits l_u = sm_scale * q . k_u; o = sum_u softmax(l)_u v_u; lse = log sum_u exp(l_u).
    Returns (o [n, d], lse [n]) in fp64.
    """
    logits = (q_rows @ k[tokens].T) * sm_scale
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    z = e.sum(axis=1, keepdims=True)
    o = (e @ v[tokens]) / z
    lse = (m + np.log(z))[:, 0]
    return o, lse


def block_sparse_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, rows: np.ndarray,
                           qblocks: Sequence[int], sm_scale: float | None = None,
                           block: int = BLOCK):
    """Attention of the listed query blocks over their kept KV blocks (one head, fp64 inputs).

    rows[i] is the kept-block list of query block i (entries < 0 are ignored). Returns a
    list of (o [n_i, d], lse [n_i]) in the order of qblocks.
    """
    d = q.shape[1]
    scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    out = []
    for i in qblocks:
        s, e = block_token_range(int(i), q.shape[0], block)
        kept = [int(j) for j in rows[int(i)] if j >= 0]
        out.append(attend_rows(q[s:e], k, v, kept_token_index(kept, k.shape[0], block), scale))
    return out


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, qblocks: Sequence[int],
                    sm_scale: float | None = None, block: int = BLOCK):
    """Attention over every KV token (the density = 1 case), same return as above."""
    nkb = num_blocks(k.shape[0], block)
    all_rows = np.tile(np.arange(nkb), (num_blocks(q.shape[0], block), 1))
    return block_sparse_attention(q, k, v, all_rows, qblocks, sm_scale, block)


def retained_mass(lse_kept: np.ndarray, lse_dense: np.ndarray) -> np.ndarray:
    """Per query row, the dense softmax mass on the kept tokens: exp(lse_kept - lse_dense).

    Averaged over the rows of a query block this is the block energy of eq. (5) of the
    CalibAtt notes, summed over the kept key blocks.
    """
    return np.exp(lse_kept - lse_dense)


def block_energy(q: np.ndarray, k: np.ndarray, qblock: int, key_blocks: Sequence[int],
                 sm_scale: float | None = None, block: int = BLOCK) -> float:
    """Eq. (5) of the CalibAtt notes, summed over key_blocks: (1/n_i) sum_t sum_u P_tu.

    P is the dense softmax over all KV tokens; rows t are the valid tokens of query block
    `qblock` (n_i of them) and columns u the valid tokens of key_blocks.
    """
    d = q.shape[1]
    scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    s, e = block_token_range(qblock, q.shape[0], block)
    logits = (q[s:e] @ k.T) * scale
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    p /= p.sum(axis=1, keepdims=True)
    cols = kept_token_index(key_blocks, k.shape[0], block)
    return float(p[:, cols].sum() / (e - s))


def kept_token_count(kept_blocks: Sequence[int], n_kv: int, block: int = BLOCK) -> int:
    """Valid KV tokens in the listed blocks (a ragged last block counts its valid tokens)."""
    return int(len(kept_token_index(kept_blocks, n_kv, block)))


def dense_probabilities(q_rows: np.ndarray, k: np.ndarray, sm_scale: float | None = None) -> np.ndarray:
    """Dense softmax rows P_tu = exp(l_tu) / sum_u exp(l_tu), l_tu = sm_scale * q_t . k_u."""
    scale = 1.0 / math.sqrt(q_rows.shape[1]) if sm_scale is None else sm_scale
    logits = (q_rows @ k.T) * scale
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    return p / p.sum(axis=1, keepdims=True)


def token_topk_bound(q_rows: np.ndarray, k: np.ndarray, budget, sm_scale: float | None = None) -> np.ndarray:
    """Token-wise upper bound on the retained mass (digest section 关键结果与论文证据, bullet
    跨尺度复用损失, Figure 3): for each query row, the largest dense softmax mass that any
    `budget` key tokens can hold, i.e. the sum of the row's `budget` largest probabilities.
    `budget` is one count for all rows or one per row; a block mask keeping `budget` tokens
    can retain at most this much."""
    p = dense_probabilities(q_rows, k, sm_scale)
    srt = -np.sort(-p, axis=1)
    b = np.broadcast_to(np.asarray(budget, dtype=np.int64), (p.shape[0],))
    out = np.empty(p.shape[0])
    for t in range(p.shape[0]):
        out[t] = srt[t, :int(b[t])].sum()
    return out


def mass_report(q: np.ndarray, k: np.ndarray, rows: np.ndarray, qblocks: Sequence[int],
                sm_scale: float | None = None, block: int = BLOCK):
    """For each listed query block i with kept blocks rows[i]: the mean over its valid rows t of
    the retained mass R_t (dense softmax mass on the kept tokens; eq. (5) of the CalibAtt notes
    divided by nothing else) and of the token-wise bound U_t with the same token budget.
    Returns (E [len(qblocks)], U [len(qblocks)], R rows, U rows) with the per-row arrays
    concatenated in qblocks order."""
    E, U, R_rows, U_rows = [], [], [], []
    for i in qblocks:
        s, e = block_token_range(int(i), q.shape[0], block)
        tokens = kept_token_index(rows[i], k.shape[0], block)
        p = dense_probabilities(q[s:e], k, sm_scale)
        r = p[:, tokens].sum(axis=1)
        u = token_topk_bound(q[s:e], k, len(tokens), sm_scale)
        E.append(r.mean())
        U.append(u.mean())
        R_rows.append(r)
        U_rows.append(u)
    return np.array(E), np.array(U), np.concatenate(R_rows), np.concatenate(U_rows)



def reference_mass(q: np.ndarray, k: np.ndarray, kept_ref_blocks: np.ndarray, n_text: int, n_ctx: int,
                   qblocks: Sequence[int], sm_scale: float | None = None, block: int = BLOCK) -> np.ndarray:
    """Retained attention mass over the reference context (关键结果与论文证据, bullet 跨clip边界,
    Figure 4): for each listed query block i, the mean over its valid rows t of
    sum_{u in kept reference tokens} P_tu / sum_{u in all reference tokens} P_tu, with P the
    dense softmax of row t over every KV token and kept_ref_blocks[i] the kept reference
    blocks (block ids of the whole KV, all inside [n_text, n_text + n_ctx))."""
    ref = np.arange(n_text, n_text + n_ctx)
    out = []
    for i in qblocks:
        s, e = block_token_range(int(i), q.shape[0], block)
        p = dense_probabilities(q[s:e], k, sm_scale)
        tokens = kept_token_index(kept_ref_blocks[i], k.shape[0], block)
        out.append((p[:, tokens].sum(axis=1) / p[:, ref].sum(axis=1)).mean())
    return np.array(out)


def reference_reuse_report(q_now: np.ndarray, q_prev: np.ndarray, k: np.ndarray, n_text: int, n_ctx: int,
                           budget_frac: float, qblocks: Sequence[int], sm_scale: float | None = None,
                           block: int = BLOCK):
    """Fresh against reused selection over the reference context under one reference budget
    (关键结果与论文证据, bullet 跨clip边界; Figure 4). The reference context of the current clip
    is the preceding clip's final scale, so its key blocks are the tokens that clip's final
    scale selected among. Per query block i the budget is ceil(budget_frac * n_ref) of the
    n_ref reference blocks; fresh: the best of them by the current queries' block scores;
    reused: the best by the preceding clip's queries of the same query block (same position
    in the clip). Ties go to the lower index. Segments must be whole blocks.
    Returns (fresh rows [nqb, K], reused rows [nqb, K], E_fresh, E_reused) with block ids of
    the whole KV and E over qblocks (reference_mass)."""
    assert n_text % block == 0 and n_ctx % block == 0 and q_now.shape == q_prev.shape
    nb_text, n_ref = n_text // block, n_ctx // block
    k_ref = ceil_exact(budget_frac * n_ref)
    kbar = pool_blocks(k[n_text:n_text + n_ctx], block)
    fresh = select_rows(block_scores(pool_blocks(q_now, block), kbar), 0, k_ref) + nb_text
    reused = select_rows(block_scores(pool_blocks(q_prev, block), kbar), 0, k_ref) + nb_text
    e_fresh = reference_mass(q_now, k, fresh, n_text, n_ctx, qblocks, sm_scale, block)
    e_reused = reference_mass(q_now, k, reused, n_text, n_ctx, qblocks, sm_scale, block)
    return fresh, reused, e_fresh, e_reused

# --------------------------------------------------------------------------- mask reuse across scales

def raster_block_map(grid_now: Sequence[int], grid_prev: Sequence[int], block: int = BLOCK) -> np.ndarray:
    """For every block of a scale's current tokens, laid out on grid_now = (T', H', W') in raster
    order (frame, row, column), the block of the previous scale's grid_prev = (T, H, W) that holds
    the nearest raster position (digest section 关键结果与论文证据, bullet 重算频率, Figure 5:
    a mask computed at one scale and reused at the next needs this correspondence; the pages do
    not give it). A block is represented by its middle token c = start + (n - 1) // 2; along
    each axis the new cell centre (x + 1/2) / X' falls in the old cell floor((2x + 1) X / (2 X')),
    clipped to the last cell; the old token is unravelled back to a raster index and divided
    by the block size."""
    Tn, Hn, Wn = (int(x) for x in grid_now)
    To, Ho, Wo = (int(x) for x in grid_prev)
    n_now = Tn * Hn * Wn
    out = np.empty(num_blocks(n_now, block), dtype=np.int64)
    for b in range(len(out)):
        s, e = block_token_range(b, n_now, block)
        c = s + (e - s - 1) // 2
        t, rem = divmod(c, Hn * Wn)
        h, w = divmod(rem, Wn)
        to = min(To - 1, (2 * t + 1) * To // (2 * Tn))
        ho = min(Ho - 1, (2 * h + 1) * Ho // (2 * Hn))
        wo = min(Wo - 1, (2 * w + 1) * Wo // (2 * Wn))
        out[b] = ((to * Ho + ho) * Wo + wo) // block
    return out


def map_scores(S_prev: np.ndarray, n_prefix_blocks: int, grid_prev: Sequence[int], grid_now: Sequence[int],
               block: int = BLOCK) -> np.ndarray:
    """Block scores of the previous scale carried to the current one (reuse instead of
    recompute, Figure 5): S_now[i', j'] = S_prev[m(i'), c(j')], m = raster_block_map (query
    blocks are current-scale blocks), c(j') = j' for the KV prefix of text and reference-context
    blocks (the same tokens at every scale of a clip) and n_prefix + m(j' - n_prefix) for the
    current-scale blocks. S_prev is [nqb_prev, n_prefix + nb_cur_prev]."""
    m = raster_block_map(grid_now, grid_prev, block)
    cols = np.concatenate([np.arange(n_prefix_blocks), n_prefix_blocks + m])
    assert S_prev.shape == (num_blocks(int(np.prod(grid_prev)), block),
                            n_prefix_blocks + num_blocks(int(np.prod(grid_prev)), block))
    return S_prev[np.ix_(m, cols)]


def reused_rows(S_prev: np.ndarray, n_prefix_blocks: int, grid_prev: Sequence[int], grid_now: Sequence[int],
                n_forced: int, k_topk: int, block: int = BLOCK) -> np.ndarray:
    """Kept blocks of the current scale chosen from the previous scale's mapped scores: the
    clip-aware forced prefix, then the current scale's own budget of K_topk by the joint Top-K
    rule (ties to the lower index), exactly as a fresh selection but without new scores."""
    return select_rows(map_scores(S_prev, n_prefix_blocks, grid_prev, grid_now, block), n_forced, k_topk)


__all__ = [
    "BLOCK", "BUDGET_LITERAL", "BUDGET_CANDIDATES", "bf16_bits_to_f64", "num_blocks",
    "block_token_range", "forced_block_count", "row_budget", "pool_blocks", "block_scores",
    "select_rows", "select_row", "select_head", "select", "kept_token_index", "attend_rows",
    "block_sparse_attention", "dense_attention", "retained_mass", "block_energy",
    "kept_token_count", "dense_probabilities", "token_topk_bound", "mass_report", "reference_mass",
    "reference_reuse_report", "raster_block_map", "map_scores", "reused_rows",
]

