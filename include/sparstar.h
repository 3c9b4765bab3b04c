/*
 * sparstar.h — C ABI of the B200 (sm_100a) SparSTAR block-sparse attention library.
 *
 * The library computes, for one expensive scale of a SpaceTime-AutoRegressive video model,
 * the training-free dynamic block-sparse attention described in the SparSTAR digest
 * ("SparSTAR的贡献：每尺度动态重建", pchao.org, section 方法概览 "method overview") and in the
 * English abstract ("SparSTAR: Sparse Attention for SpaceTime AutoRegressive Video
 * Synthesis", newx.sg, section Abstract):
 *   per head, Q and the mixed KV context (text ‖ reference context ‖ current-scale tokens)
 *   are cut into 128-token blocks; each block is mean-pooled; every (query block, key
 *   block) pair is scored from the pooled vectors; text blocks (and, in Clip 1, the image
 *   pyramid blocks) are always kept; the rest of each query-block row is filled by a joint
 *   Top-K; forward-only attention then runs over the kept blocks only.
 *
 * Conventions fixed by this library where the pages are silent:
 *   score      S_ij = mean(q_i) . mean(k_j) / sqrt(d), fp32;
 *   budget     SPARSTAR_BUDGET_LITERAL: each row holds max(ceil(density * nkb), n_forced)
 *              blocks; SPARSTAR_BUDGET_CANDIDATES: Top-K adds ceil(density * n_cand)
 *              blocks to the forced ones;
 *   ties       equal scores rank the lower block index first; -0.0 equals +0.0;
 *   ragged     a partial last block is pooled over (and attends to) its valid tokens only;
 *   blocks     counted over the concatenated KV; a block holding any forced token is forced;
 *   attention  no causal mask; softmax scale sm_scale (<= 0 selects 1/sqrt(d)).
 *
 * Memory layout (all device pointers, row-major, contiguous, 16-byte aligned):
 *   q   bf16 [H, Nq,  d]      k, v bf16 [H, Nkv, d]      o bf16 [H, Nq, d]
 *   lse fp32 [H, Nq]          (natural-log sum of exp of the scaled logits; optional)
 *   idx int32 [H, nqb, kmax]  (kept KV block ids of each row, ascending; only the first
 *                              cnt entries of a row are written and read)
 *   cnt int32 [H, nqb]
 * with nqb = ceil(Nq/128), nkb = ceil(Nkv/128), Nkv = n_text + n_ctx + n_cur.
 *
 * Ownership: the caller allocates and owns every buffer; the library allocates no device
 * memory in these calls. All calls are asynchronous on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and return after enqueuing. Argument errors are detected on
 * the host before anything is enqueued and leave every output untouched.
 *
 * Device-side faults never trap: each kernel bounds its waits and index reads, records a
 * flag in a per-device status word, and exits. sparstar_device_status() reports it.
 */
#ifndef SPARSTAR_H
#define SPARSTAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPARSTAR_BLOCK 128
/* 2: adds sparstar_map_scores and sparstar_read_probe (every version-1 entry point unchanged). */
#define SPARSTAR_ABI_VERSION 2

/* Return codes. */
#define SPARSTAR_OK 0
#define SPARSTAR_ERR_ARG 1             /* bad pointer, size, alignment, density or clip */
#define SPARSTAR_ERR_UNSUPPORTED 2     /* head_dim not in {64,128}, device not sm_100, size beyond a limit,
                                         or a library build whose attention kernels launch with
                                         too few registers for their setmaxnreg split */
#define SPARSTAR_ERR_WORKSPACE 3       /* workspace NULL or smaller than sparstar_workspace_size() */
#define SPARSTAR_ERR_CUDA 4            /* a CUDA runtime/driver call failed */
#define SPARSTAR_ERR_DEVICE_TIMEOUT 5  /* a kernel's bounded wait expired (reported by sparstar_device_status) */
#define SPARSTAR_ERR_DEVICE_BOUNDS 6   /* a kernel clamped an out-of-range idx/cnt entry */

/* Budget readings (see the header comment). */
#define SPARSTAR_BUDGET_LITERAL 0
#define SPARSTAR_BUDGET_CANDIDATES 1

/* KV context = n_text text tokens ‖ n_ctx reference tokens ‖ n_cur current-scale tokens.
 * In Clip 1 the reference tokens are the image pyramid, in later clips the preceding
 * clip's final scale (digest, section 这篇论文解决什么问题 and bullet clip感知保留策略). */
typedef struct sparstar_segments {
    int64_t n_text;
    int64_t n_ctx;
    int64_t n_cur;
} sparstar_segments;

/* Block counts and per-row budget of one scale. */
typedef struct sparstar_plan {
    int64_t nqb;       /* query blocks, ceil(Nq/128) */
    int64_t nkb;       /* KV blocks, ceil(Nkv/128) */
    int64_t n_forced;  /* forced (always kept) KV blocks, a prefix 0..n_forced-1 */
    int64_t n_cand;    /* nkb - n_forced, the blocks Top-K chooses from */
    int32_t k_total;   /* blocks kept per row (= every row's cnt) */
    int32_t k_topk;    /* of which chosen by Top-K */
} sparstar_plan;

/* Host only. Block partition, clip-aware forced prefix and row budget (digest, 方法概览:
 * 128-token blocks; text, plus Clip-1 pyramid, kept dense; the rest filled by joint Top-K).
 * clip >= 1; 0 < density <= 1; budget_mode is SPARSTAR_BUDGET_*. n_q may be 0.
 * Returns SPARSTAR_ERR_ARG on bad input (out untouched). */
int sparstar_make_plan(int64_t n_q, sparstar_segments seg, int clip, double density,
                       int budget_mode, sparstar_plan* out);

/* Host only. Bytes of device workspace that sparstar_select / sparstar_forward need for
 * these sizes (the pooled block means, each stored as a bf16 hi/lo pair, and, unless the
 * caller passes `scores`, the fp32 score matrix). Writes *bytes; returns SPARSTAR_ERR_ARG
 * on bad sizes. */
int sparstar_workspace_size(int heads, int64_t n_q, sparstar_segments seg, int head_dim,
                            size_t* bytes);

/* Block selection (digest, 方法概览: block partition and aggregate scoring, clip-aware
 * retention, joint Top-K, per-head masks). Reads q [H,Nq,d] and k [H,Nkv,d] (bf16, device),
 * writes idx [H,nqb,kmax] (first plan.k_total entries of each row, ascending) and
 * cnt [H,nqb] (= plan.k_total). If `scores` is not NULL it must hold H*nqb*nkb floats and
 * receives every S_ij (forced columns included); it is then used instead of workspace for
 * the scores. Rows whose budget is already filled by the forced blocks (k_topk == 0), or
 * that keep every block, do not depend on the scores: q and k are then not read unless
 * `scores` was requested.
 * workspace: device, >= sparstar_workspace_size() bytes, 256-byte aligned.
 * Requirements: heads >= 1, n_q >= 0, Nkv >= 1, head_dim in {64,128}, kmax >= k_total,
 * n_cand <= 16384. n_q == 0 is a no-op. */
int sparstar_select(const void* q, const void* k, int heads, int64_t n_q,
                    sparstar_segments seg, int head_dim, int clip, double density,
                    int budget_mode, int32_t* idx, int32_t* cnt, int32_t kmax,
                    float* scores, void* workspace, size_t workspace_bytes, void* stream);

/* Clip-aware retention and joint Top-K on scores the caller supplies (digest, 方法概览: the
 * forced blocks are kept, the rest of each row is filled by a joint Top-K; the selection
 * steps of sparstar_select without pooling and scoring). scores: fp32 [rows, nkb] device,
 * 4-byte aligned; columns 0..n_forced-1 are the forced blocks and are not read. Row r of
 * idx [rows, kmax] receives 0..n_forced-1, then the k_topk highest-scoring columns in
 * [n_forced, nkb) in ascending order: equal scores go to the lower column, NaN ranks below
 * every number, -0.0 equals +0.0. cnt[r] = n_forced + k_topk. Entries of idx past that
 * count are not written. The result is exact: no tolerance applies to the ranking.
 * Requirements: rows >= 0, 0 <= n_forced <= nkb, 0 <= k_topk <= nkb - n_forced,
 * kmax >= n_forced + k_topk (else SPARSTAR_ERR_ARG); rows <= 2^31 - 1 and, when the scores
 * are read (0 < k_topk < nkb - n_forced), nkb - n_forced <= 16384 (else
 * SPARSTAR_ERR_UNSUPPORTED); scores may be NULL when they are not read. rows == 0 is a
 * no-op. Requires an sm_100 device. */
int sparstar_topk(const float* scores, int64_t rows, int nkb, int n_forced, int k_topk,
                  int32_t* idx, int32_t* cnt, int32_t kmax, void* stream);

/* Forward-only block-sparse attention over the kept tiles (digest, 方法概览 bullet
 * FastFlex执行路径: attention executed over the selected blocks only, with online softmax).
 * For every valid query token t of query block i of head h:
 *   o_t = sum over valid KV tokens u of the blocks idx[h][i][0..cnt-1] of
 *         softmax_u(sm_scale * q_t . k_u) v_u,   lse_t = log sum_u exp(sm_scale * q_t . k_u).
 * q [H,Nq,d], k/v [H,Nkv,d] bf16 device; o [H,Nq,d] bf16 device (written);
 * lse fp32 [H,Nq] device or NULL. idx entries must lie in [0,nkb) and cnt in [1,kmax]:
 * out-of-range entries are clamped and SPARSTAR_ERR_DEVICE_BOUNDS is recorded.
 * Requires an sm_100 device. n_q == 0 is a no-op. */
int sparstar_attn(const void* q, const void* k, const void* v, int heads, int64_t n_q,
                  int64_t n_kv, int head_dim, const int32_t* idx, const int32_t* cnt,
                  int32_t kmax, float sm_scale, void* o, float* lse, void* stream);

/* sparstar_select followed by sparstar_attn on the same stream (the whole per-scale path). */
int sparstar_forward(const void* q, const void* k, const void* v, int heads, int64_t n_q,
                     sparstar_segments seg, int head_dim, int clip, double density,
                     int budget_mode, float sm_scale, int32_t* idx, int32_t* cnt,
                     int32_t kmax, void* o, float* lse, void* workspace,
                     size_t workspace_bytes, void* stream);

/* Block selection for callers that cannot allocate device memory: the same computation
 * and outputs as sparstar_select (with scores == NULL), but the scratch it needs (pooled
 * block means and the score matrix) lives in a fixed array inside the library instead of
 * a caller-provided workspace. The paper has no counterpart; this exists for callers that
 * run where cudaMalloc is unavailable or forbidden, e.g. inside a host framework that owns
 * all device memory through its own pool, a plugin that must not allocate, or code that
 * runs while a memory-capping policy is in force.
 * The array holds SPARSTAR_NOALLOC_SCRATCH_BYTES bytes on every device that loads the
 * library, until the process exits. When the rows depend on the scores (0 < k_topk < n_cand
 * in the plan), sizes whose sparstar_workspace_size() exceeds it are rejected with
 * SPARSTAR_ERR_UNSUPPORTED before anything is enqueued; rows that do not depend on the
 * scores (forced-only rows, or rows keeping every block) use no scratch and have no limit
 * beyond those of sparstar_select.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream capture.
 * All calls on a device share the one array and it keeps the last call's contents; every
 * value a call reads from it is written earlier by the same call, so nothing needs
 * clearing. Calls whose kernels overlap on the GPU (different streams without ordering,
 * or several host threads) race on the array: serialize them.
 * No cudaMalloc, cudaFree or allocating library routine is called. Other arguments,
 * requirements and return codes are those of sparstar_select. */
#define SPARSTAR_NOALLOC_SCRATCH_BYTES ((size_t)128 << 20)
int sparstar_select_noalloc(const void* q, const void* k, int heads, int64_t n_q,
                            sparstar_segments seg, int head_dim, int clip, double density,
                            int budget_mode, int32_t* idx, int32_t* cnt, int32_t kmax,
                            void* stream);

/* Block-size variants (the pages' block-size ablation, section 实验如何设计?, bullet on the
 * supplementary experiments): the same calls with the block size of the partition as an
 * argument, block in {64, 128} (anything else: SPARSTAR_ERR_UNSUPPORTED). Every count in the
 * plan (nqb, nkb, n_forced, budgets) and every index in idx is then in units of `block`
 * tokens; a ragged last block holds the remaining tokens. The functions without the suffix
 * are these with block = SPARSTAR_BLOCK (128). The no-allocation entry point, the retained
 * mass and the token-wise bound work on 128-token blocks only. */
int sparstar_make_plan_ex(int64_t n_q, sparstar_segments seg, int clip, double density,
                          int budget_mode, int block, sparstar_plan* out);
int sparstar_workspace_size_ex(int heads, int64_t n_q, sparstar_segments seg, int head_dim,
                               int block, size_t* bytes);
int sparstar_select_ex(const void* q, const void* k, int heads, int64_t n_q,
                       sparstar_segments seg, int head_dim, int clip, double density,
                       int budget_mode, int block, int32_t* idx, int32_t* cnt, int32_t kmax,
                       float* scores, void* workspace, size_t workspace_bytes, void* stream);
int sparstar_attn_ex(const void* q, const void* k, const void* v, int heads, int64_t n_q,
                     int64_t n_kv, int head_dim, int block, const int32_t* idx,
                     const int32_t* cnt, int32_t kmax, float sm_scale, void* o, float* lse,
                     void* stream);
int sparstar_forward_ex(const void* q, const void* k, const void* v, int heads, int64_t n_q,
                        sparstar_segments seg, int head_dim, int clip, double density,
                        int budget_mode, int block, float sm_scale, int32_t* idx, int32_t* cnt,
                        int32_t kmax, void* o, float* lse, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Retained attention mass of a block mask (digest, 关键结果与论文证据, bullet 跨尺度复用损失,
 * Figure 3; block energy of eq. (5) of the CalibAtt notes): for every valid query token t,
 * R_t = exp(lse_kept[t] - lse_dense[t]), the share of its dense softmax mass on the kept
 * tokens, and per query block the mean of R_t over its valid tokens.
 * lse_kept / lse_dense: fp32 [H,Nq] device, natural-log LSEs of sparstar_attn with the mask
 * and with every block kept (cnt = nkb). r_token: fp32 [H,Nq] device or NULL;
 * e_block: fp32 [H,nqb] device. n_q == 0 is a no-op. */
int sparstar_retained_mass(const float* lse_kept, const float* lse_dense, int heads,
                           int64_t n_q, float* r_token, float* e_block, void* stream);

/* Latent grid of a scale's current-scale tokens in raster order (frame, row, column):
 * frames * height * width == n_cur. */
typedef struct sparstar_grid {
    int64_t frames;
    int64_t height;
    int64_t width;
} sparstar_grid;

/* Mask reuse across scales (digest, 关键结果与论文证据, bullet 重算频率, Figure 5: the mask
 * recomputed at every scale, every second scale, or once and transferred). Carries the block
 * scores of a previous scale of the same clip (from sparstar_select with `scores`) to the
 * current scale, so that sparstar_topk can fill the current scale's rows without new scores:
 *   scores_now[h][i][j] = scores_prev[h][m(i)][c(j)],
 * with m(b) the previous-scale block that holds the nearest raster position of current block b
 * (b's middle token c = 128 b + (n_b - 1) / 2 on grid_now, each axis x of size X' moved to the
 * cell (2x + 1) X / (2 X') of grid_prev, clipped to X - 1, and ravelled back), and c(j) = j for
 * the text and reference blocks (the same tokens at every scale) and n_prefix + m(j - n_prefix)
 * for the current-scale blocks. Query blocks are current-scale blocks. The pages give no block
 * correspondence between scales; this nearest-position map is this library's reading.
 * scores_prev fp32 [H, ceil(n_cur_prev/128), n_prefix + ceil(n_cur_prev/128)] device,
 * scores_now fp32 [H, ceil(n_cur_now/128), n_prefix + ceil(n_cur_now/128)] device (written),
 * n_prefix = (n_text + n_ctx) / 128. Requirements: 1 <= heads <= 65535; grids of positive
 * sizes whose products equal each scale's n_cur; equal n_text and n_ctx in both scales, each a
 * multiple of 128 (else SPARSTAR_ERR_ARG); n_prefix + ceil(n_cur_now/128) <= 49152 (else
 * SPARSTAR_ERR_UNSUPPORTED). Exact: a gather, no arithmetic on the scores. */
int sparstar_map_scores(const float* scores_prev, int heads, sparstar_segments seg_prev,
                        sparstar_grid grid_prev, sparstar_segments seg_now, sparstar_grid grid_now,
                        float* scores_now, void* stream);

/* Device bytes of the workspace of sparstar_token_bound: four [H,Nq] arrays of 4 bytes. */
int sparstar_token_bound_workspace_size(int heads, int64_t n_q, size_t* bytes);

/* Token-wise upper bound on the retained mass (same passage): for every valid query token t
 * of query block i, U_t = the sum of the B_i largest dense softmax probabilities of row t
 * over all Nkv tokens, B_i = the number of valid KV tokens in the blocks
 * idx[h][i][0..cnt-1]; per query block the mean of U_t. Computed from the dense logits
 * sm_scale * q . k (recomputed on the tensor cores, every (query block, KV block) tile, four
 * times) normalised by lse_dense; the B_i-th largest value is located to 2^-14 in log2 and
 * the boundary bin's mean stands in for its last values (relative error of U below 5e-5
 * beyond the logits' own rounding). q [H,Nq,d], k [H,Nkv,d] bf16 device; idx/cnt as for
 * sparstar_attn (out-of-range entries are skipped and SPARSTAR_ERR_DEVICE_BOUNDS recorded);
 * lse_dense fp32 [H,Nq] (natural log, from sparstar_attn with every block kept);
 * sm_scale <= 0 selects 1/sqrt(d). u_token: fp32 [H,Nq] device or NULL; u_block: fp32
 * [H,nqb] device. workspace: device, >= sparstar_token_bound_workspace_size() bytes,
 * 256-byte aligned. ceil(n_kv/128) <= 4095 (the counting passes keep 16-bit counts; else
 * SPARSTAR_ERR_UNSUPPORTED). Requires an sm_100 device. n_q == 0 is a no-op. */
int sparstar_token_bound(const void* q, const void* k, int heads, int64_t n_q, int64_t n_kv,
                         int head_dim, const int32_t* idx, const int32_t* cnt, int32_t kmax,
                         const float* lse_dense, float sm_scale, float* u_token, float* u_block,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Synchronizes `stream`, then returns SPARSTAR_OK, SPARSTAR_ERR_DEVICE_TIMEOUT or
 * SPARSTAR_ERR_DEVICE_BOUNDS from the current device's status word (timeout wins), or
 * SPARSTAR_ERR_CUDA if the synchronization itself failed. clear != 0 resets the word. */
int sparstar_device_status(void* stream, int clear);

/* Self-test of failure reporting: enqueues one thread that waits, with the same bounded
 * mbarrier wait the kernels use, on a barrier nothing completes. After the wait limit (2 s
 * of %globaltimer) the thread records a timeout in the device status word and the kernel
 * returns normally, so a later sparstar_device_status() returns SPARSTAR_ERR_DEVICE_TIMEOUT
 * and the CUDA context stays usable. Requires an sm_100 device. */
int sparstar_selftest_wait_timeout(void* stream);

/* Measurement aid, not a step of the method: reads `bytes` bytes at `src` (device, 16-byte
 * aligned, a multiple of 16) once, with the streaming 16-byte loads of the pooling kernel,
 * and XORs them into *sink (device, 4 bytes). Its duration gives the read-only streaming
 * bandwidth that the read-bound selection is measured against (a copy reads and writes).
 * bytes == 0 is a no-op; bad pointers or sizes give SPARSTAR_ERR_ARG. */
int sparstar_read_probe(const void* src, size_t bytes, unsigned* sink, void* stream);

/* Static text for a return code (never NULL). */
const char* sparstar_strerror(int code);

/* SPARSTAR_ABI_VERSION of the loaded library. */
int sparstar_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSTAR_H */
