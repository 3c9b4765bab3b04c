// Forward-only block-sparse flash attention over kept 128x128 tiles, for sm_100a.
//
// Computes the attention of the SparSTAR digest ("SparSTAR的贡献：每尺度动态重建", pchao.org),
// section 方法概览, bullet FastFlex执行路径: only the KV blocks listed for a query block are
// visited, with an online softmax across them. The pages' executor (a FlexAttention
// variant) is prior art for other hardware; this kernel is written for Blackwell:
//
//   * persistent grid, one CTA per SM; a CTA owns two "slots", each working through its own
//     sequence of (head, query block) items, so the softmax of one slot overlaps the tensor
//     core work of the other;
//   * warp 8 (TMA): loads the slot's 128xd Q tile once per item and, per kept block, the K
//     and V tiles into a ring of shared-memory stages (128-byte swizzle; each CTA loads its own;
//     Q with an L2 evict-first policy, K/V evict-last, and O is written with streaming stores,
//     so that the K/V of the head in flight stays in L2);
//   * warp 9 (MMA, one thread): S = Q K^T into tensor memory (tcgen05.mma, M=128, N=128,
//     K=16 steps), then O += P V with P read from tensor memory;
//   * warps 10-11: idle, they complete the producer warpgroup so that setmaxnreg can move
//     its registers to the softmax warps;
//   * warps 0-3 / 4-7 (softmax of slot 0 / 1, one thread per query row): tcgen05.ld of the
//     S row, masking of a ragged last KV block, running max with a lazy rescale (the
//     running max only moves when a tile's max exceeds it by more than 8 in log2 units,
//     so P stays <= 256 and O is rarely rescaled), exp2, row sum, bf16 P written back over
//     S with tcgen05.st, and the epilogue O / l -> bf16, lse = ln 2 * (m + log2 l).
//
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 [384,384+d).
// P of slot s overwrites the first 64 columns of S_s as packed bf16 pairs.
//
// Ordering: tcgen05.mma ops issued by one thread execute in order, and a tcgen05.commit
// arrives once all earlier ops of that thread are done. S_s(n+1) is issued after
// PV_s(n), so when the softmax sees S_s(n+1) complete, PV_s(n) is complete too: it may
// rescale O_s and overwrite P_s without further waits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparstar {

// B = block size of the partition (128, or 64 for the block-size variant): a query block is B
// rows of the 128-row MMA tile (with B = 64 the other 64 rows are computed and dropped), and a
// KV tile is 128 tokens: one KV block, or with B = 64 two consecutive entries of the kept
// list, each loaded as its own 64-row box into one half of the stage (a 64-row box at a
// 1 KB-aligned offset lands in the same swizzled layout as rows 64-127 of a 128-row box).
// An odd last entry fills both halves with the same block and the second half is masked.
template <int D, int B = 128>
struct AttnConfig {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static_assert(B == 64 || B == 128, "block must be 64 or 128");
  static constexpr int kRows = 128;                    // query rows per MMA tile
  static constexpr int kCols = 128;                    // KV tokens per tile
  static constexpr int kBlocksPerTile = kCols / B;     // KV blocks per tile
  static constexpr int kSC = kCols / 32;               // 32-column chunks of an S row
  static constexpr int kChunks = D / 64;               // 128-byte swizzle chunks per row
  static constexpr uint32_t kQChunkBytes = 128 * 128;  // 128 rows x 128 bytes
  static constexpr uint32_t kKVChunkBytes = kCols * 128;  // 128 rows x 128 bytes
  static constexpr uint32_t kKVBoxBytes = B * 128;     // one KV block's rows of a chunk
  static constexpr uint32_t kQTileBytes = kChunks * kQChunkBytes;
  static constexpr uint32_t kKVTileBytes = kChunks * kKVChunkBytes;
  static constexpr int kStages = (D == 128) ? 4 : 8;  // K/V ring depth
  static constexpr int kSlots = 2;
  // 8 softmax warps (warpgroups 0 and 1), then the producer warpgroup: TMA warp, MMA warp and
  // two idle warps. Three warps share each SM sub-partition's 16 K-register file, so the block
  // launches at 168 registers a thread; setmaxnreg then moves registers from the producer
  // warpgroup (whose code needs 76) to the softmax warpgroups, which would spill at 168.
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = (65536 / kThreads) & ~7;  // 168
  static constexpr int kRegsSoftmax = 208;             // per thread, warpgroups 0 and 1
  static constexpr int kRegsProducer = 80;             // per thread, warpgroup 2
  static constexpr int kRegsNeeded = 256 * kRegsSoftmax + 128 * kRegsProducer;
  static_assert(kRegsNeeded <= kThreads * kLaunchRegs, "setmaxnreg split above the launch allocation");
  static constexpr int kLoadWarp = 8;
  static constexpr int kMmaWarp = 9;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemS = 0;                // + 128 * slot
  static constexpr uint32_t kTmemO = 256;              // + 128 * slot
  static constexpr uint32_t kSmemBytes = 1024 /*align*/ + kSlots * kQTileBytes + kStages * kKVTileBytes + 512;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kCols, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
};

struct AttnParams {
  const int32_t* idx;   // [H, nqb, kmax]
  const int32_t* cnt;   // [H, nqb]
  __nv_bfloat16* o;     // [H, Nq, D]
  float* lse;           // [H, Nq] or nullptr
  unsigned* status;     // device status word
  int64_t n_q, n_kv;
  int nqb, nkb, kmax, n_items;
  float scale_log2;     // sm_scale * log2(e)
};

// Work sequence of one slot: items slot_id, slot_id + stride, ... (head-major order).
struct SlotSeq {
  int item;     // current item, or -1 when the slot is finished
  int nblk;     // kept blocks of the current item
  int ntiles;   // tiles of the current item (kept blocks / blocks per tile, rounded up)
  int n;        // current tile within the item
  int k;        // number of items started before the current one
  int h, qb;
};

__device__ __forceinline__ int clamp_count(int c, int kmax, unsigned* status, bool report) {
  if (c < 1 || c > kmax) {
    if (report) atomicOr(status, kStatusBounds);
    c = c < 1 ? 1 : kmax;
  }
  return c;
}

__device__ __forceinline__ int clamp_block(int j, int nkb, unsigned* status, bool report) {
  if (j < 0 || j >= nkb) {
    if (report) atomicOr(status, kStatusBounds);
    j = j < 0 ? 0 : nkb - 1;
  }
  return j;
}

template <int BPT>
__device__ __forceinline__ void seq_begin(SlotSeq& s, const AttnParams& p, bool report) {
  if (s.item >= p.n_items) {
    s.item = -1;
    return;
  }
  s.h = s.item / p.nqb;
  s.qb = s.item - s.h * p.nqb;
  s.nblk = clamp_count(__ldg(p.cnt + s.item), p.kmax, p.status, report);
  s.ntiles = BPT == 1 ? s.nblk : (s.nblk + BPT - 1) / BPT;
  s.n = 0;
}

template <int BPT>
__device__ __forceinline__ void seq_init(SlotSeq& s, int slot_id, const AttnParams& p, bool report) {
  s.item = slot_id;
  s.k = 0;
  seq_begin<BPT>(s, p, report);
}

// Advance to the next tile; returns true when a new item started.
template <int BPT>
__device__ __forceinline__ bool seq_next(SlotSeq& s, int stride, const AttnParams& p, bool report) {
  if (++s.n < s.ntiles) return false;
  s.item += stride;
  ++s.k;
  seq_begin<BPT>(s, p, report);
  return true;
}

// KV block of part `half` of the current tile; a part past the end of the kept list (the odd
// last entry with two blocks per tile) repeats the tile's first block.
template <int BPT>
__device__ __forceinline__ int seq_block(const SlotSeq& s, const AttnParams& p, bool report, int half = 0) {
  int e = s.n * BPT + half;
  if (BPT > 1 && e >= s.nblk) e = s.n * BPT;
  const int j = __ldg(p.idx + static_cast<int64_t>(s.item) * p.kmax + e);
  return clamp_block(j, p.nkb, p.status, report);
}

// ------------------------------------------------------------------------ softmax helpers

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Max of a (32*NC)-column S row held as NC 32-register chunks: 8 independent chains, chain i
// covering column i of every group of 8 columns (3-input max over two groups per step), then
// a short tree (dependency depth 11 instead of 128 for NC = 4).
template <int NC>
__device__ __forceinline__ float row_max(const uint32_t (&r)[NC][32]) {
  constexpr int G = 4 * NC;  // groups of 8 columns
  auto col = [&](int c) { return __uint_as_float(r[c >> 5][c & 31]); };
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = col(i);
#pragma unroll
  for (int g = 1; g + 1 < G; g += 2)
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmax3(m[i], col(8 * g + i), col(8 * g + 8 + i));
  if ((G - 1) % 2 == 1) {  // the last group has no partner
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], col(8 * (G - 1) + i));
  }
  return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

template <int D, int B = 128>
__global__ void __launch_bounds__(AttnConfig<D, B>::kThreads, 1)
    attn_sparse_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnConfig<D, B>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled tiles
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* q_tile = smem;                                   // [slot] kQTileBytes each
  uint8_t* ring = smem + C::kSlots * C::kQTileBytes;        // [stage] kKVTileBytes each
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + C::kStages * C::kKVTileBytes);
  uint64_t* full = bars;                      // [kStages] TMA -> MMA
  uint64_t* empty = full + C::kStages;        // [kStages] MMA -> TMA
  uint64_t* q_full = empty + C::kStages;      // [2]
  uint64_t* q_empty = q_full + 2;             // [2]
  uint64_t* s_full = q_empty + 2;             // [2] MMA -> softmax
  uint64_t* p_full = s_full + 2;              // [2] softmax -> MMA
  uint64_t* o_full = p_full + 2;              // [2] MMA -> softmax (end of item)
  uint64_t* drain = o_full + 2;               // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int stride = gridDim.x * C::kSlots;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&o_full[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == C::kLoadWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Each role lowers or raises its register count inside its own branch (a count changed
  // before a merge point would bind the code after it for every warp).
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegsProducer));
  if (warp == C::kLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      SlotSeq seq0, seq1;
      seq_init<C::kBlocksPerTile>(seq0, blockIdx.x * 2 + 0, p, true);
      seq_init<C::kBlocksPerTile>(seq1, blockIdx.x * 2 + 1, p, true);
      uint32_t ring_it = 0;
      int last_q_k0 = -1, last_q_k1 = -1;
      bool ok = true;
      // Q is read once per item: evicted first. K/V of the current head is re-read by every
      // query block that keeps it: kept last.
      const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();

      auto load_q = [&](int s, SlotSeq& sq, int& last_k) -> bool {
        if (!mbar_wait(&q_empty[s], (sq.k & 1) ^ 1, abort_flag, p.status)) return false;
        mbar_arrive_expect_tx(&q_full[s], C::kQTileBytes);
        const uint32_t dst = smem_u32(q_tile + s * C::kQTileBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d_hint(dst + c * C::kQChunkBytes, &tm_q, &q_full[s], c * 64, sq.qb * B, sq.h, pol_q);
        last_k = sq.k;
        return true;
      };
      auto load_kv = [&](SlotSeq& sq, const CUtensorMap* map) -> bool {
        int jb[C::kBlocksPerTile];
#pragma unroll
        for (int b = 0; b < C::kBlocksPerTile; ++b) jb[b] = seq_block<C::kBlocksPerTile>(sq, p, true, b);
        const uint32_t stage = ring_it % C::kStages;
        const uint32_t phase = (ring_it / C::kStages) & 1u;
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) return false;
        mbar_arrive_expect_tx(&full[stage], C::kKVTileBytes);
        const uint32_t dst = smem_u32(ring + stage * C::kKVTileBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
          for (int b = 0; b < C::kBlocksPerTile; ++b)
            tma_load_3d_hint(dst + c * C::kKVChunkBytes + b * C::kKVBoxBytes, map, &full[stage], c * 64, jb[b] * B,
                             sq.h, pol_kv);
        ++ring_it;
        return true;
      };
      // One step of a slot: V of its current tile, then Q (new item) and K of its next tile.
      auto step = [&](int s, SlotSeq& sq, int& last_k) {
        if (!ok || sq.item < 0) return;
        ok = load_kv(sq, &tm_v);
        if (!ok) return;
        const bool new_item = seq_next<C::kBlocksPerTile>(sq, stride, p, true);
        if (sq.item < 0) return;
        if (new_item) ok = load_q(s, sq, last_k);
        if (ok) ok = load_kv(sq, &tm_k);
      };

      if (seq0.item >= 0) ok = load_q(0, seq0, last_q_k0) && load_kv(seq0, &tm_k);
      if (ok && seq1.item >= 0) ok = load_q(1, seq1, last_q_k1) && load_kv(seq1, &tm_k);
      while (ok && (seq0.item >= 0 || seq1.item >= 0)) {
        step(0, seq0, last_q_k0);
        step(1, seq1, last_q_k1);
      }
      // Drain: wait until every load issued into a stage or Q buffer has landed, so no TMA
      // write is in flight when the CTA exits (matters only after an abort).
      for (uint32_t st = 0; st < C::kStages; ++st) {
        if (ring_it > st) {
          const uint32_t last_use = ring_it - 1 - ((ring_it - 1 - st) % C::kStages);
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[st], (last_use / C::kStages) & 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
      auto drain_q = [&](int s, int last_k) {
        if (last_k < 0) return;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&q_full[s], last_k & 1) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      };
      drain_q(0, last_q_k0);
      drain_q(1, last_q_k1);
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the schedule (waits and bookkeeping are warp-uniform, so addresses
    // and descriptors stay in uniform registers); one elected lane issues each batch of
    // tcgen05.mma / tcgen05.commit. Issue cost, not tensor time, bounds a lane-0-only loop.
    SlotSeq seq0, seq1;
    seq_init<C::kBlocksPerTile>(seq0, blockIdx.x * 2 + 0, p, false);
    seq_init<C::kBlocksPerTile>(seq1, blockIdx.x * 2 + 1, p, false);
    uint32_t ring_it = 0;
    uint32_t tiles0 = 0u, tiles1 = 0u;
    bool ok = true;
    // A descriptor's start field is addr >> 4 in 14 bits; shared-memory addresses stay below
    // 2^18, so desc(addr + off) = desc(addr) + (off >> 4) for 16-byte multiples off.
    const uint64_t q_desc = smem_desc_sw128(smem_u32(q_tile), 16, 1024);
    const uint64_t k_desc = smem_desc_sw128(smem_u32(ring), 16, 1024);
    const uint64_t v_desc = smem_desc_sw128(smem_u32(ring), C::kKVChunkBytes, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag, p.status));
    };

    // Q and K/V stages are filled by TMA: their mbarrier completion orders the tensor core's
    // reads, so no tcgen05 fence is needed after those waits.
    auto issue_s = [&](int s, const SlotSeq& sq) -> bool {
      if (sq.n == 0 && !wait_all(&q_full[s], sq.k & 1)) return false;
      const uint32_t stage = ring_it % C::kStages;
      if (!wait_all(&full[stage], (ring_it / C::kStages) & 1u)) return false;
      const uint64_t qd = q_desc + ((s * C::kQTileBytes) >> 4);
      const uint64_t kd = k_desc + ((stage * C::kKVTileBytes) >> 4);
      const uint32_t d_tmem = tmem_base + C::kTmemS + 128u * s;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = ((kk >> 2) * C::kQChunkBytes + (kk & 3) * 32) >> 4;
          const uint32_t koff = ((kk >> 2) * C::kKVChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(d_tmem, qd + qoff, kd + koff, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&empty[stage]);
        mma_commit(&s_full[s]);
        if (sq.n == sq.ntiles - 1) mma_commit(&q_empty[s]);
      }
      __syncwarp();
      ++ring_it;
      return true;
    };
    auto issue_pv = [&](int s, const SlotSeq& sq, uint32_t& tiles) -> bool {
      if (!wait_all(&p_full[s], tiles & 1u)) return false;
      ++tiles;
      const uint32_t stage = ring_it % C::kStages;
      if (!wait_all(&full[stage], (ring_it / C::kStages) & 1u)) return false;
      tc_fence_after();  // P was written by the softmax warps with tcgen05.st
      const uint64_t vd = v_desc + ((stage * C::kKVTileBytes) >> 4);
      const uint32_t d_tmem = tmem_base + C::kTmemO + 128u * s;
      const uint32_t a_tmem = tmem_base + C::kTmemS + 128u * s;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C::kCols / 16; ++kk) {
          // P columns: 16 bf16 per K step = 8 packed 32-bit columns.
          // V tile is MN-major for this MMA: 64-element chunks of d at 128*128 bytes (LBO),
          // 8-row groups of KV tokens at 1 KB (SBO); a K step of 16 tokens advances 2 KB.
          mma_ts(d_tmem, a_tmem + kk * 8, vd + ((kk * 2048) >> 4), C::kIdescPV, (sq.n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[stage]);
        if (sq.n == sq.ntiles - 1) mma_commit(&o_full[s]);
      }
      __syncwarp();
      ++ring_it;
      return true;
    };
    // One step of a slot: O += P V for its current tile, then S of its next tile.
    auto step = [&](int s, SlotSeq& sq, uint32_t& tiles) {
      if (!ok || sq.item < 0) return;
      ok = issue_pv(s, sq, tiles);
      if (!ok) return;
      seq_next<C::kBlocksPerTile>(sq, stride, p, false);
      if (sq.item < 0) return;
      ok = issue_s(s, sq);
    };

    if (seq0.item >= 0) ok = issue_s(0, seq0);
    if (ok && seq1.item >= 0) ok = issue_s(1, seq1);
    while (ok && (seq0.item >= 0 || seq1.item >= 0)) {
      step(0, seq0, tiles0);
      step(1, seq1, tiles1);
    }
    // Drain: all issued MMAs complete before TMEM is released.
    if (elect_one()) mma_commit(drain);
    __syncwarp();
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
    __syncwarp();
  }  // warps 10 and 11 only complete the warpgroup
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegsSoftmax));
    // ------------------------------------------------------------ softmax / epilogue
    const int s = warp >> 2;          // slot
    const int wq = warp & 3;          // TMEM lane quarter
    const int row = wq * 32 + lane;   // query row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + C::kTmemS + 128u * s;
    const uint32_t t_o = tmem_base + lane_off + C::kTmemO + 128u * s;
    const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
    SlotSeq seq;
    seq_init<C::kBlocksPerTile>(seq, blockIdx.x * 2 + s, p, false);
    uint32_t tiles = 0, items = 0;
    bool ok = true;
    while (ok && seq.item >= 0) {
      float m_run = -INFINITY, l_run = 0.f;
      for (int n = 0; n < seq.ntiles && ok; ++n) {
        seq.n = n;
        // valid columns of each part of the tile (a ragged last KV block; 0 for the repeated
        // half of an odd last entry)
        int n_valid[C::kBlocksPerTile];
        bool ragged = false;
#pragma unroll
        for (int b = 0; b < C::kBlocksPerTile; ++b) {
          const int j = seq_block<C::kBlocksPerTile>(seq, p, false, b);
          n_valid[b] = (j == p.nkb - 1) ? static_cast<int>(p.n_kv - static_cast<int64_t>(j) * B) : B;
          if (b > 0 && n * C::kBlocksPerTile + b >= seq.nblk) n_valid[b] = 0;
          ragged |= n_valid[b] < B;
        }
        // tcgen05.ld/st below are warp-collective: every lane must take the same path.
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[s], tiles & 1u, abort_flag, p.status))) {
          ok = false;
          break;
        }
        ++tiles;
        tc_fence_after();
        if (B < C::kRows && wq * 32 >= B) {
          // 64-token blocks: rows B..127 of the MMA tile belong to no query block and are never
          // stored, so their warps release P (whatever S left there) without a softmax
          tc_fence_before();
          mbar_arrive(&p_full[s]);
          continue;
        }
        uint32_t r[C::kSC][32];
#pragma unroll
        for (int c = 0; c < C::kSC; ++c) tmem_ld32(t_s + 32 * c, r[c]);
        tmem_wait_ld();
        if (ragged) {
#pragma unroll
          for (int c = 0; c < C::kSC; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if ((32 * c + e) % B >= n_valid[(32 * c + e) / B]) r[c][e] = __float_as_uint(-INFINITY);
        }
        const float mx_scaled = row_max<C::kSC>(r) * p.scale_log2;
        float alpha = 1.f;
        if (mx_scaled > m_run + 8.f) {
          alpha = ex2_approx(m_run - mx_scaled);  // m_run = -inf on the first tile -> 0
          l_run *= alpha;
          m_run = mx_scaled;
        }
        // O is rescaled by the whole warp when any of its rows moved its max (alpha = 1
        // leaves the other rows unchanged); the first tile overwrites O instead.
        const bool rescale = n > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.f);
        const float2 neg_m2 = make_float2(-m_run, -m_run);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < C::kSC; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(r[c][2 * e]), __uint_as_float(r[c][2 * e + 1])),
                                        scale2, neg_m2);
            const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            acc[e & 3] = __fadd2_rn(acc[e & 3], pr);
            pk[e] = pack_bf16x2(pr.x, pr.y);
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) r[c][e] = pk[e];
          if (c & 1) {
            // P: kCols bf16 = kCols/2 packed columns over the start of S; each 32-column
            // store leaves as soon as its two chunks are done (one wait for all at the end)
            uint32_t p32[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              p32[e] = r[c - 1][e];
              p32[16 + e] = r[c][e];
            }
            tmem_st32(t_s + 16 * (c - 1), p32);
          }
        }
        const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
        const float2 a = __fadd2_rn(a01, a23);
        l_run += a.x + a.y;
        if (rescale) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(t_o + 32 * c, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(t_o + 32 * c, ov);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[s]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16, lse
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&o_full[s], items & 1u, abort_flag, p.status))) break;
      ++items;
      tc_fence_after();
      const int64_t t = static_cast<int64_t>(seq.qb) * B + row;
      const bool valid = row < B && t < p.n_q;  // with B = 64, rows 64-127 belong to the next block
      const float inv_l = 1.f / l_run;
      __nv_bfloat16* orow = p.o + (static_cast<int64_t>(seq.h) * p.n_q + t) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(t_o + 32 * c, ov);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            __stcs(dst + v4, make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]));
        }
      }
      if (valid && p.lse != nullptr)
        __stcs(p.lse + static_cast<int64_t>(seq.h) * p.n_q + t, (m_run + log2f(l_run)) * 0.6931471805599453f);
      tc_fence_before();
      seq.n = seq.ntiles - 1;
      seq_next<C::kBlocksPerTile>(seq, stride, p, false);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace sparstar
