// Retained attention mass of a block mask and its token-wise upper bound, for sm_100a.
//
// The analysis of the SparSTAR digest ("SparSTAR的贡献：每尺度动态重建", pchao.org), section
// 关键结果与论文证据, bullet 跨尺度复用损失 (Figure 3): how much of the dense softmax mass a
// per-scale block Top-K keeps, against the best any choice of the same number of key tokens
// could keep.
//
//   * retained mass of query token t: R_t = sum over kept tokens u of P_tu, where P is the
//     dense softmax of row t; R_t = exp(lse_kept(t) - lse_dense(t)). Averaged over the valid
//     rows of a query block it is the block energy of eq. (5) of the CalibAtt notes
//     ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention",
//     papernotes.org, section 关键设计 1), summed over the kept key blocks.
//   * token-wise bound: U_t = the sum of the B largest P_tu over all valid key tokens, with
//     B = the number of valid key tokens in the kept blocks of t's query block.
//
// mass_kernel computes R and its block means from the two LSEs. The bound needs the dense
// logits again: bound_pass_kernel recomputes S = Q K^T for every (query block, key block)
// tile on the tensor cores (TMA -> tcgen05.mma -> tensor memory) and bins x = log2 P_tu of
// each row into 32 equal bins of a per-row interval. The first three passes only count: after
// each, the row keeps the bin holding its B-th largest value as the next interval and takes
// the count of the bins above it off B. The last pass sums P over every value above the final
// interval (width 64/32^4 = 2^-14 in log2 units) in registers, bins the few values inside it
// by count and mass, and takes the boundary bin's mean for the still missing values
// (relative error below 2^-15 * ln 2 of U). Bins are cells of one fixed grid:
// y = log2 P + 64 is rounded the same way in every pass, and the bin of pass p is
// floor(y * 2^(5p-1)) (an exact power-of-two scaling), so a value's cell in pass p+1 always
// lies inside its cell of pass p and no value is counted twice or lost at a bin edge.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparstar {

constexpr int kBoundBins = 32;
constexpr int kBoundPasses = 4;
constexpr float kBoundLo = -64.0f;  // log2 P below 2^-64 never matters for a bound on mass
constexpr float kBoundYTop = 63.999996185302734f;  // the largest float below 64 (= -kBoundLo)
constexpr uint32_t kBoundMagicBits = 0x4B400000u;   // bit pattern of 1.5 * 2^23
// Count histograms per thread in the counting passes: value e of a group of 8 updates histogram
// e % kBoundSubs, so four read-modify-writes are independent (no shared-memory address can
// repeat among them). Counts are 16-bit: a histogram gets 16 values a tile, so up to
// kBoundMaxKvBlocks tiles never overflow one.
constexpr int kBoundSubs = 4;
constexpr int kBoundMaxKvBlocks = 65535 / 16;
constexpr uint32_t kBoundCells = kBoundBins + 2;  // the interval's bins and two cells outside it
// Last pass, inside a warp's region: a 32-bit count histogram [bin][lane] at 0 and the fp32
// mass histogram [bin][lane] from here.
constexpr uint32_t kBoundMassOffset = kBoundBins * 32 * 4;

// 1 / bin width of a pass: widths 2, 1/16, 1/512, 1/16384 (pass 0 covers [-64, 0) in 32 bins)
__device__ __forceinline__ float bound_inv_width(int pass) {
  return static_cast<float>(1u << (5 * pass)) * 0.5f;
}

// R_t and the per-block means. One CTA of 128 threads per (query block, head).
__global__ void __launch_bounds__(128) mass_kernel(const float* __restrict__ lse_kept, const float* __restrict__ lse_dense,
                                                   int64_t n_q, int nqb, float* __restrict__ r_token,
                                                   float* __restrict__ e_block) {
  __shared__ float part[4];
  const int qb = blockIdx.x, h = blockIdx.y;
  const int64_t t = static_cast<int64_t>(qb) * 128 + threadIdx.x;
  const bool valid = t < n_q;
  float r = 0.f;
  if (valid) {
    const int64_t o = static_cast<int64_t>(h) * n_q + t;
    r = expf(lse_kept[o] - lse_dense[o]);
    if (r_token != nullptr) r_token[o] = r;
  }
  float s = r;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    const int64_t n_valid = n_q - static_cast<int64_t>(qb) * 128 < 128 ? n_q - static_cast<int64_t>(qb) * 128 : 128;
    e_block[static_cast<int64_t>(h) * nqb + qb] = (part[0] + part[1] + part[2] + part[3]) / static_cast<float>(n_valid);
  }
}

// Per-row state of the bound passes ([H, n_q] each).
struct BoundState {
  int* lo_idx;        // interval start of the current pass, in that pass's bin widths from -64
  int* need;          // B minus the values already counted above the interval
  float* above_sum;   // mass of the values counted above the interval
  float* u;           // result (written by the last pass)
};

// B per row from the mask, and the initial state. One CTA of 128 threads per (query block, head).
__global__ void __launch_bounds__(128) bound_init_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                                                         int kmax, int64_t n_q, int64_t n_kv, int nqb, BoundState st,
                                                         unsigned* status) {
  __shared__ int budget;
  const int qb = blockIdx.x, h = blockIdx.y;
  const int64_t row = static_cast<int64_t>(h) * nqb + qb;
  const int nkb = static_cast<int>((n_kv + 127) / 128);
  if (threadIdx.x == 0) {
    int c = cnt[row];
    if (c < 0 || c > kmax) {
      atomicOr(status, kStatusBounds);
      c = c < 0 ? 0 : kmax;
    }
    int64_t b = 0;
    for (int e = 0; e < c; ++e) {
      int j = idx[row * kmax + e];
      if (j < 0 || j >= nkb) {
        atomicOr(status, kStatusBounds);
        continue;
      }
      b += (j == nkb - 1) ? n_kv - static_cast<int64_t>(j) * 128 : 128;
    }
    budget = static_cast<int>(b);
  }
  __syncthreads();
  const int64_t t = static_cast<int64_t>(qb) * 128 + threadIdx.x;
  if (t < n_q) {
    const int64_t o = static_cast<int64_t>(h) * n_q + t;
    st.lo_idx[o] = 0;
    st.need[o] = budget;
    st.above_sum[o] = 0.f;
  }
}

template <int D>
struct BoundConfig {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kChunkBytes = 128 * 128;
  static constexpr uint32_t kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kThreads = 320;  // 8 binning warps + TMA warp + MMA warp
  static constexpr int kLoadWarp = 8;
  static constexpr int kMmaWarp = 9;
  static constexpr uint32_t kTmemCols = 256;  // S0, S1
  // Per binning warp: kBoundSubs 16-bit count histograms [sub][bin + junk][lane] (the last pass
  // reuses the region for one count histogram and a fp32 mass histogram); then 128 floats for
  // the second half's row sums.
  static constexpr uint32_t kWarpHistBytes = kBoundSubs * kBoundCells * 32 * 2;
  static constexpr uint32_t kHistBytes = 8 * kWarpHistBytes + 128 * 4;
  static constexpr uint32_t kSmemBytes = 1024 + kTileBytes + kStages * kTileBytes + kHistBytes + 256;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false);
};

struct BoundParams {
  BoundState st;
  const float* lse_dense;  // [H, n_q], natural log
  float* u_block;          // [H, nqb] (last pass)
  unsigned* status;
  int64_t n_q, n_kv;
  int nqb, nkb, n_items, pass;
  float scale_log2;        // sm_scale * log2(e)
};

// One pass over every (head, query block) item; each item visits all key blocks.
template <int D>
__global__ void __launch_bounds__(BoundConfig<D>::kThreads, 1)
    bound_pass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const BoundParams p) {
  using C = BoundConfig<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* q_tile = smem;
  uint8_t* ring = smem + C::kTileBytes;
  uint8_t* hist = ring + C::kStages * C::kTileBytes;                                 // [8][kWarpHistBytes]
  float* above_part = reinterpret_cast<float*>(hist + 8 * C::kWarpHistBytes);        // [128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(above_part + 128);
  uint64_t* full = bars;                // [kStages]
  uint64_t* empty = full + C::kStages;  // [kStages]
  uint64_t* q_full = empty + C::kStages;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_empty + 1;       // [2]
  uint64_t* s_free = s_full + 2;        // [2], 256 arrivals
  uint64_t* drain = s_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 256);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == C::kLoadWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == C::kLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t ring_it = 0;
      int k = 0, q_loads = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++k) {
        const int h = item / p.nqb, qb = item - h * p.nqb;
        if (!mbar_wait(q_empty, (k & 1) ^ 1, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(q_full, C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) tma_load_3d(smem_u32(q_tile) + c * C::kChunkBytes, &tm_q, q_full, c * 64, qb * 128, h);
        ++q_loads;
        for (int j = 0; j < p.nkb; ++j) {
          const uint32_t stage = ring_it % C::kStages;
          if (!mbar_wait(&empty[stage], ((ring_it / C::kStages) & 1u) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::kTileBytes);
          const uint32_t dst = smem_u32(ring + stage * C::kTileBytes);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) tma_load_3d(dst + c * C::kChunkBytes, &tm_k, &full[stage], c * 64, j * 128, h);
          ++ring_it;
        }
      }
      // Drain: every issued load lands before the CTA exits (matters only after an abort).
      for (uint32_t s = 0; s < C::kStages; ++s) {
        if (ring_it > s) {
          const uint32_t last_use = ring_it - 1 - ((ring_it - 1 - s) % C::kStages);
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s], (last_use / C::kStages) & 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
      if (q_loads > 0) {
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(q_full, (q_loads - 1) & 1) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (whole warp, elected lane)
    uint32_t ring_it = 0, tile = 0;
    bool ok = true;
    const uint64_t q_desc = smem_desc_sw128(smem_u32(q_tile), 16, 1024);
    const uint64_t k_desc = smem_desc_sw128(smem_u32(ring), 16, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag, p.status));
    };
    int k = 0;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++k) {
      if (!wait_all(q_full, k & 1)) break;
      for (int j = 0; j < p.nkb; ++j, ++tile) {
        const uint32_t b = tile & 1u;
        // S buffer b is free once the binning warps have read S(tile - 2)
        if (tile >= 2 && !wait_all(&s_free[b], ((tile >> 1) - 1) & 1u)) {
          ok = false;
          break;
        }
        const uint32_t stage = ring_it % C::kStages;
        if (!wait_all(&full[stage], (ring_it / C::kStages) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t kd = k_desc + ((stage * C::kTileBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * C::kChunkBytes + (kk & 3) * 32) >> 4;
            mma_ss(tmem_base + 128u * b, q_desc + off, kd + off, C::kIdescQK, kk > 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          mma_commit(&s_full[b]);
          if (j == p.nkb - 1) mma_commit(q_empty);
        }
        __syncwarp();
        ++ring_it;
      }
    }
    if (elect_one()) mma_commit(drain);
    __syncwarp();
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ binning warps
    // Warps w and w+4 share TMEM lane quarter w%4 (32 query rows); warp w bins key columns
    // 0-63 of each S tile, warp w+4 columns 64-127, each into its own histograms.
    //   passes 0 .. kBoundPasses-2: counts only, in 34 cells: cells 1..32 are the interval's
    //     bins, cell 0 holds values one bin below it and cell 33 every other value outside it;
    //   last pass: every value above the interval adds its P to a register sum, values inside
    //     the interval go to count + mass bins (a handful per row), the rest is skipped.
    const int wq = warp & 3, half = warp >> 2;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint8_t* my_hist = hist + warp * C::kWarpHistBytes + lane * 2;    // [sub][cell][lane] u16
    uint32_t* hn32 = reinterpret_cast<uint32_t*>(hist + warp * C::kWarpHistBytes) + lane;  // last pass
    float* hm = reinterpret_cast<float*>(hist + warp * C::kWarpHistBytes + kBoundMassOffset) + lane;
    static_assert(kBoundMassOffset + kBoundBins * 32 * 4 <= C::kWarpHistBytes, "last-pass histograms overflow");
    constexpr uint32_t kCellBytes = 32 * 2;                              // one cell of all 32 lanes
    constexpr uint32_t kSubBytes = kBoundCells * kCellBytes;
    const float inv_w = bound_inv_width(p.pass);
    const bool last_pass = p.pass == kBoundPasses - 1;
    const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
    const float2 w2 = make_float2(inv_w, inv_w);
    uint32_t tile = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      const int h = item / p.nqb, qb = item - h * p.nqb;
      const int64_t t = static_cast<int64_t>(qb) * 128 + row;
      const bool valid_row = t < p.n_q;
      const int64_t o = static_cast<int64_t>(h) * p.n_q + (valid_row ? t : 0);
      const int lo_idx = valid_row ? p.st.lo_idx[o] : 0;
      const int need_in = valid_row ? p.st.need[o] : 0;
      // need < 0: fewer values above 2^-64 than B, so all of them are in the top B
      const bool take_all = need_in < 0;
      // y = s * scale_log2 + (64 - lse * log2 e): the same rounding in every pass
      const float y_off = (valid_row ? -p.lse_dense[o] * 1.4426950408889634f : 0.f) - kBoundLo;
      const float2 off2 = make_float2(y_off, y_off);
      // Interval of this pass in y: [lo_idx, lo_idx + 32) / inv_w (exact: powers of two, lo_idx < 2^21).
      // y is held below 64 (the top cell of every pass keeps a value at or above 2^0 by rounding).
      const float lo_f = static_cast<float>(lo_idx);
      const float y_top = (lo_f + static_cast<float>(kBoundBins)) / inv_w;  // the interval's top
      const float y_in = lo_f / inv_w;              // the interval's bottom
      // cell - 1 = floor(y * inv_w - lo_idx) = bits(y * inv_w + 1.5 * 2^23 - lo_idx, rounded down) - bits(1.5 * 2^23)
      const float magic = 12582912.0f - lo_f;   // exact integer
      const float2 magic2 = make_float2(magic, magic);

#pragma unroll 4
      for (int bb = 0; bb < kBoundSubs * kBoundCells; ++bb) *reinterpret_cast<uint16_t*>(my_hist + bb * kCellBytes) = 0u;
      float above = 0.f;   // last pass: P summed over the values above the interval
      const float y_above = take_all ? 0.f : y_top;  // take_all: every value above 2^-64
      for (int j = 0; j < p.nkb; ++j, ++tile) {
        const uint32_t b = tile & 1u;
        const int n_valid = (j == p.nkb - 1) ? static_cast<int>(p.n_kv - static_cast<int64_t>(j) * 128) : 128;
        const int cols = n_valid - 64 * half;  // valid columns of this half (may be <= 0)
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[b], (tile >> 1) & 1u, abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[2][32];
        const uint32_t ts = tmem_base + lane_off + 128u * b + 64u * half;
        tmem_ld32(ts, r[0]);
        tmem_ld32(ts + 32, r[1]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&s_free[b]);  // S is in registers: the buffer may be overwritten
        if (cols < 64) {  // a ragged last KV block: invalid columns become -inf (below every interval)
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * c + e >= cols) r[c][e] = 0xFF800000u;
        }
        if (!last_pass) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int e0 = 0; e0 < 32; e0 += kBoundSubs) {
              // value e0 + u goes to histogram u: the four loads, then the four stores
              // cell = bin + 1 = bits(tm) - bits(1.5 * 2^23) + 1; a value below the interval by more
              // than a bin gives a smaller (or negative) tm, whose difference wraps above 33
              uint32_t off[kBoundSubs];
#pragma unroll
              for (int u = 0; u < kBoundSubs; u += 2) {
                const int e = e0 + u;
                float2 yy = __ffma2_rn(make_float2(__uint_as_float(r[c][e]), __uint_as_float(r[c][e + 1])), scale2, off2);
                yy = make_float2(fminf(yy.x, kBoundYTop), fminf(yy.y, kBoundYTop));
                const float2 tm = __ffma2_rd(yy, w2, magic2);
                const uint32_t c0 = min(__float_as_uint(tm.x) - (kBoundMagicBits - 1u), kBoundCells - 1u);
                const uint32_t c1 = min(__float_as_uint(tm.y) - (kBoundMagicBits - 1u), kBoundCells - 1u);
                off[u] = c0 * kCellBytes + u * kSubBytes;
                off[u + 1] = c1 * kCellBytes + (u + 1) * kSubBytes;
              }
              uint32_t cnt[kBoundSubs];
#pragma unroll
              for (int u = 0; u < kBoundSubs; ++u) cnt[u] = *reinterpret_cast<const uint16_t*>(my_hist + off[u]);
#pragma unroll
              for (int u = 0; u < kBoundSubs; ++u) *reinterpret_cast<uint16_t*>(my_hist + off[u]) = static_cast<uint16_t>(cnt[u] + 1u);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              float yv[8];
              bool any_in = false;
#pragma unroll
              for (int e2 = 0; e2 < 8; e2 += 2) {
                const int e = 8 * g + e2;
                const float2 yy = __ffma2_rn(make_float2(__uint_as_float(r[c][e]), __uint_as_float(r[c][e + 1])), scale2, off2);
                yv[e2] = fminf(yy.x, kBoundYTop);
                yv[e2 + 1] = fminf(yy.y, kBoundYTop);
                const float2 xx = __fadd2_rn(yy, make_float2(kBoundLo, kBoundLo));  // log2 P
                above += (yv[e2] >= y_above ? ex2_approx(xx.x) : 0.f) + (yv[e2 + 1] >= y_above ? ex2_approx(xx.y) : 0.f);
                any_in |= (yv[e2] >= y_in && yv[e2] < y_top) | (yv[e2 + 1] >= y_in && yv[e2 + 1] < y_top);
              }
              if (!__any_sync(0xFFFFFFFFu, any_in && !take_all)) continue;
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const bool in = !take_all && yv[e] >= y_in && yv[e] < y_top;
                const int bi = in ? static_cast<int>(__float_as_uint(__fmaf_rd(yv[e], inv_w, magic)) - kBoundMagicBits) : 0;
                hn32[bi * 32] += in ? 1u : 0u;
                hm[bi * 32] += in ? ex2_approx(yv[e] + kBoundLo) : 0.f;
              }
            }
          }
        }
      }
      // Both halves of every row are binned: combine and move the interval. The two warps of
      // a lane quarter reach both named barriers on every path (an aborted wait only ends
      // the tile loop early), so neither can be left waiting at one.
      if (last_pass && half == 1) above_part[row] = above;
      asm volatile("bar.sync %0, %1;" ::"r"(1 + wq), "r"(64) : "memory");
      if (ok && half == 0 && valid_row) {
        // the partner warp (w + 4) of this lane quarter binned the row's other 64 columns
        const uint8_t* other = my_hist + 4 * C::kWarpHistBytes;
        const uint32_t* hn32_2 = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(hn32) + 4 * C::kWarpHistBytes);
        const float* hm2 = reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(hm) + 4 * C::kWarpHistBytes);
        int need = need_in;
        if (!last_pass) {
          if (need > 0) {
            int bin = kBoundBins - 1;
            for (; bin >= 0; --bin) {  // bin b of the interval is cell b + 1
              int nb = 0;
              for (int u = 0; u < kBoundSubs; ++u) {
                const uint32_t at = u * kSubBytes + (bin + 1) * kCellBytes;
                nb += *reinterpret_cast<const uint16_t*>(my_hist + at) + *reinterpret_cast<const uint16_t*>(other + at);
              }
              if (nb >= need) break;
              need -= nb;
            }
            if (bin >= 0) {
              p.st.lo_idx[o] = (lo_idx + bin) * kBoundBins;  // that bin, in the next pass's widths
              p.st.need[o] = need;
            } else {
              p.st.need[o] = -1;  // only reachable in pass 0: fewer values above 2^-64 than B
            }
          }
        } else {
          float u = above + above_part[row];
          if (!take_all && need == 0) u = 0.f;  // an empty mask (B = 0) bounds nothing
          if (!take_all && need > 0) {
            for (int bin = kBoundBins - 1; bin >= 0; --bin) {
              const int nb = static_cast<int>(hn32[bin * 32] + hn32_2[bin * 32]);
              const float mb = hm[bin * 32] + hm2[bin * 32];
              if (nb >= need) {  // the boundary bin's mean stands in for its top `need` values
                u += mb * (static_cast<float>(need) / static_cast<float>(nb));
                break;
              }
              need -= nb;
              u += mb;
            }
          }
          p.st.u[o] = u;
        }
      }
      asm volatile("bar.sync %0, %1;" ::"r"(1 + wq), "r"(64) : "memory");  // histograms reused next item
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Block means of the bound. One CTA of 128 threads per (query block, head).
__global__ void __launch_bounds__(128) bound_block_kernel(const float* __restrict__ u, int64_t n_q, int nqb,
                                                          float* __restrict__ u_token, float* __restrict__ u_block) {
  __shared__ float part[4];
  const int qb = blockIdx.x, h = blockIdx.y;
  const int64_t t = static_cast<int64_t>(qb) * 128 + threadIdx.x;
  float s = 0.f;
  if (t < n_q) {
    const int64_t o = static_cast<int64_t>(h) * n_q + t;
    s = u[o];
    if (u_token != nullptr) u_token[o] = s;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    const int64_t n_valid = n_q - static_cast<int64_t>(qb) * 128 < 128 ? n_q - static_cast<int64_t>(qb) * 128 : 128;
    u_block[static_cast<int64_t>(h) * nqb + qb] = (part[0] + part[1] + part[2] + part[3]) / static_cast<float>(n_valid);
  }
}

}  // namespace sparstar
