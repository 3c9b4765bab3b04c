// Block selection kernels: mean pooling, block scores and per-row Top-K.
//
// Follows the SparSTAR digest ("SparSTAR的贡献：每尺度动态重建", pchao.org), section 方法概览:
// Q and KV are cut into 128-token blocks, each block is mean-pooled, every (query block,
// key block) pair gets an aggregate score from the pooled vectors, the clip-aware forced
// blocks are kept, and the rest of each row is filled by a joint Top-K, per head. The block
// size is a template parameter (128, or 64 for the block-size variant of the pages'
// ablation, section 实验如何设计?, bullet on supplementary experiments).
//
// Kernels:
//   pool_kernel      one CTA per block: 16-byte streaming loads, fp32 sums, shuffle +
//                    shared-memory reduction, divide by the valid token count; the mean m is
//                    stored as two bf16 numbers hi = bf16(m), lo = bf16(m - hi).
//   score_tc_kernel  S = qbar kbar^T / sqrt(d) on the tensor cores: persistent CTAs over
//                    128 x 128 tiles of (query block, KV block) pairs, TMA-fed,
//                    tcgen05.mma accumulating hi.hi + hi.lo + lo.hi in fp32 tensor memory.
//                    Error bound: hi = bf16(m), lo = bf16(m - hi) leave e = m - hi - lo with
//                    |e| <= 2^-16 |m| and |lo| <= 2^-8 |m|, so each dropped term (hi_q e_k,
//                    e_q k, lo_q lo_k) is at most about 2^-16 |q_c k_c|; with the fp32
//                    accumulation of 3d products the error stays below
//                    2^-14 sum_c |qbar_c kbar_c| / sqrt(d), far inside the 1e-3 tie gap.
//   topk_warp_kernel one warp per (head, query block) row, staged in shared memory with
//                    16-byte copies, each lane owning a contiguous run: the K-th largest key
//                    is bracketed by a value histogram, then resolved among <= 32 keys
//                    (a rank count or a warp bitonic sort); ties taken lowest index first;
//                    each lane marks its taken candidates in a bit mask, one warp scan places
//                    the runs and the row leaves with coalesced stores.
//   topk_kernel      one CTA per row, 8-bit radix select in shared memory (rows with more than
//                    3965 candidates).
//   fill_kernel      rows that do not depend on scores (K_topk == 0 or every block kept):
//                    the row is the identity prefix 0..K_total-1.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sparstar {

// ------------------------------------------------------------------------ pooling

__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// grid.x = H * (nq_blocks + nk_blocks) (Q blocks of a head first, then its K blocks);
// nq_blocks may be 0 (pool K only). 256 threads. Outputs [H, n_blocks, D] bf16 hi and lo.
template <int D, int B = 128>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, int64_t n_q,
                                                   int64_t n_kv, int nq_blocks, int nk_blocks,
                                                   __nv_bfloat16* __restrict__ q_hi, __nv_bfloat16* __restrict__ q_lo,
                                                   __nv_bfloat16* __restrict__ k_hi, __nv_bfloat16* __restrict__ k_lo) {
  constexpr int kChunks = D / 8;           // 16-byte chunks per token row
  constexpr int kRowGroups = 256 / kChunks;
  constexpr int kRowsPerThread = B / kRowGroups;  // B = tokens per block (128, or 64)
  __shared__ float part[8][D];
  griddep_launch_dependents();  // the score kernel may be scheduled early; it waits for this grid

  const int per_head = nq_blocks + nk_blocks;
  const int h = blockIdx.x / per_head;
  const int r = blockIdx.x - h * per_head;
  const __nv_bfloat16* src;
  __nv_bfloat16 *dst_hi, *dst_lo;
  int64_t n_tok;
  int64_t b;
  if (r < nq_blocks) {
    b = r;
    n_tok = n_q;
    src = q + static_cast<int64_t>(h) * n_q * D;
    const int64_t o = (static_cast<int64_t>(h) * nq_blocks + b) * D;
    dst_hi = q_hi + o;
    dst_lo = q_lo + o;
  } else {
    b = r - nq_blocks;
    n_tok = n_kv;
    src = k + static_cast<int64_t>(h) * n_kv * D;
    const int64_t o = (static_cast<int64_t>(h) * nk_blocks + b) * D;
    dst_hi = k_hi + o;
    dst_lo = k_lo + o;
  }
  const int64_t row0 = b * B;
  const int n_valid = static_cast<int>(min(static_cast<int64_t>(B), n_tok - row0));
  const int c = threadIdx.x % kChunks;
  const int rg = threadIdx.x / kChunks;

  uint4 v[kRowsPerThread];
#pragma unroll
  for (int m = 0; m < kRowsPerThread; ++m) {
    const int rr = rg + m * kRowGroups;
    if (rr < n_valid)
      v[m] = ld_stream_16(src + (row0 + rr) * D + c * 8);
    else
      v[m] = make_uint4(0u, 0u, 0u, 0u);
  }
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < kRowsPerThread; ++m) add_bf16x8(acc, v[m]);
#pragma unroll
  for (int off = kChunks; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xFFFFFFFFu, acc[e], off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < kChunks)
#pragma unroll
    for (int e = 0; e < 8; ++e) part[warp][lane * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += part[w][threadIdx.x];
    const float m = s / static_cast<float>(n_valid);
    const __nv_bfloat16 hi = __float2bfloat16_rn(m);
    dst_hi[threadIdx.x] = hi;
    dst_lo[threadIdx.x] = __float2bfloat16_rn(m - __bfloat162float(hi));
  }
}

// Measurement aid: one read of n16 16-byte chunks with the pooling kernel's streaming loads
// (grid-stride, four loads in flight per thread), XOR-folded so the loads are not dead code,
// one atomicXor per warp into *sink. Its rate is the read-only streaming bandwidth.
__global__ void __launch_bounds__(512) read_probe_kernel(const uint4* __restrict__ src, int64_t n16,
                                                         unsigned* __restrict__ sink) {
  uint32_t acc = 0u;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ld_stream_16(src + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = ld_stream_16(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc ^= __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

// ------------------------------------------------------------------------ scores

template <int D>
struct ScoreConfig {
  static constexpr int kChunks = D / 64;                    // 128-byte swizzle chunks per row
  static constexpr uint32_t kChunkBytes = 128 * 128;        // 128 rows x 128 B
  static constexpr uint32_t kTileBytes = kChunks * kChunkBytes;  // hi (or lo) of 128 block means
  static constexpr int kStages = 2;                         // K (hi + lo) ring
  static constexpr int kThreads = 192;                      // TMA warp, MMA warp, 4 epilogue warps
  static constexpr int kStageRow = 65;                      // floats per staged row (64 + pad)
  static constexpr uint32_t kStageBytes = 4 * 32 * kStageRow * 4;   // per epilogue warp: 32 rows x 64
  static constexpr uint32_t kSmemBytes = 1024 + 2 * kTileBytes + kStages * 2 * kTileBytes + kStageBytes + 256;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false);
  static constexpr uint32_t kTmemCols = 256;                // two 128-column accumulators
};

// S = qbar kbar^T / sqrt(d) for every (head, 128 query blocks, 128 KV blocks) tile, as
// hi.hi + hi.lo + lo.hi bf16 products (fp32 accumulation in tensor memory). Persistent: CTA c
// takes a contiguous run of tiles in (head, query tile, KV tile) order, so consecutive tiles
// share the query tile, which stays in shared memory; KV tiles stream through a two-stage
// TMA ring while the previous tile's epilogue runs on the other accumulator. The epilogue
// thread of each row takes the row out of tensor memory, frees the accumulator and writes
// the row with 16-byte stores when rows of S are 16-byte aligned (nkb a multiple of 4);
// otherwise it goes through a padded staging buffer and coalesced 4-byte row stores.
// Out-of-range rows load as zero and are not stored.
template <int D>
__global__ void __launch_bounds__(ScoreConfig<D>::kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_ql,
                    const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_kl,
                    float* __restrict__ S, int heads, int nqb, int nkb, float inv_sqrt_d, unsigned* status) {
  using C = ScoreConfig<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* q_s = smem;                                // [hi | lo]
  uint8_t* k_s = smem + 2 * C::kTileBytes;            // [stage][hi | lo]
  float* stage_buf = reinterpret_cast<float*>(k_s + C::kStages * 2 * C::kTileBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stage_buf) + C::kStageBytes);
  uint64_t* full = bars;                  // [kStages]
  uint64_t* empty = full + C::kStages;    // [kStages]
  uint64_t* q_full = empty + C::kStages;
  uint64_t* q_empty = q_full + 1;
  uint64_t* acc_full = q_empty + 1;       // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2], 128 arrivals
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int n_mt = (nqb + 127) / 128, n_nt = (nkb + 127) / 128;
  const int n_tiles = heads * n_mt * n_nt;
  const int per_cta = (n_tiles + gridDim.x - 1) / gridDim.x;
  const int t_begin = blockIdx.x * per_cta;
  const int t_end = min(n_tiles, t_begin + per_cta);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // pooled means come from the preceding pool kernel

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int q_key = -1, q_loads = 0;
      uint32_t ring_it = 0;
      for (int t = t_begin; t < t_end; ++t) {
        const int nt = t % n_nt, hm = t / n_nt, mt = hm % n_mt, h = hm / n_mt;
        if (hm != q_key) {  // a new query tile: once the MMAs of the previous one are done
          if (!mbar_wait(q_empty, (q_loads & 1) ^ 1, abort_flag, status)) break;
          mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            tma_load_3d(smem_u32(q_s) + c * C::kChunkBytes, &tm_qh, q_full, c * 64, mt * 128, h);
            tma_load_3d(smem_u32(q_s) + C::kTileBytes + c * C::kChunkBytes, &tm_ql, q_full, c * 64, mt * 128, h);
          }
          q_key = hm;
          ++q_loads;
        }
        const uint32_t st = ring_it % C::kStages;
        if (!mbar_wait(&empty[st], ((ring_it / C::kStages) & 1u) ^ 1u, abort_flag, status)) break;
        mbar_arrive_expect_tx(&full[st], 2 * C::kTileBytes);
        const uint32_t dst = smem_u32(k_s) + st * 2 * C::kTileBytes;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(dst + c * C::kChunkBytes, &tm_kh, &full[st], c * 64, nt * 128, h);
          tma_load_3d(dst + C::kTileBytes + c * C::kChunkBytes, &tm_kl, &full[st], c * 64, nt * 128, h);
        }
        ++ring_it;
      }
      // Drain: every issued load lands before the CTA exits (matters only after an abort).
      for (uint32_t s2 = 0; s2 < C::kStages; ++s2) {
        if (ring_it > s2) {
          const uint32_t last_use = ring_it - 1 - ((ring_it - 1 - s2) % C::kStages);
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s2], (last_use / C::kStages) & 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp, elected lane)
    const uint64_t qh_d = smem_desc_sw128(smem_u32(q_s), 16, 1024);
    const uint64_t ql_d = qh_d + (C::kTileBytes >> 4);
    const uint64_t k_d = smem_desc_sw128(smem_u32(k_s), 16, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag, status));
    };
    int q_key = -1, q_loads = 0;
    uint32_t ring_it = 0, acc_it = 0;
    for (int t = t_begin; t < t_end; ++t, ++acc_it) {
      const int hm = t / n_nt;
      if (hm != q_key) {
        if (!wait_all(q_full, q_loads & 1)) break;
        q_key = hm;
        ++q_loads;
      }
      const uint32_t a = acc_it & 1u;
      if (acc_it >= 2 && !wait_all(&acc_empty[a], ((acc_it >> 1) - 1) & 1u)) break;
      const uint32_t st = ring_it % C::kStages;
      if (!wait_all(&full[st], (ring_it / C::kStages) & 1u)) break;
      tc_fence_after();
      const uint64_t kh_d = k_d + ((st * 2 * C::kTileBytes) >> 4);
      const uint64_t kl_d = kh_d + (C::kTileBytes >> 4);
      const bool last_of_q = (t + 1 == t_end) || ((t + 1) / n_nt != hm);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(tmem + 128u * a, qh_d + off, kh_d + off, C::kIdesc, kk > 0 ? 1u : 0u);
          mma_ss(tmem + 128u * a, qh_d + off, kl_d + off, C::kIdesc, 1u);
          mma_ss(tmem + 128u * a, ql_d + off, kh_d + off, C::kIdesc, 1u);
        }
        mma_commit(&empty[st]);
        mma_commit(&acc_full[a]);
        if (last_of_q) mma_commit(q_empty);
      }
      __syncwarp();
      ++ring_it;
    }
    if (elect_one()) mma_commit(drain);
    __syncwarp();
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int wq = warp & 3;                 // TMEM lane quarter: rows 32*wq .. 32*wq + 31
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float* stg = stage_buf + (warp - 2) * 32 * C::kStageRow;
    uint32_t acc_it = 0;
    for (int t = t_begin; t < t_end; ++t, ++acc_it) {
      const int nt = t % n_nt, hm = t / n_nt, mt = hm % n_mt, h = hm / n_mt;
      const uint32_t a = acc_it & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[a], (acc_it >> 1) & 1u, abort_flag, status))) break;
      tc_fence_after();
      const int j0 = nt * 128;
      const int n_cols = min(128, nkb - j0);
      const int i_base = mt * 128 + wq * 32;
      if ((nkb & 3) == 0) {
        // Rows of S are 16-byte aligned. Each lane takes its whole row (128 columns) out of
        // tensor memory and frees the accumulator; then, 32 columns at a time, the warp's
        // 32 rows pass through the staging buffer (row stride 36 floats: the row-wise 16-byte
        // writes and the line-wise reads are both free of bank conflicts) and every store
        // instruction writes four whole 128-byte row lines.
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + 128u * a + 32u * c, r[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&acc_empty[a]);
        constexpr int kRow4 = 9;  // float4 per staged row
        float4* st4 = reinterpret_cast<float4*>(stg);
        const int sub = lane >> 3, chunk = lane & 7;
#pragma unroll
        for (int qc = 0; qc < 4; ++qc) {
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4)
            st4[lane * kRow4 + c4] =
                make_float4(__uint_as_float(r[qc][4 * c4]) * inv_sqrt_d, __uint_as_float(r[qc][4 * c4 + 1]) * inv_sqrt_d,
                            __uint_as_float(r[qc][4 * c4 + 2]) * inv_sqrt_d,
                            __uint_as_float(r[qc][4 * c4 + 3]) * inv_sqrt_d);
          __syncwarp();
          const int col = 32 * qc + 4 * chunk;
          if (col < n_cols) {  // n_cols is a multiple of 4 here
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
              const int rr = 4 * s8 + sub;
              const int i = i_base + rr;
              if (i < nqb)
                *reinterpret_cast<float4*>(S + (static_cast<int64_t>(h) * nqb + i) * nkb + j0 + col) =
                    st4[rr * kRow4 + chunk];
            }
          }
          __syncwarp();
        }
        continue;
      }
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t r[2][32];
        tmem_ld32(tmem + lane_off + 128u * a + 64u * half, r[0]);
        tmem_ld32(tmem + lane_off + 128u * a + 64u * half + 32u, r[1]);
        tmem_wait_ld();
        if (half == 1) {  // the accumulator is in registers: the MMA may reuse it
          tc_fence_before();
          mbar_arrive(&acc_empty[a]);
        }
        // lane = row: stage this warp's 32 rows x 64 columns (row stride 65 floats, so both
        // the row-wise writes here and the column-wise reads below hit 32 distinct banks)
        float* my_row = stg + lane * C::kStageRow;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) my_row[32 * c + e] = __uint_as_float(r[c][e]) * inv_sqrt_d;
        __syncwarp();
        const int col0 = 64 * half;
#pragma unroll 4
        for (int rr = 0; rr < 32; ++rr) {
          const int i = i_base + rr;
          if (i >= nqb) break;
          float* srow = S + (static_cast<int64_t>(h) * nqb + i) * nkb + j0 + col0;
          const float* src = stg + rr * C::kStageRow;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int col = lane + 32 * cc;
            if (col0 + col < n_cols) srow[col] = src[col];
          }
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------ scores across scales

// Latent grid of a scale's current tokens, raster order (frame, row, column).
struct GridDims {
  int64_t t, h, w;
};

// Block of the previous scale's grid that holds the nearest raster position of block b of the
// current grid: b's middle token c = start + (n - 1) / 2 is unravelled on `now`, each axis x of
// size X' goes to the old cell (2x + 1) X / (2 X') (clipped to X - 1), and the old token is
// ravelled on `prev` and divided by the block size. All integer arithmetic.
__device__ __forceinline__ int64_t raster_block(int64_t b, int64_t n_now, const GridDims& now, const GridDims& prev,
                                                int block) {
  const int64_t s = b * block;
  const int64_t e = min(s + block, n_now);
  const int64_t c = s + (e - s - 1) / 2;
  const int64_t hw = now.h * now.w;
  const int64_t t = c / hw, rem = c - t * hw;
  const int64_t h = rem / now.w, w = rem - h * now.w;
  const int64_t to = min(prev.t - 1, (2 * t + 1) * prev.t / (2 * now.t));
  const int64_t ho = min(prev.h - 1, (2 * h + 1) * prev.h / (2 * now.h));
  const int64_t wo = min(prev.w - 1, (2 * w + 1) * prev.w / (2 * now.w));
  return ((to * prev.h + ho) * prev.w + wo) / block;
}

constexpr int kMapRowsPerCta = 8;

// S_now[h, i, j] = S_prev[h, m(i), c(j)] with m = raster_block (query blocks are current-scale
// blocks) and c(j) = j on the KV prefix (text and reference blocks, the same tokens at every
// scale), n_prefix + m(j - n_prefix) on the current-scale blocks. grid = (ceil(nqb_now / 8),
// heads), 256 threads; the column map (nkb_now ints) is built once per CTA in shared memory.
__global__ void __launch_bounds__(256) map_scores_kernel(const float* __restrict__ s_prev, float* __restrict__ s_now,
                                                         int nqb_prev, int nkb_prev, int nqb_now, int nkb_now,
                                                         int n_prefix, int64_t n_now, GridDims now, GridDims prev) {
  extern __shared__ int col_map[];
  for (int j = threadIdx.x; j < nkb_now; j += blockDim.x)
    col_map[j] = j < n_prefix ? j : n_prefix + static_cast<int>(raster_block(j - n_prefix, n_now, now, prev, 128));
  __syncthreads();
  const int h = blockIdx.y;
  const int i0 = blockIdx.x * kMapRowsPerCta;
  const int i1 = min(nqb_now, i0 + kMapRowsPerCta);
  for (int i = i0; i < i1; ++i) {
    const int mi = static_cast<int>(raster_block(i, n_now, now, prev, 128));
    const float* src = s_prev + (static_cast<int64_t>(h) * nqb_prev + mi) * nkb_prev;
    float* dst = s_now + (static_cast<int64_t>(h) * nqb_now + i) * nkb_now;
    for (int j = threadIdx.x; j < nkb_now; j += blockDim.x) dst[j] = __ldg(src + col_map[j]);
  }
}

// ------------------------------------------------------------------------ Top-K

// Order-preserving key: larger score -> larger key; -0.0 maps like +0.0; NaN ranks last.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = s == 0.0f ? 0u : __float_as_uint(s);  // -0.0 -> +0.0
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return s != s ? 0u : k;
}

// Exclusive prefix sum over the 128 threads of the block (4 warps); returns the total too.
__device__ __forceinline__ uint32_t block_exclusive_scan_128(uint32_t v, uint32_t* warp_tot, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, inc, off);
    if (lane >= off) inc += n;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  uint32_t before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t t = warp_tot[w];
    if (w < warp) before += t;
    total += t;
  }
  return before + inc - v;
}

// One CTA (128 threads) per row; grid.x = H * nqb. Dynamic smem: n_cand keys.
// Requires 1 <= k_topk < n_cand (other rows go through fill_kernel).
__global__ void __launch_bounds__(128) topk_kernel(const float* __restrict__ S, int nkb, int n_forced, int k_topk,
                                                   int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                                                   int kmax) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[4];
  __shared__ uint32_t s_digit, s_krem;
  const int n_cand = nkb - n_forced;
  const int64_t row = blockIdx.x;
  const float* srow = S + row * nkb + n_forced;
  griddep_wait();  // scores come from the preceding score kernel
  for (int j = threadIdx.x; j < n_cand; j += 128) keys[j] = score_key(srow[j]);

  uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k_topk);
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[threadIdx.x] = 0u;
    hist[threadIdx.x + 128] = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < n_cand; j += 128) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255-8l down to 248-8l (descending order)
      const int lane = threadIdx.x;
      uint32_t c[8], local = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[255 - 8 * lane - e];
        local += c[e];
      }
      uint32_t inc = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, inc, off);
        if (lane >= off) inc += n;
      }
      uint32_t before = inc - local;  // keys with a larger digit than this lane's range
      if (before < krem && krem <= inc) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (before + c[e] >= krem) {
            s_digit = static_cast<uint32_t>(255 - 8 * lane - e);
            s_krem = krem - before;
            break;
          }
          before += c[e];
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    krem = s_krem;
    __syncthreads();
  }
  const uint32_t T = prefix;  // key of the K-th largest; take `krem` of the keys equal to T

  const int chunk = (n_cand + 127) / 128;
  const int j0 = threadIdx.x * chunk;
  const int j1 = min(j0 + chunk, n_cand);
  uint32_t n_eq = 0;
  for (int j = j0; j < j1; ++j) n_eq += (keys[j] == T);
  uint32_t total;
  const uint32_t eq_before = block_exclusive_scan_128(n_eq, warp_tot, total);
  uint32_t n_sel = 0, eq_seen = eq_before;
  for (int j = j0; j < j1; ++j) {
    const uint32_t key = keys[j];
    if (key > T) {
      ++n_sel;
    } else if (key == T) {
      if (eq_seen < krem) ++n_sel;
      ++eq_seen;
    }
  }
  const uint32_t sel_before = block_exclusive_scan_128(n_sel, warp_tot, total);
  int32_t* out = idx + row * kmax;
  for (int f = threadIdx.x; f < n_forced; f += 128) out[f] = f;
  uint32_t pos = static_cast<uint32_t>(n_forced) + sel_before;
  const uint32_t row_end = static_cast<uint32_t>(n_forced + k_topk);  // never write past the row
  eq_seen = eq_before;
  for (int j = j0; j < j1; ++j) {
    const uint32_t key = keys[j];
    bool take = key > T;
    if (key == T) {
      take = eq_seen < krem;
      ++eq_seen;
    }
    if (take && pos < row_end) out[pos++] = n_forced + j;
  }
  if (threadIdx.x == 0) cnt[row] = n_forced + k_topk;
}

// Rows equal to the identity prefix 0..k_total-1; grid.x = rows, 128 threads.
__global__ void __launch_bounds__(128) fill_kernel(int k_total, int32_t* __restrict__ idx,
                                                   int32_t* __restrict__ cnt, int kmax) {
  const int64_t row = blockIdx.x;
  for (int c = threadIdx.x; c < k_total; c += 128) idx[row * kmax + c] = c;
  if (threadIdx.x == 0) cnt[row] = k_total;
}

// Top-K of one row by one warp. The row is staged in shared memory (`sv`, 32*KPL floats,
// NaN past the row) and lane l owns the contiguous candidates [l*KPL, (l+1)*KPL), read as
// float4. The K-th largest key T is located in steps, all exact:
//   1. the row's score range (NaN ignored);
//   2. the range is split into 256 equal-width bins (binning is monotone in the score, so
//      every key of a higher bin is larger than every key of a lower one; NaN and the
//      padding go to bin 0, the padding is then taken out of its count); a per-warp
//      histogram and a warp scan give the bin b* holding the K-th largest key and the
//      count of keys above it; each candidate's bin is kept, four to a word;
//   3. while the set in question (first b*) holds more than 32 keys, it is narrowed by a
//      histogram over 256 sub-ranges of its ranking keys;
//   4. the set's <= 32 keys are gathered (per-lane counts, one warp scan) and ranked (a
//      count over the set when it holds at most 12 keys, else a warp bitonic sort); T is
//      read off it, with the number of keys > T and == T;
//   5. each lane marks its taken candidates in a bit mask (every key > T and, of the keys
//      == T, the lowest-index ones); one warp scan of the counts places each lane's run in
//      the staging buffer, in index order, and the row leaves with coalesced stores.
// Keys: NaN ranks below every number; -0.0 equals +0.0. `hist` holds 256 words, `gat` 32
// (the set's keys), `binw` 8*KPL words (the packed bins).
__device__ __forceinline__ uint32_t rank_key(float x) { return x != x ? 1u : max(score_key(x), 2u); }

// The number whose ranking key is k (k >= 2; the key of zero gives +0.0).
__device__ __forceinline__ float key_number(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Bin of the need-th largest key (need >= 1) from a 256-bin histogram, scanning from bin 255
// down; lane l owns bins 255-8l .. 248-8l. Returns the bin, the count of keys above it and
// the count inside it (warp-uniform).
__device__ __forceinline__ void find_bin_desc(const uint32_t* hist, uint32_t need, uint32_t& bin, uint32_t& above,
                                              uint32_t& inside) {
  const int lane = threadIdx.x & 31;
  const uint32_t full = 0xFFFFFFFFu;
  uint32_t cnt[8], local = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    cnt[e] = hist[255 - 8 * lane - e];
    local += cnt[e];
  }
  uint32_t inc = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(full, inc, off);
    if (lane >= off) inc += n;
  }
  uint32_t before = inc - local;
  const bool owner = before < need && need <= inc;
  uint32_t b_l = 0, a_l = 0, i_l = 0;
  if (owner) {
    bool done = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (!done && before + cnt[e] >= need) {
        b_l = 255u - 8u * lane - e;
        a_l = before;
        i_l = cnt[e];
        done = true;
      }
      before += cnt[e];
    }
  }
  const int src = __ffs(__ballot_sync(full, owner)) - 1;
  bin = __shfl_sync(full, b_l, src);
  above = __shfl_sync(full, a_l, src);
  inside = __shfl_sync(full, i_l, src);
}

__device__ __forceinline__ uint32_t warp_exclusive_scan(uint32_t v, uint32_t& total) {
  const int lane = threadIdx.x & 31;
  uint32_t inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, inc, off);
    if (lane >= off) inc += n;
  }
  total = __shfl_sync(0xFFFFFFFFu, inc, 31);
  return inc - v;
}

template <int KPL>
__device__ __forceinline__ void topk_row_warp(const float* __restrict__ cand, int n_cand, int n_forced, int k_topk,
                                              int32_t* __restrict__ out, float* sv, uint32_t* hist, uint32_t* gat,
                                              uint32_t* binw) {
  static_assert(KPL % 4 == 0 && KPL <= 128, "keys per lane: a multiple of 4, at most 128 (two take words)");
  constexpr int Q = KPL / 4;  // float4 groups per lane
  const int lane = threadIdx.x & 31;
  const uint32_t full = 0xFFFFFFFFu;
  const uint32_t K = static_cast<uint32_t>(k_topk);
  // Stage the row at slot offset dl = (cand mod 16 bytes) / 4, so that whole 16-byte chunks
  // inside the row move with one copy each; the ragged first and last chunks move element by
  // element and every slot outside the row holds NaN. Candidate j sits in slot j + dl
  // (requires dl + n_cand <= 32 * KPL).
  const int dl = static_cast<int>((reinterpret_cast<uintptr_t>(cand) >> 2) & 3u);
  const float* base = cand - dl;  // 16-byte aligned
#pragma unroll
  for (int u = 0; u < Q; ++u) {
    const int c = lane + 32 * u;  // chunk: slots 4c .. 4c+3
    const int j = 4 * c - dl;     // candidate in its first slot
    if (j >= 0 && j + 3 < n_cand) {
      asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_u32(sv + 4 * c)), "l"(base + 4 * c)
                   : "memory");
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (j + e >= 0 && j + e < n_cand)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(sv + 4 * c + e)),
                       "l"(base + 4 * c + e)
                       : "memory");
        else
          sv[4 * c + e] = __uint_as_float(0x7FC00000u);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) hist[lane * 8 + e] = 0u;
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncwarp();
  const float4* my = reinterpret_cast<const float4*>(sv) + lane * Q;
  uint32_t* myb = binw + lane * Q;
  const int j0 = lane * KPL - dl;  // candidate index of this lane's first slot
  // 1. score range (fminf/fmaxf skip NaN)
  float lo0 = INFINITY, lo1 = INFINITY, hi0 = -INFINITY, hi1 = -INFINITY;
#pragma unroll 3
  for (int g = 0; g < Q; ++g) {
    const float4 v = my[g];
    lo0 = fminf(lo0, fminf(v.x, v.y));
    lo1 = fminf(lo1, fminf(v.z, v.w));
    hi0 = fmaxf(hi0, fmaxf(v.x, v.y));
    hi1 = fmaxf(hi1, fmaxf(v.z, v.w));
  }
  float smin = fminf(lo0, lo1), smax = fmaxf(hi0, hi1);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    smin = fminf(smin, __shfl_xor_sync(full, smin, off));
    smax = fmaxf(smax, __shfl_xor_sync(full, smax, off));
  }
  // 2. value bins: f = fma(x, scale, offset) clamped to [0, 255] (NaN -> 0) and rounded to
  // nearest by adding 1.5 * 2^23 (the integer lands in the low byte); monotone in x.
  // First try: bins 1..255 over the upper half [mid, max] of the range and bin 0 for every
  // key below it, NaN and the padding (bin 0 is not counted). If fewer than K keys reach
  // bin 1, the K-th largest lies below mid: bin the whole range [min, max] into 0..255
  // instead, the padding taken out of bin 0 afterwards. A range that is empty, constant or
  // not finite puts every key in bin 0 of the second form and leaves the work to step 3.
  auto bin_bits = [](float x, float sc, float of) -> uint32_t {
    const float f = fminf(fmaxf(fmaf(x, sc, of), 0.f), 255.f);
    return __float_as_uint(__fadd_rn(f, 12582912.0f));  // bin in the low byte
  };
  const float mid = 0.5f * smin + 0.5f * smax;
  float scale = 255.f / (smax - mid);
  float offset = 1.f - mid * scale;
  const bool split_ok = smax > mid && mid > smin && fabsf(scale) <= 3.0e38f && fabsf(offset) <= 3.0e38f;
  uint32_t bstar = 0, c_hi = 0, nb = 0;
  bool found = false;
  if (split_ok) {
    __syncwarp();
#pragma unroll 3
    for (int g = 0; g < Q; ++g) {
      const float4 v = my[g];
      const uint32_t b0 = bin_bits(v.x, scale, offset), b1 = bin_bits(v.y, scale, offset);
      const uint32_t b2 = bin_bits(v.z, scale, offset), b3 = bin_bits(v.w, scale, offset);
      if (b0 & 0xFFu) atomicAdd(&hist[b0 & 0xFFu], 1u);
      if (b1 & 0xFFu) atomicAdd(&hist[b1 & 0xFFu], 1u);
      if (b2 & 0xFFu) atomicAdd(&hist[b2 & 0xFFu], 1u);
      if (b3 & 0xFFu) atomicAdd(&hist[b3 & 0xFFu], 1u);
      myb[g] = __byte_perm(__byte_perm(b0, b1, 0x0040u), __byte_perm(b2, b3, 0x0040u), 0x5410u);
    }
    __syncwarp();
    uint32_t upper = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) upper += hist[lane * 8 + e];
    upper = __reduce_add_sync(full, upper);
    if (upper >= K) {
      find_bin_desc(hist, K, bstar, c_hi, nb);
      found = true;
    }
  }
  if (!found) {
    scale = 256.f / (smax - smin);
    offset = -smin * scale;
    if (!(smax > smin) || !(fabsf(scale) <= 3.0e38f) || !(fabsf(offset) <= 3.0e38f)) {
      scale = 0.f;
      offset = 0.f;
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 8; ++e) hist[lane * 8 + e] = 0u;
    __syncwarp();
#pragma unroll 3
    for (int g = 0; g < Q; ++g) {
      const float4 v = my[g];
      const uint32_t b0 = bin_bits(v.x, scale, offset), b1 = bin_bits(v.y, scale, offset);
      const uint32_t b2 = bin_bits(v.z, scale, offset), b3 = bin_bits(v.w, scale, offset);
      atomicAdd(&hist[b0 & 0xFFu], 1u);
      atomicAdd(&hist[b1 & 0xFFu], 1u);
      atomicAdd(&hist[b2 & 0xFFu], 1u);
      atomicAdd(&hist[b3 & 0xFFu], 1u);
      myb[g] = __byte_perm(__byte_perm(b0, b1, 0x0040u), __byte_perm(b2, b3, 0x0040u), 0x5410u);
    }
    __syncwarp();
    if (lane == 0) hist[0] -= static_cast<uint32_t>(32 * KPL - n_cand);  // the padding
    __syncwarp();
    find_bin_desc(hist, K, bstar, c_hi, nb);
  }
  uint32_t need = K - c_hi;  // 1 <= need <= nb
  auto valid = [&](int j) { return j >= 0 && j < n_cand; };
  // 3. narrow the set while it holds more than 32 keys: the set's ranking keys span
  // [klo, khi); each round splits that span into at most 256 sub-ranges of 2^s keys.
  bool by_key = false;
  uint32_t klo = 0;
  uint64_t khi = 0;
  if (nb > 32u) {
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
    for (int i = 0; i < KPL; ++i) {
      if (valid(j0 + i) && ((myb[i >> 2] >> (8 * (i & 3))) & 0xFFu) == bstar) {
        const uint32_t k = rank_key(sv[lane * KPL + i]);
        mn = min(mn, k);
        mx = max(mx, k);
      }
    }
    klo = __reduce_min_sync(full, mn);
    khi = static_cast<uint64_t>(__reduce_max_sync(full, mx)) + 1u;
    by_key = true;
    while (nb > 32u && khi - klo > 1u) {
      const uint64_t span = khi - klo;
      const int bits = 64 - __clzll(static_cast<long long>(span - 1u));
      const int s = bits > 8 ? bits - 8 : 0;
      __syncwarp();
#pragma unroll
      for (int e = 0; e < 8; ++e) hist[lane * 8 + e] = 0u;
      __syncwarp();
      for (int i = 0; i < KPL; ++i) {
        const uint32_t k = rank_key(sv[lane * KPL + i]);
        if (valid(j0 + i) && k >= klo && static_cast<uint64_t>(k) < khi) atomicAdd(&hist[(k - klo) >> s], 1u);
      }
      __syncwarp();
      uint32_t b2, a2, n2;
      find_bin_desc(hist, need, b2, a2, n2);
      const uint64_t kb = klo;
      klo = static_cast<uint32_t>(kb + (static_cast<uint64_t>(b2) << s));
      const uint64_t top = kb + (static_cast<uint64_t>(b2 + 1u) << s);
      khi = top < khi ? top : khi;
      c_hi += a2;
      need -= a2;
      nb = n2;
    }
  }
  // 4. T = the need-th largest key of the set: its <= 32 keys are gathered (each lane counts
  // its members, a warp scan places them), then ranked (a count over the set when it is small,
  // else a warp bitonic sort).
  uint32_t T, gt_set, eq_set;
  if (by_key && khi - klo == 1u) {
    T = klo;  // every key of the set is equal
    gt_set = 0;
    eq_set = nb;
  } else {
    auto member = [&](int i) -> bool {
      if (!valid(j0 + i)) return false;
      if (by_key) {
        const uint32_t k = rank_key(sv[lane * KPL + i]);
        return k >= klo && static_cast<uint64_t>(k) < khi;
      }
      return ((myb[i >> 2] >> (8 * (i & 3))) & 0xFFu) == bstar;
    };
    const uint32_t rep = bstar * 0x01010101u;
    // bins can be matched four at a time unless the padding (bin 0 of the whole-range
    // binning) could be among the matches
    const bool by_word = !by_key && bstar != 0u;
    uint32_t n_mine = 0;
    if (by_word) {
#pragma unroll 3
      for (int g = 0; g < Q; ++g) n_mine += __popc(__vcmpeq4(myb[g], rep)) >> 3;
    } else {
      for (int i = 0; i < KPL; ++i) n_mine += member(i) ? 1u : 0u;
    }
    uint32_t n_all;
    uint32_t at = warp_exclusive_scan(n_mine, n_all);
    if (by_word) {
#pragma unroll 3
      for (int g = 0; g < Q; ++g) {
        uint32_t m = __vcmpeq4(myb[g], rep);  // 0xFF in each byte whose bin is b*
        while (m != 0u) {
          const int e = (__ffs(m) - 1) >> 3;
          m &= ~(0xFFu << (8 * e));
          gat[at++] = rank_key(sv[lane * KPL + 4 * g + e]);
        }
      }
    } else if (n_mine != 0u) {
      for (int i = 0; i < KPL; ++i)
        if (member(i)) gat[at++] = rank_key(sv[lane * KPL + i]);
    }
    __syncwarp();
    const bool in_set = lane < static_cast<int>(nb);
    uint32_t g = in_set ? gat[lane] : 0u;
    if (nb <= 12u) {
      // rank = keys above this one, equal keys at lower lanes counted as above
      uint32_t rank = 0;
      for (int m = 0; m < static_cast<int>(nb); ++m) {
        const uint32_t o = __shfl_sync(full, g, m);
        rank += (o > g || (o == g && m < lane)) ? 1u : 0u;
      }
      const uint32_t hit = __ballot_sync(full, in_set && rank == need - 1u);
      T = __shfl_sync(full, g, __ffs(hit) - 1);
    } else {
#pragma unroll
      for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
          const uint32_t other = __shfl_xor_sync(full, g, jj);
          const bool descending_block = (lane & kk) == 0;
          const bool first = (lane & jj) == 0;
          g = (first == descending_block) ? max(g, other) : min(g, other);
        }
      }
      T = __shfl_sync(full, g, static_cast<int>(need) - 1);
    }
    gt_set = __popc(__ballot_sync(full, in_set && g > T));
    eq_set = __popc(__ballot_sync(full, in_set && g == T));
  }
  const uint32_t need_eq = need - gt_set;  // keys == T to take, 1 <= need_eq <= eq_set
  // 5. mark the taken candidates of this lane, then write them in index order
  uint64_t take0 = 0, take1 = 0;  // bit i of take0 / take1: candidate j0 + i / j0 + 64 + i taken
  if (need_eq == eq_set && T >= 2u) {
    // every key == T is taken and T is a number: take x >= T (NaN and padding compare false)
    const float tf = key_number(T);
#pragma unroll 3
    for (int g = 0; g < Q; ++g) {
      const float4 v = my[g];
      const uint64_t m4 = (v.x >= tf ? 1u : 0u) | (v.y >= tf ? 2u : 0u) | (v.z >= tf ? 4u : 0u) | (v.w >= tf ? 8u : 0u);
      if (4 * g < 64)
        take0 |= m4 << (4 * g);
      else
        take1 |= m4 << (4 * g - 64);
    }
  } else {
    uint32_t n_eq = 0;
    for (int i = 0; i < KPL; ++i) n_eq += (valid(j0 + i) && rank_key(sv[lane * KPL + i]) == T) ? 1u : 0u;
    uint32_t eq_total;
    uint32_t eq_rank = warp_exclusive_scan(n_eq, eq_total);
    for (int i = 0; i < KPL; ++i) {
      if (!valid(j0 + i)) continue;
      const uint32_t k = rank_key(sv[lane * KPL + i]);
      bool t = k > T;
      if (k == T) {
        t = eq_rank < need_eq;
        ++eq_rank;
      }
      if (t) {
        if (i < 64)
          take0 |= 1ull << i;
        else
          take1 |= 1ull << (i - 64);
      }
    }
  }
  // each lane's taken candidates go to its run in the (now free) staging buffer, then the
  // row leaves with coalesced stores
  for (int f = lane; f < n_forced; f += 32) out[f] = f;
  uint32_t n_take = __popcll(take0) + __popcll(take1), total;
  uint32_t pos = warp_exclusive_scan(n_take, total);
  int32_t* ordered = reinterpret_cast<int32_t*>(sv);
  __syncwarp();
#pragma unroll
  for (int w = 0; w < (KPL > 64 ? 2 : 1); ++w) {
    uint64_t take = w == 0 ? take0 : take1;
    while (take != 0ull) {
      const int i = __ffsll(static_cast<long long>(take)) - 1 + 64 * w;
      take &= take - 1ull;
      if (pos < K) ordered[pos] = n_forced + j0 + i;
      ++pos;
    }
  }
  __syncwarp();
  for (uint32_t p = lane; p < K; p += 32) out[n_forced + p] = ordered[p];
}

// One warp per row, topk_cta_warps(KPL) rows per CTA (two for the longest rows, so that the
// static shared memory stays under 48 KB); grid.x = ceil(H * nqb / topk_cta_warps(KPL)).
// Requires 1 <= k_topk < n_cand and n_cand + 3 <= 32 * KPL (room for the row's slot offset).
__host__ __device__ constexpr int topk_cta_warps(int kpl) { return kpl > 64 ? 2 : 4; }

template <int KPL>
struct TopkSmem {
  static constexpr int kW = topk_cta_warps(KPL);
  alignas(16) float sv[kW][32 * KPL];
  uint32_t binw[kW][8 * KPL];
  uint32_t hist[kW][256];
  uint32_t gat[kW][32];
};

template <int KPL>
__global__ void __launch_bounds__(32 * topk_cta_warps(KPL)) topk_warp_kernel(const float* __restrict__ S,
                                                                             int64_t rows, int nkb, int n_forced,
                                                                             int k_topk, int32_t* __restrict__ idx,
                                                                             int32_t* __restrict__ cnt, int kmax) {
  __shared__ TopkSmem<KPL> sm;
  const int w = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * topk_cta_warps(KPL) + w;
  griddep_wait();  // scores come from the preceding score kernel
  if (row >= rows) return;
  topk_row_warp<KPL>(S + row * nkb + n_forced, nkb - n_forced, n_forced, k_topk, idx + row * kmax, sm.sv[w],
                     sm.hist[w], sm.gat[w], sm.binw[w]);
  if ((threadIdx.x & 31) == 0) cnt[row] = n_forced + k_topk;
}

}  // namespace sparstar
