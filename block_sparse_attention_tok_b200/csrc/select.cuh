// Block selection kernels: mean pooling, block scores and per-row Top-K.
//
// Follows the SparSTAR digest ("SparSTAR的贡献：每尺度动态重建", pchao.org), section 方法概览:
// Q and KV are cut into 128-token blocks, each block is mean-pooled, every (query block,
// key block) pair gets an aggregate score from the pooled vectors, the clip-aware forced
// blocks are kept, and the rest of each row is filled by a joint Top-K, per head.
//
// Kernels (all fp32 arithmetic on bf16 inputs):
//   pool_kernel   one CTA per 128-token block: 16-byte streaming loads, fp32 sums,
//                 shuffle + shared-memory reduction, divide by the valid token count.
//   score_kernel  64x64 tiles of S = qbar kbar^T * (1/sqrt(d)) per head, fp32 FFMA with a
//                 4x4 register tile per thread.
//   topk_kernel   one CTA per (head, query block) row: order-preserving 32-bit keys,
//                 8-bit MSB radix select of the K-th largest key, ties at the threshold
//                 taken lowest index first, ascending emit after the forced prefix.
//   fill_kernel   rows that do not depend on scores (K_topk == 0 or every block kept):
//                 the row is the identity prefix 0..K_total-1.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

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
// nq_blocks may be 0 (pool K only). 256 threads.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, int64_t n_q,
                                                   int64_t n_kv, int nq_blocks, int nk_blocks,
                                                   float* __restrict__ qbar, float* __restrict__ kbar) {
  constexpr int kChunks = D / 8;           // 16-byte chunks per token row
  constexpr int kRowGroups = 256 / kChunks;
  constexpr int kRowsPerThread = 128 / kRowGroups;
  __shared__ float part[8][D];

  const int per_head = nq_blocks + nk_blocks;
  const int h = blockIdx.x / per_head;
  const int r = blockIdx.x - h * per_head;
  const __nv_bfloat16* src;
  float* dst;
  int64_t n_tok;
  int64_t b;
  if (r < nq_blocks) {
    b = r;
    n_tok = n_q;
    src = q + static_cast<int64_t>(h) * n_q * D;
    dst = qbar + (static_cast<int64_t>(h) * nq_blocks + b) * D;
  } else {
    b = r - nq_blocks;
    n_tok = n_kv;
    src = k + static_cast<int64_t>(h) * n_kv * D;
    dst = kbar + (static_cast<int64_t>(h) * nk_blocks + b) * D;
  }
  const int64_t row0 = b * 128;
  const int n_valid = static_cast<int>(min(static_cast<int64_t>(128), n_tok - row0));
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
    dst[threadIdx.x] = s / static_cast<float>(n_valid);
  }
}

// ------------------------------------------------------------------------ scores

// grid = (ceil(nkb/64), ceil(nqb/64), H); 256 threads; dynamic smem 2*64*(D+4) floats.
template <int D>
__global__ void __launch_bounds__(256) score_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                    int nqb, int nkb, float inv_sqrt_d, float* __restrict__ S) {
  constexpr int LD = D + 4;
  extern __shared__ __align__(16) float smem_f[];
  float* qs = smem_f;
  float* ks = smem_f + 64 * LD;
  const int h = blockIdx.z;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const float* qh = qbar + static_cast<int64_t>(h) * nqb * D;
  const float* kh = kbar + static_cast<int64_t>(h) * nkb * D;
  constexpr int kVec = 64 * D / 4;
  for (int e = threadIdx.x; e < kVec; e += 256) {
    const int row = e / (D / 4), c4 = e % (D / 4);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (i0 + row < nqb) a = *reinterpret_cast<const float4*>(qh + static_cast<int64_t>(i0 + row) * D + c4 * 4);
    if (j0 + row < nkb) b = *reinterpret_cast<const float4*>(kh + static_cast<int64_t>(j0 + row) * D + c4 * 4);
    *reinterpret_cast<float4*>(qs + row * LD + c4 * 4) = a;
    *reinterpret_cast<float4*>(ks + row * LD + c4 * 4) = b;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 4
  for (int c = 0; c < D; c += 4) {
    float4 av[4], bv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) av[a] = *reinterpret_cast<const float4*>(qs + (ty + 16 * a) * LD + c);
#pragma unroll
    for (int b = 0; b < 4; ++b) bv[b] = *reinterpret_cast<const float4*>(ks + (tx + 16 * b) * LD + c);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        acc[a][b] = fmaf(av[a].x, bv[b].x, acc[a][b]);
        acc[a][b] = fmaf(av[a].y, bv[b].y, acc[a][b]);
        acc[a][b] = fmaf(av[a].z, bv[b].z, acc[a][b]);
        acc[a][b] = fmaf(av[a].w, bv[b].w, acc[a][b]);
      }
  }
  float* Sh = S + static_cast<int64_t>(h) * nqb * nkb;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i >= nqb) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + tx + 16 * b;
      if (j < nkb) Sh[static_cast<int64_t>(i) * nkb + j] = acc[a][b] * inv_sqrt_d;
    }
  }
}

// ------------------------------------------------------------------------ Top-K

// Order-preserving key: larger score -> larger key; -0.0 maps like +0.0; NaN ranks last.
__device__ __forceinline__ uint32_t score_key(float s) {
  if (s != s) return 0u;
  if (s == 0.0f) s = 0.0f;
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
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

}  // namespace sparstar
