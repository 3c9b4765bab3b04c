// Host side of the C ABI declared in include/sparstar.h, and the single translation unit
// that instantiates every kernel of the library.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "sparstar.h"
#include "attn_sm100.cuh"
#include "mass_sm100.cuh"
#include "select.cuh"

namespace sparstar {

// Per-device status word: bit kStatusTimeout / kStatusBounds, set by kernels, read by
// sparstar_device_status(). A __device__ variable exists once per device that loads the
// library, so no allocation is needed.
__device__ unsigned g_status = 0u;

// Self-test of the bounded wait: one thread waits, with the library's mbar_wait, on an
// mbarrier that nothing ever completes. The wait ends at its time limit, raises the CTA's
// abort flag and records a timeout in the status word; the kernel then returns normally.
__global__ void wait_timeout_selftest_kernel(unsigned* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, &abort_flag, status);
}

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxCandidates = 16384;  // Top-K keys held in shared memory (64 KB)
constexpr int64_t kMaxMapColumns = 49152;  // columns of a mapped score row (192 KB column map)

struct DeviceInfo {
  bool ready = false;
  int major = 0, minor = 0, sms = 0;
  unsigned* status = nullptr;
  bool attrs_set = false;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SPARSTAR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SPARSTAR_ERR_CUDA;
    d.major = prop.major;
    d.minor = prop.minor;
    d.sms = prop.multiProcessorCount;
    void* sym = nullptr;
    if (cudaGetSymbolAddress(&sym, g_status) != cudaSuccess) return SPARSTAR_ERR_CUDA;
    d.status = static_cast<unsigned*>(sym);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return SPARSTAR_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return SPARSTAR_OK;
}

int set_kernel_attrs(DeviceInfo* d) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (d->attrs_set) return SPARSTAR_OK;
  bool ok = true;
  ok &= cudaFuncSetAttribute(attn_sparse_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnConfig<128>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(attn_sparse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnConfig<64>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(attn_sparse_kernel<128, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnConfig<128, 64>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(attn_sparse_kernel<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnConfig<64, 64>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(bound_pass_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BoundConfig<128>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(bound_pass_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BoundConfig<64>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(score_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ScoreConfig<128>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(score_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ScoreConfig<64>::kSmemBytes) == cudaSuccess;
  ok &= cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kMaxCandidates * 4)) == cudaSuccess;
  ok &= cudaFuncSetAttribute(map_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kMaxMapColumns * 4)) == cudaSuccess;
  if (!ok) return SPARSTAR_ERR_CUDA;
  // The attention kernels raise the softmax warps' registers with setmaxnreg, drawing on the
  // block's launch allocation; a build that launched with fewer registers would wait there
  // for good, so such a build is refused before any launch.
  auto regs_ok = [](auto kernel, int threads, int needed) {
    cudaFuncAttributes a;
    return cudaFuncGetAttributes(&a, kernel) == cudaSuccess && a.numRegs * threads >= needed;
  };
  if (!regs_ok(attn_sparse_kernel<128>, AttnConfig<128>::kThreads, AttnConfig<128>::kRegsNeeded) ||
      !regs_ok(attn_sparse_kernel<64>, AttnConfig<64>::kThreads, AttnConfig<64>::kRegsNeeded) ||
      !regs_ok(attn_sparse_kernel<128, 64>, AttnConfig<128, 64>::kThreads, AttnConfig<128, 64>::kRegsNeeded) ||
      !regs_ok(attn_sparse_kernel<64, 64>, AttnConfig<64, 64>::kThreads, AttnConfig<64, 64>::kRegsNeeded))
    return SPARSTAR_ERR_UNSUPPORTED;
  d->attrs_set = true;
  return SPARSTAR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_blocks(int64_t n, int64_t block = SPARSTAR_BLOCK) { return (n + block - 1) / block; }
bool valid_block(int block) { return block == 64 || block == 128; }

// ceil(x) with a 1e-9 guard, so that a product such as 0.1875 * 16 = 3.0 stays 3.
int64_t ceil_guarded(double x) { return static_cast<int64_t>(std::ceil(x - 1e-9)); }

bool valid_segments(const sparstar_segments& s) { return s.n_text >= 0 && s.n_ctx >= 0 && s.n_cur >= 0; }

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

int launch_status() { return cudaGetLastError() == cudaSuccess ? SPARSTAR_OK : SPARSTAR_ERR_CUDA; }

// Workspace: [q_hi | q_lo] [k_hi | k_lo] [scores]: the block means as bf16 hi/lo pairs
// ([H, n_blocks, d] each) and the fp32 score matrix [H, nqb, nkb].
struct Workspace {
  size_t q_hi, q_lo, k_hi, k_lo, scores, total;
};

Workspace workspace_layout(int heads, int64_t nqb, int64_t nkb, int d, bool need_scores) {
  Workspace w;
  const size_t qb = static_cast<size_t>(heads) * nqb * d * 2, kb = static_cast<size_t>(heads) * nkb * d * 2;
  w.q_hi = 0;
  w.q_lo = align256(qb);
  w.k_hi = w.q_lo + align256(qb);
  w.k_lo = w.k_hi + align256(kb);
  w.scores = w.k_lo + align256(kb);
  w.total = w.scores + (need_scores ? align256(static_cast<size_t>(heads) * nqb * nkb * sizeof(float)) : 0);
  return w;
}

// Launch with programmatic stream serialization: the kernel may be scheduled while the
// previous kernel of the stream drains; it calls griddep_wait() before reading that
// kernel's output.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Keys per lane of the warp Top-K: the smallest supported count that covers n_cand
// candidates, or 0 when the shared-memory radix kernel has to be used.
int topk_keys_per_lane(int64_t n_cand) {
  for (int kpl : {8, 16, 24, 36, 48, 64, 76, 124})
    if (n_cand <= 32 * kpl) return kpl;
  return 0;
}

// Top-K of `rows` score rows of nkb columns (1 <= k_topk < nkb - n_forced <= kMaxCandidates):
// one warp per row up to 3965 candidates, else one CTA per row. Launched with programmatic
// stream serialization, so it may start while a preceding score kernel drains.
void launch_topk(const float* S, int64_t rows, int nkb, int n_forced, int k_topk, int32_t* idx, int32_t* cnt,
                 int kmax, cudaStream_t st) {
  auto warp_kernel = [&](auto kernel, int kpl) {
    const int w = topk_cta_warps(kpl);
    launch_after(kernel, dim3(static_cast<unsigned>((rows + w - 1) / w)), dim3(32 * w), 0, st, S, rows, nkb, n_forced,
                 k_topk, idx, cnt, kmax);
  };
  switch (topk_keys_per_lane(nkb - n_forced + 3)) {  // + the staging slot offset (<= 3)
    case 8: warp_kernel(topk_warp_kernel<8>, 8); break;
    case 16: warp_kernel(topk_warp_kernel<16>, 16); break;
    case 24: warp_kernel(topk_warp_kernel<24>, 24); break;
    case 36: warp_kernel(topk_warp_kernel<36>, 36); break;
    case 48: warp_kernel(topk_warp_kernel<48>, 48); break;
    case 64: warp_kernel(topk_warp_kernel<64>, 64); break;
    case 76: warp_kernel(topk_warp_kernel<76>, 76); break;
    case 124: warp_kernel(topk_warp_kernel<124>, 124); break;
    default:
      launch_after(topk_kernel, dim3(static_cast<unsigned>(rows)), dim3(128),
                   static_cast<size_t>(nkb - n_forced) * 4, st, S, nkb, n_forced, k_topk, idx, cnt, kmax);
  }
}

int make_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, unsigned box_rows = 128) {
  // 3-D view [heads][rows][d] of bf16; box = 64 elements x box_rows rows x 1 head, 128B swizzle.
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SPARSTAR_OK : SPARSTAR_ERR_CUDA;
}


}  // namespace
}  // namespace sparstar

using namespace sparstar;

extern "C" {

int sparstar_abi_version(void) { return SPARSTAR_ABI_VERSION; }

const char* sparstar_strerror(int code) {
  switch (code) {
    case SPARSTAR_OK: return "ok";
    case SPARSTAR_ERR_ARG: return "invalid argument";
    case SPARSTAR_ERR_UNSUPPORTED: return "unsupported head_dim, device or size";
    case SPARSTAR_ERR_WORKSPACE: return "workspace missing or too small";
    case SPARSTAR_ERR_CUDA: return "CUDA call failed";
    case SPARSTAR_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case SPARSTAR_ERR_DEVICE_BOUNDS: return "device clamped an out-of-range index or count";
    default: return "unknown status";
  }
}

int sparstar_make_plan_ex(int64_t n_q, sparstar_segments seg, int clip, double density, int budget_mode, int block,
                          sparstar_plan* out) {
  if (out == nullptr || n_q < 0 || !valid_segments(seg) || clip < 1 || !(density > 0.0) || !(density <= 1.0) ||
      (budget_mode != SPARSTAR_BUDGET_LITERAL && budget_mode != SPARSTAR_BUDGET_CANDIDATES))
    return SPARSTAR_ERR_ARG;
  if (!valid_block(block)) return SPARSTAR_ERR_UNSUPPORTED;
  const int64_t n_kv = seg.n_text + seg.n_ctx + seg.n_cur;
  if (n_kv < 1) return SPARSTAR_ERR_ARG;
  sparstar_plan p;
  p.nqb = ceil_blocks(n_q, block);
  p.nkb = ceil_blocks(n_kv, block);
  const int64_t forced_tokens = seg.n_text + (clip == 1 ? seg.n_ctx : 0);
  p.n_forced = ceil_blocks(forced_tokens, block);
  if (p.n_forced > p.nkb) p.n_forced = p.nkb;
  p.n_cand = p.nkb - p.n_forced;
  int64_t k_total, k_topk;
  if (budget_mode == SPARSTAR_BUDGET_LITERAL) {
    k_total = ceil_guarded(density * static_cast<double>(p.nkb));
    if (k_total < p.n_forced) k_total = p.n_forced;
    if (k_total > p.nkb) k_total = p.nkb;
    k_topk = k_total - p.n_forced;
  } else {
    k_topk = ceil_guarded(density * static_cast<double>(p.n_cand));
    if (k_topk > p.n_cand) k_topk = p.n_cand;
    if (k_topk < 0) k_topk = 0;
    k_total = p.n_forced + k_topk;
  }
  if (k_total > INT32_MAX) return SPARSTAR_ERR_UNSUPPORTED;
  p.k_total = static_cast<int32_t>(k_total);
  p.k_topk = static_cast<int32_t>(k_topk);
  *out = p;
  return SPARSTAR_OK;
}

int sparstar_make_plan(int64_t n_q, sparstar_segments seg, int clip, double density, int budget_mode,
                       sparstar_plan* out) {
  return sparstar_make_plan_ex(n_q, seg, clip, density, budget_mode, SPARSTAR_BLOCK, out);
}

int sparstar_workspace_size_ex(int heads, int64_t n_q, sparstar_segments seg, int head_dim, int block, size_t* bytes) {
  if (bytes == nullptr || heads < 1 || n_q < 0 || !valid_segments(seg)) return SPARSTAR_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return SPARSTAR_ERR_UNSUPPORTED;
  if (!valid_block(block)) return SPARSTAR_ERR_UNSUPPORTED;
  const int64_t n_kv = seg.n_text + seg.n_ctx + seg.n_cur;
  if (n_kv < 1) return SPARSTAR_ERR_ARG;
  *bytes = workspace_layout(heads, ceil_blocks(n_q, block), ceil_blocks(n_kv, block), head_dim, true).total;
  return SPARSTAR_OK;
}

int sparstar_workspace_size(int heads, int64_t n_q, sparstar_segments seg, int head_dim, size_t* bytes) {
  return sparstar_workspace_size_ex(heads, n_q, seg, head_dim, SPARSTAR_BLOCK, bytes);
}

int sparstar_select_ex(const void* q, const void* k, int heads, int64_t n_q, sparstar_segments seg, int head_dim,
                       int clip, double density, int budget_mode, int block, int32_t* idx, int32_t* cnt, int32_t kmax,
                       float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  sparstar_plan plan;
  int rc = sparstar_make_plan_ex(n_q, seg, clip, density, budget_mode, block, &plan);
  if (rc != SPARSTAR_OK) return rc;
  if (heads < 1) return SPARSTAR_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return SPARSTAR_ERR_UNSUPPORTED;
  if (n_q == 0) return SPARSTAR_OK;
  if (q == nullptr || k == nullptr || idx == nullptr || cnt == nullptr || !aligned16(q) || !aligned16(k) ||
      (scores != nullptr && !aligned16(scores)) || kmax < plan.k_total)
    return SPARSTAR_ERR_ARG;
  const int64_t rows = static_cast<int64_t>(heads) * plan.nqb;
  if (rows > INT32_MAX || static_cast<int64_t>(heads) * (plan.nqb + plan.nkb) > INT32_MAX ||
      plan.nqb > 65535 * 64LL || plan.n_cand > kMaxCandidates || heads > 65535)
    return SPARSTAR_ERR_UNSUPPORTED;
  const bool needs_scores = plan.k_topk > 0 && plan.k_topk < plan.n_cand;
  const bool compute_scores = needs_scores || scores != nullptr;
  const Workspace ws = workspace_layout(heads, plan.nqb, plan.nkb, head_dim, scores == nullptr);
  if (compute_scores && (workspace == nullptr || workspace_bytes < ws.total ||
                         (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
    return SPARSTAR_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev)) != SPARSTAR_OK) return rc;
  if ((rc = set_kernel_attrs(dev)) != SPARSTAR_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n_kv = seg.n_text + seg.n_ctx + seg.n_cur;
  const int nqb = static_cast<int>(plan.nqb), nkb = static_cast<int>(plan.nkb);

  if (compute_scores) {
    if (dev->major != 10) return SPARSTAR_ERR_UNSUPPORTED;  // tensor-core scores need sm_100
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    auto* q_hi = reinterpret_cast<__nv_bfloat16*>(wsb + ws.q_hi);
    auto* q_lo = reinterpret_cast<__nv_bfloat16*>(wsb + ws.q_lo);
    auto* k_hi = reinterpret_cast<__nv_bfloat16*>(wsb + ws.k_hi);
    auto* k_lo = reinterpret_cast<__nv_bfloat16*>(wsb + ws.k_lo);
    float* S = scores != nullptr ? scores : reinterpret_cast<float*>(wsb + ws.scores);
    CUtensorMap tqh, tql, tkh, tkl;
    if (make_map(&tqh, q_hi, nqb, heads, head_dim) != SPARSTAR_OK ||
        make_map(&tql, q_lo, nqb, heads, head_dim) != SPARSTAR_OK ||
        make_map(&tkh, k_hi, nkb, heads, head_dim) != SPARSTAR_OK ||
        make_map(&tkl, k_lo, nkb, heads, head_dim) != SPARSTAR_OK)
      return SPARSTAR_ERR_CUDA;
    const unsigned pool_grid = static_cast<unsigned>(heads) * static_cast<unsigned>(nqb + nkb);
    const int score_tiles = heads * ((nqb + 127) / 128) * ((nkb + 127) / 128);
    const dim3 sgrid(static_cast<unsigned>(score_tiles < dev->sms ? score_tiles : dev->sms));
    const float inv_sqrt_d = 1.0f / std::sqrt(static_cast<float>(head_dim));
    const auto* qb16 = static_cast<const __nv_bfloat16*>(q);
    const auto* kb16 = static_cast<const __nv_bfloat16*>(k);
    if (head_dim == 128) {
      if (block == 128)
        pool_kernel<128, 128><<<pool_grid, 256, 0, st>>>(qb16, kb16, n_q, n_kv, nqb, nkb, q_hi, q_lo, k_hi, k_lo);
      else
        pool_kernel<128, 64><<<pool_grid, 256, 0, st>>>(qb16, kb16, n_q, n_kv, nqb, nkb, q_hi, q_lo, k_hi, k_lo);
      launch_after(score_tc_kernel<128>, sgrid, dim3(ScoreConfig<128>::kThreads), ScoreConfig<128>::kSmemBytes, st, tqh,
                   tql, tkh, tkl, S, heads, nqb, nkb, inv_sqrt_d, dev->status);
    } else {
      if (block == 128)
        pool_kernel<64, 128><<<pool_grid, 256, 0, st>>>(qb16, kb16, n_q, n_kv, nqb, nkb, q_hi, q_lo, k_hi, k_lo);
      else
        pool_kernel<64, 64><<<pool_grid, 256, 0, st>>>(qb16, kb16, n_q, n_kv, nqb, nkb, q_hi, q_lo, k_hi, k_lo);
      launch_after(score_tc_kernel<64>, sgrid, dim3(ScoreConfig<64>::kThreads), ScoreConfig<64>::kSmemBytes, st, tqh,
                   tql, tkh, tkl, S, heads, nqb, nkb, inv_sqrt_d, dev->status);
    }
    if ((rc = launch_status()) != SPARSTAR_OK) return rc;
    if (needs_scores) {
      const int n_forced = static_cast<int>(plan.n_forced);
      launch_topk(S, rows, nkb, n_forced, static_cast<int>(plan.k_topk), idx, cnt, kmax, st);
      return launch_status();
    }
  }
  fill_kernel<<<static_cast<unsigned>(rows), 128, 0, st>>>(plan.k_total, idx, cnt, kmax);
  return launch_status();
}

int sparstar_select(const void* q, const void* k, int heads, int64_t n_q, sparstar_segments seg, int head_dim,
                    int clip, double density, int budget_mode, int32_t* idx, int32_t* cnt, int32_t kmax,
                    float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  return sparstar_select_ex(q, k, heads, n_q, seg, head_dim, clip, density, budget_mode, SPARSTAR_BLOCK, idx, cnt,
                            kmax, scores, workspace, workspace_bytes, stream);
}

int sparstar_topk(const float* scores, int64_t rows, int nkb, int n_forced, int k_topk, int32_t* idx, int32_t* cnt,
                  int32_t kmax, void* stream) {
  if (rows < 0 || nkb < 1 || n_forced < 0 || n_forced > nkb || k_topk < 0 || k_topk > nkb - n_forced ||
      kmax < n_forced + k_topk)
    return SPARSTAR_ERR_ARG;
  const int n_cand = nkb - n_forced;
  const bool reads_scores = k_topk > 0 && k_topk < n_cand;
  if (rows > INT32_MAX || (reads_scores && n_cand > kMaxCandidates)) return SPARSTAR_ERR_UNSUPPORTED;
  if (rows == 0) return SPARSTAR_OK;
  if (idx == nullptr || cnt == nullptr ||
      (reads_scores && (scores == nullptr || (reinterpret_cast<uintptr_t>(scores) & 3u) != 0)))
    return SPARSTAR_ERR_ARG;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != SPARSTAR_OK) return rc;
  if (dev->major != 10) return SPARSTAR_ERR_UNSUPPORTED;
  if ((rc = set_kernel_attrs(dev)) != SPARSTAR_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (reads_scores)
    launch_topk(scores, rows, nkb, n_forced, k_topk, idx, cnt, kmax, st);
  else
    fill_kernel<<<static_cast<unsigned>(rows), 128, 0, st>>>(n_forced + k_topk, idx, cnt, kmax);
  return launch_status();
}

int sparstar_attn_ex(const void* q, const void* k, const void* v, int heads, int64_t n_q, int64_t n_kv, int head_dim,
                     int block, const int32_t* idx, const int32_t* cnt, int32_t kmax, float sm_scale, void* o,
                     float* lse, void* stream) {
  if (heads < 1 || n_q < 0 || n_kv < 1 || kmax < 1) return SPARSTAR_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return SPARSTAR_ERR_UNSUPPORTED;
  if (!valid_block(block)) return SPARSTAR_ERR_UNSUPPORTED;
  if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SPARSTAR_ERR_ARG;
  if (n_q == 0) return SPARSTAR_OK;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || idx == nullptr || cnt == nullptr ||
      !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0))
    return SPARSTAR_ERR_ARG;
  const int64_t nqb = ceil_blocks(n_q, block), nkb = ceil_blocks(n_kv, block);
  if (static_cast<int64_t>(heads) * nqb > INT32_MAX / 2 || n_q > INT32_MAX || n_kv > INT32_MAX || nkb > INT32_MAX)
    return SPARSTAR_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != SPARSTAR_OK) return rc;
  if (dev->major != 10) return SPARSTAR_ERR_UNSUPPORTED;
  if ((rc = set_kernel_attrs(dev)) != SPARSTAR_OK) return rc;
  CUtensorMap tq, tk, tv;
  const unsigned kv_rows = static_cast<unsigned>(block);
  if (make_map(&tq, q, n_q, heads, head_dim) != SPARSTAR_OK ||
      make_map(&tk, k, n_kv, heads, head_dim, kv_rows) != SPARSTAR_OK ||
      make_map(&tv, v, n_kv, heads, head_dim, kv_rows) != SPARSTAR_OK)
    return SPARSTAR_ERR_CUDA;
  AttnParams p;
  p.idx = idx;
  p.cnt = cnt;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = dev->status;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.nqb = static_cast<int>(nqb);
  p.nkb = static_cast<int>(nkb);
  p.kmax = kmax;
  p.n_items = static_cast<int>(heads * nqb);
  const float scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int slots_needed = (p.n_items + 1) / 2;
  const int grid = slots_needed < dev->sms ? slots_needed : dev->sms;
  if (block == 128) {
    if (head_dim == 128)
      attn_sparse_kernel<128><<<grid, AttnConfig<128>::kThreads, AttnConfig<128>::kSmemBytes, st>>>(tq, tk, tv, p);
    else
      attn_sparse_kernel<64><<<grid, AttnConfig<64>::kThreads, AttnConfig<64>::kSmemBytes, st>>>(tq, tk, tv, p);
  } else {
    if (head_dim == 128)
      attn_sparse_kernel<128, 64><<<grid, AttnConfig<128, 64>::kThreads, AttnConfig<128, 64>::kSmemBytes, st>>>(tq, tk, tv, p);
    else
      attn_sparse_kernel<64, 64><<<grid, AttnConfig<64, 64>::kThreads, AttnConfig<64, 64>::kSmemBytes, st>>>(tq, tk, tv, p);
  }
  return launch_status();
}

int sparstar_attn(const void* q, const void* k, const void* v, int heads, int64_t n_q, int64_t n_kv, int head_dim,
                  const int32_t* idx, const int32_t* cnt, int32_t kmax, float sm_scale, void* o, float* lse,
                  void* stream) {
  return sparstar_attn_ex(q, k, v, heads, n_q, n_kv, head_dim, SPARSTAR_BLOCK, idx, cnt, kmax, sm_scale, o, lse, stream);
}

int sparstar_retained_mass(const float* lse_kept, const float* lse_dense, int heads, int64_t n_q, float* r_token,
                           float* e_block, void* stream) {
  if (heads < 1 || heads > 65535 || n_q < 0) return SPARSTAR_ERR_ARG;
  if (n_q == 0) return SPARSTAR_OK;
  if (lse_kept == nullptr || lse_dense == nullptr || e_block == nullptr) return SPARSTAR_ERR_ARG;
  const int64_t nqb = ceil_blocks(n_q);
  if (nqb > INT32_MAX) return SPARSTAR_ERR_UNSUPPORTED;
  mass_kernel<<<dim3(static_cast<unsigned>(nqb), static_cast<unsigned>(heads)), 128, 0,
                static_cast<cudaStream_t>(stream)>>>(lse_kept, lse_dense, n_q, static_cast<int>(nqb), r_token, e_block);
  return launch_status();
}

int sparstar_token_bound_workspace_size(int heads, int64_t n_q, size_t* bytes) {
  if (bytes == nullptr || heads < 1 || n_q < 0) return SPARSTAR_ERR_ARG;
  *bytes = 4 * align256(static_cast<size_t>(heads) * static_cast<size_t>(n_q) * 4);
  return SPARSTAR_OK;
}

int sparstar_token_bound(const void* q, const void* k, int heads, int64_t n_q, int64_t n_kv, int head_dim,
                         const int32_t* idx, const int32_t* cnt, int32_t kmax, const float* lse_dense, float sm_scale,
                         float* u_token, float* u_block, void* workspace, size_t workspace_bytes, void* stream) {
  if (heads < 1 || heads > 65535 || n_q < 0 || n_kv < 1 || kmax < 1) return SPARSTAR_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return SPARSTAR_ERR_UNSUPPORTED;
  if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SPARSTAR_ERR_ARG;
  if (n_q == 0) return SPARSTAR_OK;
  if (q == nullptr || k == nullptr || idx == nullptr || cnt == nullptr || lse_dense == nullptr ||
      u_block == nullptr || !aligned16(q) || !aligned16(k))
    return SPARSTAR_ERR_ARG;
  size_t need = 0;
  sparstar_token_bound_workspace_size(heads, n_q, &need);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SPARSTAR_ERR_WORKSPACE;
  const int64_t nqb = ceil_blocks(n_q), nkb = ceil_blocks(n_kv);
  if (static_cast<int64_t>(heads) * nqb > INT32_MAX / 2 || n_q > INT32_MAX || n_kv > INT32_MAX || nqb > 65535 * 64LL ||
      nkb > kBoundMaxKvBlocks)
    return SPARSTAR_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != SPARSTAR_OK) return rc;
  if (dev->major != 10) return SPARSTAR_ERR_UNSUPPORTED;
  if ((rc = set_kernel_attrs(dev)) != SPARSTAR_OK) return rc;
  CUtensorMap tq, tk;
  if (make_map(&tq, q, n_q, heads, head_dim) != SPARSTAR_OK || make_map(&tk, k, n_kv, heads, head_dim) != SPARSTAR_OK)
    return SPARSTAR_ERR_CUDA;
  const size_t arr = align256(static_cast<size_t>(heads) * static_cast<size_t>(n_q) * 4);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  BoundParams p;
  p.st.lo_idx = reinterpret_cast<int*>(w);
  p.st.need = reinterpret_cast<int*>(w + arr);
  p.st.above_sum = reinterpret_cast<float*>(w + 2 * arr);
  p.st.u = reinterpret_cast<float*>(w + 3 * arr);
  p.lse_dense = lse_dense;
  p.u_block = u_block;
  p.status = dev->status;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.nqb = static_cast<int>(nqb);
  p.nkb = static_cast<int>(nkb);
  p.n_items = static_cast<int>(heads * nqb);
  const float scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 rows_grid(static_cast<unsigned>(nqb), static_cast<unsigned>(heads));
  bound_init_kernel<<<rows_grid, 128, 0, st>>>(idx, cnt, kmax, n_q, n_kv, p.nqb, p.st, dev->status);
  if ((rc = launch_status()) != SPARSTAR_OK) return rc;
  const int grid = p.n_items < dev->sms ? p.n_items : dev->sms;
  for (int pass = 0; pass < kBoundPasses; ++pass) {
    p.pass = pass;
    if (head_dim == 128)
      bound_pass_kernel<128><<<grid, BoundConfig<128>::kThreads, BoundConfig<128>::kSmemBytes, st>>>(tq, tk, p);
    else
      bound_pass_kernel<64><<<grid, BoundConfig<64>::kThreads, BoundConfig<64>::kSmemBytes, st>>>(tq, tk, p);
    if ((rc = launch_status()) != SPARSTAR_OK) return rc;
  }
  bound_block_kernel<<<rows_grid, 128, 0, st>>>(p.st.u, n_q, p.nqb, u_token, u_block);
  return launch_status();
}

int sparstar_forward_ex(const void* q, const void* k, const void* v, int heads, int64_t n_q, sparstar_segments seg,
                        int head_dim, int clip, double density, int budget_mode, int block, float sm_scale,
                        int32_t* idx, int32_t* cnt, int32_t kmax, void* o, float* lse, void* workspace,
                        size_t workspace_bytes, void* stream) {
  int rc = sparstar_select_ex(q, k, heads, n_q, seg, head_dim, clip, density, budget_mode, block, idx, cnt, kmax,
                              nullptr, workspace, workspace_bytes, stream);
  if (rc != SPARSTAR_OK) return rc;
  const int64_t n_kv = seg.n_text + seg.n_ctx + seg.n_cur;
  return sparstar_attn_ex(q, k, v, heads, n_q, n_kv, head_dim, block, idx, cnt, kmax, sm_scale, o, lse, stream);
}

int sparstar_forward(const void* q, const void* k, const void* v, int heads, int64_t n_q, sparstar_segments seg,
                     int head_dim, int clip, double density, int budget_mode, float sm_scale, int32_t* idx,
                     int32_t* cnt, int32_t kmax, void* o, float* lse, void* workspace, size_t workspace_bytes,
                     void* stream) {
  return sparstar_forward_ex(q, k, v, heads, n_q, seg, head_dim, clip, density, budget_mode, SPARSTAR_BLOCK, sm_scale,
                             idx, cnt, kmax, o, lse, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- no-allocation selection
// Scratch of sparstar_select_noalloc: a fixed device array per device that loads the library.
// Host code must not pass `g_select_scratch` itself to a kernel (on the host it names a
// host-side stand-in); it passes the device address looked up once per device below.
static __device__ __align__(256) unsigned char g_select_scratch[SPARSTAR_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mutex;
void* g_scratch_ptr[sparstar::kMaxDevices] = {};
}  // namespace

int sparstar_select_noalloc(const void* q, const void* k, int heads, int64_t n_q, sparstar_segments seg,
                            int head_dim, int clip, double density, int budget_mode, int32_t* idx, int32_t* cnt,
                            int32_t kmax, void* stream) {
  // Sizes are checked before any CUDA call, so an oversized request never touches the device.
  sparstar_plan plan;
  int rc = sparstar_make_plan(n_q, seg, clip, density, budget_mode, &plan);
  if (rc != SPARSTAR_OK) return rc;
  size_t need = 0;
  if ((rc = sparstar_workspace_size(heads, n_q, seg, head_dim, &need)) != SPARSTAR_OK) return rc;
  // Rows that do not depend on the scores (forced-only, or every block kept) use no scratch.
  if (!(plan.k_topk > 0 && plan.k_topk < plan.n_cand))
    return sparstar_select(q, k, heads, n_q, seg, head_dim, clip, density, budget_mode, idx, cnt, kmax, nullptr,
                           nullptr, 0, stream);
  if (need > SPARSTAR_NOALLOC_SCRATCH_BYTES) return SPARSTAR_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= sparstar::kMaxDevices) return SPARSTAR_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_select_scratch) != cudaSuccess || ptr == nullptr) return SPARSTAR_ERR_CUDA;
      g_scratch_ptr[dev] = ptr;
    }
    scratch = g_scratch_ptr[dev];
  }
  return sparstar_select(q, k, heads, n_q, seg, head_dim, clip, density, budget_mode, idx, cnt, kmax, nullptr,
                         scratch, SPARSTAR_NOALLOC_SCRATCH_BYTES, stream);
}

int sparstar_map_scores(const float* scores_prev, int heads, sparstar_segments seg_prev, sparstar_grid grid_prev,
                        sparstar_segments seg_now, sparstar_grid grid_now, float* scores_now, void* stream) {
  if (heads < 1 || heads > 65535 || !valid_segments(seg_prev) || !valid_segments(seg_now)) return SPARSTAR_ERR_ARG;
  const sparstar_grid* grids[2] = {&grid_prev, &grid_now};
  const int64_t n_cur[2] = {seg_prev.n_cur, seg_now.n_cur};
  for (int g = 0; g < 2; ++g) {
    const sparstar_grid& G = *grids[g];
    if (G.frames < 1 || G.height < 1 || G.width < 1) return SPARSTAR_ERR_ARG;
    const __int128 n = static_cast<__int128>(G.frames) * G.height * G.width;
    if (n != n_cur[g]) return SPARSTAR_ERR_ARG;  // the grid lays out exactly the current tokens
  }
  if (seg_prev.n_text != seg_now.n_text || seg_prev.n_ctx != seg_now.n_ctx ||
      seg_now.n_text % SPARSTAR_BLOCK != 0 || seg_now.n_ctx % SPARSTAR_BLOCK != 0)
    return SPARSTAR_ERR_ARG;
  const int64_t n_prefix = (seg_now.n_text + seg_now.n_ctx) / SPARSTAR_BLOCK;
  const int64_t nqb_prev = ceil_blocks(seg_prev.n_cur), nqb_now = ceil_blocks(seg_now.n_cur);
  const int64_t nkb_prev = n_prefix + nqb_prev, nkb_now = n_prefix + nqb_now;
  if (nkb_now > kMaxMapColumns || nkb_prev > INT32_MAX || static_cast<int64_t>(heads) * nqb_prev * nkb_prev > (1LL << 40))
    return SPARSTAR_ERR_UNSUPPORTED;
  if (scores_prev == nullptr || scores_now == nullptr || (reinterpret_cast<uintptr_t>(scores_prev) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(scores_now) & 3u) != 0)
    return SPARSTAR_ERR_ARG;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != SPARSTAR_OK) return rc;
  if ((rc = set_kernel_attrs(dev)) != SPARSTAR_OK) return rc;
  const GridDims now{grid_now.frames, grid_now.height, grid_now.width};
  const GridDims prev{grid_prev.frames, grid_prev.height, grid_prev.width};
  const dim3 grid(static_cast<unsigned>((nqb_now + kMapRowsPerCta - 1) / kMapRowsPerCta), static_cast<unsigned>(heads));
  map_scores_kernel<<<grid, 256, static_cast<size_t>(nkb_now) * 4, static_cast<cudaStream_t>(stream)>>>(
      scores_prev, scores_now, static_cast<int>(nqb_prev), static_cast<int>(nkb_prev), static_cast<int>(nqb_now),
      static_cast<int>(nkb_now), static_cast<int>(n_prefix), seg_now.n_cur, now, prev);
  return launch_status();
}

int sparstar_read_probe(const void* src, size_t bytes, unsigned* sink, void* stream) {
  if (bytes == 0) return SPARSTAR_OK;
  if (src == nullptr || sink == nullptr || !aligned16(src) || (bytes & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(sink) & 3u) != 0)
    return SPARSTAR_ERR_ARG;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != SPARSTAR_OK) return rc;
  read_probe_kernel<<<static_cast<unsigned>(dev->sms) * 4u, 512, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<int64_t>(bytes / 16), sink);
  return launch_status();
}

int sparstar_selftest_wait_timeout(void* stream) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != SPARSTAR_OK) return rc;
  if (dev->major != 10) return SPARSTAR_ERR_UNSUPPORTED;
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev->status);
  return launch_status();
}

int sparstar_device_status(void* stream, int clear) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != SPARSTAR_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SPARSTAR_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, dev->status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return SPARSTAR_ERR_CUDA;
  if (clear && word != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(dev->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return SPARSTAR_ERR_CUDA;
  }
  if (word & kStatusTimeout) return SPARSTAR_ERR_DEVICE_TIMEOUT;
  if (word & kStatusBounds) return SPARSTAR_ERR_DEVICE_BOUNDS;
  return SPARSTAR_OK;
}

}  // extern "C"
