// libssa.so: C ABI of content-routed block-sparse attention on B200.
//
// Host side: argument validation (synchronous, before any launch), TMA
// tensor-map encoding, and the launches of the three sm_100a kernels on the
// caller's stream.  The library allocates no device memory; its device state
// is the error word below.  The CUDA runtime is linked statically and the
// driver's tensor-map encoder is looked up at first use, so the library loads
// on a machine without a GPU (calls then fail with SSA_ERR_CUDA).
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <mutex>
#include <string>

#include "../../include/ssa.h"
#include "attend.cuh"
#include "backward.cuh"
#include "backward_tc.cuh"
#include "common.cuh"
#include "consensus.cuh"
#include "cumulant.cuh"
#include "decode.cuh"
#include "pool.cuh"
#include "route.cuh"
#include "route_tc.cuh"
#include "tree.cuh"

namespace ssa {
__global__ void probe_wait_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives: the wait must give up on its own
    mbar_wait(&bar, 0, timeout_ns, &abort_flag, kSiteProbe);
  }
  __syncthreads();
}
// Issue-rate probe of the exponential the softmax uses (ex2.approx): every
// thread runs 8 independent chains y <- 2^(-y), which stay in [0.5, 1], so
// the special-function pipe is the only busy unit.  The sum is written only
// when it is negative, which it never is, so nothing reaches memory but the
// work cannot be dropped.
__global__ void __launch_bounds__(256) ex2_rate_kernel(int32_t iters, float* sink) {
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = 0.5f + 0.0625f * i + 1e-4f * (threadIdx.x & 15);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = ex2_approx(-y[i]);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += y[i];
  if (s < 0.f) *sink = s;
}

// Scratch of ssa_forward_static: summaries, routed lists and counts live
// here instead of in a caller-provided workspace.  It is part of the loaded
// module, so every device that loads this library holds these bytes until the
// process exits.  Host code must not use the name as a pointer: on the host it
// is only a stand-in; the device address comes from cudaGetSymbolAddress.
constexpr size_t kStaticScratchBytes = static_cast<size_t>(32) << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];
}  // namespace ssa

namespace {

constexpr int32_t kVersion = 2;
thread_local std::string g_msg;

ssa_status fail(ssa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
ssa_status fail(ssa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_msg = buf;
  return s;
}

ssa_status ok() {
  g_msg.clear();
  return SSA_OK;
}

ssa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool pow2_in(int32_t x, int32_t lo, int32_t hi) {
  return x >= lo && x <= hi && (x & (x - 1)) == 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

ssa_status validate(const ssa_params* p) {
  if (p == nullptr) return fail(SSA_ERR_INVALID_ARG, "params is NULL");
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->N < 1 || p->D < 1)
    return fail(SSA_ERR_INVALID_ARG, "B, Hq, Hkv, N, D must be positive");
  if (p->Hq % p->Hkv != 0) return fail(SSA_ERR_INVALID_ARG, "Hq must be a multiple of Hkv");
  if (p->D != 64 && p->D != 128) return fail(SSA_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (!pow2_in(p->block_k, 16, 128) || !pow2_in(p->block_q, 16, 128))
    return fail(SSA_ERR_UNSUPPORTED, "block_k and block_q must be powers of two in [16, 128]");
  if (p->N % p->block_k != 0 || p->N % p->block_q != 0)
    return fail(SSA_ERR_UNSUPPORTED, "N must be a multiple of block_k and block_q");
  if (p->top_k < 0 || p->top_k > 64) return fail(SSA_ERR_UNSUPPORTED, "top_k must be in 0..64");
  if (p->window < 0) return fail(SSA_ERR_INVALID_ARG, "window must be >= 0");
  if (p->causal != 0 && p->causal != 1) return fail(SSA_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (p->causal && p->window < 1)
    return fail(SSA_ERR_INVALID_ARG, "causal attention needs window >= 1 (every query sees itself)");
  if (!p->causal && p->window != 0)
    return fail(SSA_ERR_INVALID_ARG, "the non-causal variant has no window (window must be 0)");
  if (!p->causal && p->top_k < 1)
    return fail(SSA_ERR_INVALID_ARG, "the non-causal variant needs top_k >= 1");
  if (!(p->scale >= 0.f) || !std::isfinite(p->scale))
    return fail(SSA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (p->wait_timeout_us < 0) return fail(SSA_ERR_INVALID_ARG, "wait_timeout_us must be >= 0");
  if (!std::isfinite(p->beta)) return fail(SSA_ERR_INVALID_ARG, "beta must be finite");
  if (p->consensus != 0 && p->consensus != 1)
    return fail(SSA_ERR_INVALID_ARG, "consensus must be 0 or 1");
  if (p->consensus && (p->Hq / p->Hkv) * p->top_k > ssa::kConsMaxVotes)
    return fail(SSA_ERR_UNSUPPORTED, "consensus routing needs (Hq / Hkv) * top_k <= %d",
                ssa::kConsMaxVotes);
  const int64_t nb = p->N / p->block_k;
  if (nb >= (1 << 23)) return fail(SSA_ERR_UNSUPPORTED, "N / block_k must be below 2^23");
  if (p->tree_fanout != 0) {
    if (!pow2_in(p->tree_fanout, 1, 256) || p->tree_fanout > nb)
      return fail(SSA_ERR_UNSUPPORTED,
                  "tree_fanout must be 0 or a power of two in [1, 256] and at most N / block_k");
    if (p->tree_beam < 1 || p->tree_beam > ssa::kTreeMaxBeam)
      return fail(SSA_ERR_UNSUPPORTED, "tree_beam must be in 1..%d", ssa::kTreeMaxBeam);
    if (p->beta != 0.0f)
      return fail(SSA_ERR_UNSUPPORTED, "two-level routing ranks by block means (beta must be 0)");
  } else if (p->tree_beam != 0) {
    return fail(SSA_ERR_INVALID_ARG, "tree_beam must be 0 without tree_fanout");
  }
  const int64_t rows = static_cast<int64_t>(p->B) * p->Hq * p->N;
  if (rows > (static_cast<int64_t>(1) << 31) - 1)
    return fail(SSA_ERR_UNSUPPORTED, "B * Hq * N must fit in int32");
  if (p->causal) {
    const int64_t nwin = (static_cast<int64_t>(p->window) + ssa::kAtQT - 2) / p->block_k + 2;
    if (nwin > ssa::kAtLCap)
      return fail(SSA_ERR_UNSUPPORTED, "window spans more than %d key blocks per query tile",
                  ssa::kAtLCap);
  }
  return SSA_OK;
}

uint64_t timeout_ns(const ssa_params* p) {
  return p->wait_timeout_us > 0 ? static_cast<uint64_t>(p->wait_timeout_us) * 1000ull
                                : 2000000000ull;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

ssa_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode == nullptr)
    return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (no CUDA driver?)");
  return SSA_OK;
}

// 3-D view [heads, N, D] of a bf16 tensor, box {64 columns, rows, 1}, 128B swizzle
ssa_status make_map(CUtensorMap* m, const void* base, int64_t heads, int64_t n, int64_t d,
                    uint32_t box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2),
                                 static_cast<cuuint64_t>(n * d * 2)};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SSA_OK;
}

// ---------------------------------------------------------------- launches
ssa_status launch_pool(const ssa_params* p, const void* x0, int32_t H0, int32_t blk0, float* out0,
                       const void* x1, int32_t H1, int32_t blk1, float* out1,
                       cudaStream_t stream) {
  // one warp per block; the kernel's split point is counted in warps
  ssa::PoolJob j0{static_cast<const uint4*>(x0), out0,
                  static_cast<int64_t>(p->B) * H0 * (p->N / blk0), blk0, 1.0f / blk0};
  ssa::PoolJob j1 = j0;
  j1.n_blocks = 0;  // single job: the tail warps of the grid do nothing
  int64_t n1 = 0;
  if (x1 != nullptr) {
    j1 = ssa::PoolJob{static_cast<const uint4*>(x1), out1,
                      static_cast<int64_t>(p->B) * H1 * (p->N / blk1), blk1, 1.0f / blk1};
    n1 = j1.n_blocks;
  }
  const int64_t split = j0.n_blocks;
  const int64_t total_threads = (split + n1) * 32;
  const int64_t grid = (total_threads + 255) / 256;
  if (p->D == 64)
    ssa::block_mean_kernel<64><<<static_cast<unsigned>(grid), 256, 0, stream>>>(j0, j1, split);
  else
    ssa::block_mean_kernel<128><<<static_cast<unsigned>(grid), 256, 0, stream>>>(j0, j1, split);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "block_mean_kernel launch");
  return SSA_OK;
}

template <int D, int R, int RT>
cudaError_t launch_route_t(ssa::RouteArgs a, int B, cudaStream_t stream) {
  a.n_row_tiles = (a.NQB + RT - 1) / RT;
  const size_t smem = ssa::route_smem_bytes<D, R, RT>();
  cudaError_t e = cudaFuncSetAttribute(ssa::route_kernel<D, R, RT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_row_tiles, B * a.Hq);
  ssa::route_kernel<D, R, RT><<<grid, ssa::kRouteThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int D, int KM>
cudaError_t launch_route_tc_t(ssa::RouteArgs a, int B, cudaStream_t stream) {
  a.n_row_tiles = (a.NQB + ssa::kRtcRows - 1) / ssa::kRtcRows;
  const uint32_t smem = ssa::RtcLayout<D>::SMEM_BYTES;
  dim3 grid(a.n_row_tiles, B * a.Hq);
  // with the pre-split key image one producer thread replaces the stager warps
  if (a.kimg != nullptr) {
    cudaError_t e = cudaFuncSetAttribute(ssa::route_tc_kernel<D, KM, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    ssa::route_tc_kernel<D, KM, true><<<grid, ssa::kRtcThreadsPre, smem, stream>>>(a);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(ssa::route_tc_kernel<D, KM, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  ssa::route_tc_kernel<D, KM, false><<<grid, ssa::kRtcThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_route_tc(const ssa::RouteArgs& a, int B, cudaStream_t stream) {
  if (a.top_k <= 16) return launch_route_tc_t<D, 16>(a, B, stream);
  if (a.top_k <= 32) return launch_route_tc_t<D, 32>(a, B, stream);
  return launch_route_tc_t<D, 64>(a, B, stream);
}

template <int D, int R>
cudaError_t launch_route_rt(const ssa::RouteArgs& a, int B, cudaStream_t stream) {
  // 64 query blocks per CTA reuse each summary tile the most; use 16 when 64
  // would give fewer than two CTAs per SM
  const int64_t ctas64 = static_cast<int64_t>(B) * a.Hq * ((a.NQB + 63) / 64);
  if (ctas64 < 2 * 148) return launch_route_t<D, R, 16>(a, B, stream);
  return launch_route_t<D, R, 64>(a, B, stream);
}

template <int D, int KM, int RT>
cudaError_t launch_route_rows_t(ssa::RouteArgs a, int B, cudaStream_t stream) {
  a.n_row_tiles = (a.NQB + RT - 1) / RT;
  const size_t smem = ssa::route_rows_smem_bytes<D, KM, RT>();
  cudaError_t e = cudaFuncSetAttribute(ssa::route_rows_kernel<D, KM, RT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_row_tiles, B * a.Hq);
  ssa::route_rows_kernel<D, KM, RT><<<grid, ssa::kRouteThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// Row tile: a larger tile reuses each key-summary tile over more query
// blocks, which pays as long as the grid keeps most SMs busy.  Measured on
// B200 (route ms for RT = 16 / 32 / 64 / 128): 32K tokens x 14 heads
// 0.067 / 0.072 / 0.064 / 0.089; 8K tokens x 64 heads 0.044 / 0.031 / 0.027 /
// 0.038; 16K non-causal x 32 heads 0.536 / 0.340 / 0.265 / 0.208.  Rule: the
// largest tile whose grid has at least two thirds as many CTAs as SMs.
// SSA_ROUTE_RT=16|32|64|128 forces one (a tuning hook).
template <int D, int KM>
cudaError_t launch_route_rows_km(const ssa::RouteArgs& a, int B, cudaStream_t stream) {
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  int rt = 16;
  for (const int cand : {128, 64, 32, 16}) {
    const int64_t ctas = static_cast<int64_t>(B) * a.Hq * ((a.NQB + cand - 1) / cand);
    if (3 * ctas >= 2 * static_cast<int64_t>(sms)) {
      rt = cand;
      break;
    }
  }
  if (const char* force = std::getenv("SSA_ROUTE_RT")) {
    const int f = std::atoi(force);
    if (f == 16 || f == 32 || f == 64 || f == 128) rt = f;
  }
  switch (rt) {
    case 128: return launch_route_rows_t<D, KM, 128>(a, B, stream);
    case 64: return launch_route_rows_t<D, KM, 64>(a, B, stream);
    case 32: return launch_route_rows_t<D, KM, 32>(a, B, stream);
    default: return launch_route_rows_t<D, KM, 16>(a, B, stream);
  }
}

// fp32 router: thread-per-row selection for top_k <= 32, warp lists beyond
template <int D>
cudaError_t launch_route_fp32(const ssa::RouteArgs& a, int B, cudaStream_t stream) {
  if (a.top_k <= 8) return launch_route_rows_km<D, 8>(a, B, stream);
  if (a.top_k <= 16) return launch_route_rows_km<D, 16>(a, B, stream);
  if (a.top_k <= 32) return launch_route_rows_km<D, 32>(a, B, stream);
  return launch_route_rt<D, 2>(a, B, stream);
}

// The tensor-core router ranks exactly like the fp32 one (see route_tc.cuh).
// Measured on B200 (fp32 form = thread-per-row selection): it wins once the
// score matrix is large (1M tokens: 6.5 vs 10.3 ms) and loses on smaller ones
// (16K image tokens, 32 heads: 0.35 vs 0.27 ms; 32K tokens: 0.35 vs 0.07 ms),
// where its per-tile steps are latency-bound, so it takes problems with at
// least 2^26 (query block, key block) pairs per head.
// SSA_ROUTER=fp32 / tc forces one form (the tests run both and compare).
bool use_tc_router(const ssa_params* p) {
  const char* env = std::getenv("SSA_ROUTER");
  const int64_t nb = p->N / p->block_k, nqb = p->N / p->block_q;
  if (p->top_k == 0 || nb > 65535) return false;  // queued candidates are 16-bit offsets
  if (env != nullptr && std::string(env) == "fp32") return false;
  if (env != nullptr && std::string(env) == "tc") return true;
  // admissible (query block, key block) pairs over every (b, head): the
  // tensor-core form wins from about 2^25 of them (image-zorder-16k, 32 heads
  // of 1024 x 1024 pairs, sits at the break-even; gqa-clustered-32k, 1.8M
  // causal pairs, is 3x faster in the fp32 form)
  const int64_t pairs = p->causal ? nqb * nb / 2 : nqb * nb;
  return static_cast<int64_t>(p->B) * p->Hq * pairs >= (static_cast<int64_t>(1) << 25);
}

// bytes of the tensor-core router's pre-split key image (tiles of 128 key
// blocks, bf16 hi / lo in the MMA layout) and of its norms, or 0 when the
// fp32 form routes this problem
size_t route_img_bytes(const ssa_params* p, size_t* nrm_offset) {
  if (!use_tc_router(p)) return 0;
  const size_t tiles = static_cast<size_t>(p->N / p->block_k + ssa::kRtcNT - 1) / ssa::kRtcNT;
  const size_t heads_tiles = static_cast<size_t>(p->B) * p->Hkv * tiles;
  const size_t img = align256(heads_tiles * 2 * ssa::kRtcNT * p->D * 2);
  if (nrm_offset) *nrm_offset = img;
  return img + align256(heads_tiles * ssa::kRtcNT * sizeof(float));
}

template <int D>
cudaError_t launch_rtc_split(const ssa::RouteArgs& a, int B, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(B) * a.Hkv * a.k_tiles * ssa::kRtcNT;
  const int64_t threads = rows * (D / 8);
  ssa::rtc_split_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      a.ksum, const_cast<uint8_t*>(a.kimg), const_cast<float*>(a.knrm), a.NB, a.k_tiles, rows);
  return cudaGetLastError();
}

// img (optional, route_img_bytes of scratch): with the tensor-core form the
// key summaries are split once into it and every CTA copies its tiles
ssa_status launch_route(const ssa_params* p, const float* qsum, const float* ksum, int32_t* idx,
                        int32_t* cnt, cudaStream_t stream, uint8_t* img = nullptr) {
  ssa::RouteArgs a;
  a.qsum = qsum;
  a.ksum = ksum;
  a.idx = idx;
  a.cnt = cnt;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.NQB = p->N / p->block_q;
  a.NB = p->N / p->block_k;
  a.Bq = p->block_q;
  a.Bk = p->block_k;
  a.top_k = p->top_k;
  a.causal = p->causal;
  a.n_row_tiles = 0;
  a.timeout_ns = timeout_ns(p);
  cudaError_t e;
  if (use_tc_router(p)) {
    size_t nrm_off = 0;
    if (img != nullptr && route_img_bytes(p, &nrm_off) > 0) {
      a.kimg = img;
      a.knrm = reinterpret_cast<const float*>(img + nrm_off);
      a.k_tiles = (a.NB + ssa::kRtcNT - 1) / ssa::kRtcNT;
      e = p->D == 64 ? launch_rtc_split<64>(a, p->B, stream) : launch_rtc_split<128>(a, p->B, stream);
      if (e != cudaSuccess) return cuda_fail(e, "rtc_split_kernel launch");
    }
    e = p->D == 64 ? launch_route_tc<64>(a, p->B, stream) : launch_route_tc<128>(a, p->B, stream);
  } else {
    e = p->D == 64 ? launch_route_fp32<64>(a, p->B, stream) : launch_route_fp32<128>(a, p->B, stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "route_kernel launch");
  return SSA_OK;
}

// ------------------------------------------------------------ two-level route
ssa_status launch_tree_pool(const ssa_params* p, const float* ksum, float* ksum2,
                            cudaStream_t stream) {
  const int32_t nb = p->N / p->block_k, ns = nb / p->tree_fanout;
  ssa::TreePoolArgs a{ksum, ksum2, static_cast<int64_t>(p->B) * p->Hkv * ns, nb, ns,
                      p->tree_fanout, 1.0f / static_cast<float>(p->tree_fanout)};
  const int64_t threads = a.n_nodes * (p->D / 4);
  const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
  if (grid > 0) {
    if (p->D == 64)
      ssa::tree_pool_kernel<64><<<grid, 256, 0, stream>>>(a);
    else
      ssa::tree_pool_kernel<128><<<grid, 256, 0, stream>>>(a);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "tree_pool_kernel launch");
  return SSA_OK;
}

template <int D, int KM>
cudaError_t launch_tree_select_t(const ssa::TreeSelectArgs& a, cudaStream_t stream) {
  const int64_t grid = (a.n_rows + ssa::kTreeWarps - 1) / ssa::kTreeWarps;
  ssa::tree_select_kernel<D, KM><<<static_cast<unsigned>(grid), ssa::kTreeThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_tree_select_d(const ssa::TreeSelectArgs& a, cudaStream_t stream) {
  if (a.top_k <= 8) return launch_tree_select_t<D, 8>(a, stream);
  if (a.top_k <= 16) return launch_tree_select_t<D, 16>(a, stream);
  if (a.top_k <= 32) return launch_tree_select_t<D, 32>(a, stream);
  return launch_tree_select_t<D, 64>(a, stream);
}

// upper level: the flat router over the super-block summaries (block F*Bk,
// top tree_beam); lower level: tree_select_kernel
ssa_status launch_route_tree(const ssa_params* p, const float* qsum, const float* ksum,
                             const float* ksum2, int32_t* sup_idx, int32_t* sup_cnt, int32_t* idx,
                             int32_t* cnt, cudaStream_t stream) {
  const int32_t nb = p->N / p->block_k;
  ssa::RouteArgs u;
  u.qsum = qsum;
  u.ksum = ksum2;
  u.idx = sup_idx;
  u.cnt = sup_cnt;
  u.Hq = p->Hq;
  u.Hkv = p->Hkv;
  u.NQB = p->N / p->block_q;
  u.NB = nb / p->tree_fanout;
  u.Bq = p->block_q;
  u.Bk = p->block_k * p->tree_fanout;
  u.top_k = p->tree_beam;
  u.causal = p->causal;
  u.n_row_tiles = 0;
  u.timeout_ns = timeout_ns(p);
  cudaError_t e = p->D == 64 ? launch_route_fp32<64>(u, p->B, stream)
                             : launch_route_fp32<128>(u, p->B, stream);
  if (e != cudaSuccess) return cuda_fail(e, "tree upper-level route launch");
  ssa::TreeSelectArgs a;
  a.qsum = qsum;
  a.ksum = ksum;
  a.sup_idx = sup_idx;
  a.sup_cnt = sup_cnt;
  a.idx = idx;
  a.cnt = cnt;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.NQB = p->N / p->block_q;
  a.NB = nb;
  a.Bq = p->block_q;
  a.Bk = p->block_k;
  a.top_k = p->top_k;
  a.causal = p->causal;
  int lf = 0;
  while ((1 << lf) < p->tree_fanout) ++lf;
  a.log2_f = lf;
  a.beam = p->tree_beam;
  a.n_rows = static_cast<int64_t>(p->B) * p->Hq * a.NQB;
  e = p->D == 64 ? launch_tree_select_d<64>(a, stream) : launch_tree_select_d<128>(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "tree_select_kernel launch");
  return SSA_OK;
}

// ------------------------------------------------------------------ backward
// The CUDA-core form (SSA_BWD=simt, kept as a comparison) needs delta only;
// the tensor-core form also keeps the list transpose (one bit per key tile of
// 128 keys and query chunk of 64 queries, per list head).
struct BwdWs {
  size_t delta, lse2, map, map_bytes, part_dk, part_dv, total;
  int32_t n_ktiles, map_words;
};

BwdWs bwd_ws_layout(const ssa_params* p) {
  BwdWs w;
  const size_t rows = align256(static_cast<size_t>(p->B) * p->Hq * p->N * sizeof(float));
  w.delta = 0;
  w.lse2 = rows;
  w.map = 2 * rows;
  w.n_ktiles = (p->N + ssa::kBkKT - 1) / ssa::kBkKT;
  const int32_t nqc = (p->N + ssa::kBkQC - 1) / ssa::kBkQC;
  w.map_words = (nqc + 31) / 32;
  const int32_t lh = p->consensus ? p->Hkv : p->Hq;
  w.map_bytes = static_cast<size_t>(p->B) * lh * w.n_ktiles * w.map_words * sizeof(uint32_t);
  // per-query-head shares of dk and dv when a KV head serves several query
  // heads (summed in head order afterwards)
  const size_t part = p->Hq > p->Hkv
                          ? align256(static_cast<size_t>(p->B) * p->Hq * p->N * p->D * sizeof(float))
                          : 0;
  w.part_dk = w.map + align256(w.map_bytes);
  w.part_dv = w.part_dk + part;
  w.total = w.part_dv + part;
  return w;
}

size_t bwd_ws_bytes(const ssa_params* p) { return bwd_ws_layout(p).total; }

bool use_simt_backward() {
  const char* env = std::getenv("SSA_BWD");
  return env != nullptr && std::string(env) == "simt";
}

template <int D>
cudaError_t launch_backward_d(const ssa::BwdArgs& a, int B, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(B) * a.Hq * a.N;
  ssa::bwd_delta_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(a, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = ssa::bwd_smem_bytes<D>();
  e = cudaFuncSetAttribute(ssa::bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  ssa::bwd_kernel<D><<<dim3(a.N / a.RT, B * a.Hq), ssa::kBwdThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// the two tensor-core kernels of the backward: maps[0..3] = Q, G (128-row
// boxes), K, V (the forward's key boxes) for the query-major dq kernel;
// maps[4..7] = Q, G (64-row boxes), K, V (128-row boxes) for the key-major
// dk / dv kernel
template <int D>
cudaError_t launch_backward_tc_d(const CUtensorMap* maps, const ssa::BwdTcArgs& a, int B,
                                 int Hkv, int64_t n_qctas, cudaStream_t stream) {
  const uint32_t smem_dq = ssa::DqLayout<D>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(
      ssa::bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_dq));
  if (e != cudaSuccess) return e;
  ssa::bwd_dq_kernel<D><<<static_cast<unsigned>(n_qctas), ssa::kAtThreads, smem_dq, stream>>>(
      maps[0], maps[1], maps[2], maps[3], a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const uint32_t smem_kv = ssa::DkvLayout<D>::SMEM_BYTES;
  e = cudaFuncSetAttribute(ssa::bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem_kv));
  if (e != cudaSuccess) return e;
  const int64_t n_kctas = static_cast<int64_t>(B) * a.at.Hq * a.n_ktiles;
  ssa::bwd_dkdv_kernel<D>
      <<<static_cast<unsigned>(n_kctas), ssa::DkvLayout<D>::THREADS, smem_kv, stream>>>(
          maps[4], maps[5], maps[6], maps[7], a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.at.Hq == Hkv) return e;
  const int64_t n4 = static_cast<int64_t>(B) * Hkv * a.at.N * (D / 4);
  ssa::bwd_group_sum_kernel<D><<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, stream>>>(a, n4);
  return cudaGetLastError();
}

// Query heads per attend CTA.  Consensus lists are shared by a KV group, so
// two heads of the group fill one 128-row tile (64 rows each) and every chunk
// serves all rows.  SSA_PACK=1 forces one head per tile (the tests run both).
int attend_pack(const ssa_params* p) {
  if (!p->consensus || p->Hq / p->Hkv < 2) return 1;
  const char* env = std::getenv("SSA_PACK");
  if (env != nullptr && std::string(env) == "1") return 1;
  return 2;
}

template <int D>
cudaError_t launch_attend_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const ssa::AttendArgs& a, int n_ctas, cudaStream_t stream) {
  const uint32_t smem = ssa::AtLayout<D>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(ssa::attend_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  ssa::attend_kernel<D><<<n_ctas, ssa::kAtThreads, smem, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

ssa_status launch_attend(const ssa_params* p, const void* q, const void* k, const void* v,
                         const int32_t* idx, const int32_t* cnt, void* o, float* lse,
                         cudaStream_t stream) {
  ssa_status s = get_encoder();
  if (s != SSA_OK) return s;
  CUtensorMap tq, tk, tv;
  const int pack = attend_pack(p);
  const uint32_t kv_rows = static_cast<uint32_t>(p->block_k < 64 ? p->block_k : 64);
  const uint32_t q_rows = static_cast<uint32_t>(ssa::kAtQT / pack);
  if ((s = make_map(&tq, q, static_cast<int64_t>(p->B) * p->Hq, p->N, p->D, q_rows)) != SSA_OK)
    return s;
  if ((s = make_map(&tk, k, static_cast<int64_t>(p->B) * p->Hkv, p->N, p->D, kv_rows)) != SSA_OK)
    return s;
  if ((s = make_map(&tv, v, static_cast<int64_t>(p->B) * p->Hkv, p->N, p->D, kv_rows)) != SSA_OK)
    return s;
  ssa::AttendArgs a;
  a.idx = idx;
  a.cnt = cnt;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.N = p->N;
  a.NQB = p->N / p->block_q;
  a.NB = p->N / p->block_k;
  a.Bq = p->block_q;
  a.Bk = p->block_k;
  a.top_k = p->top_k;
  a.window = p->window;
  a.causal = p->causal;
  a.idx_heads = p->consensus ? p->Hkv : p->Hq;
  a.pack = pack;
  a.n_qtiles = (p->N + static_cast<int32_t>(q_rows) - 1) / static_cast<int32_t>(q_rows);
  const float scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->D));
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = timeout_ns(p);
  const int64_t head_tiles = pack == 1 ? static_cast<int64_t>(p->B) * p->Hq
                                       : static_cast<int64_t>(p->B) * p->Hkv *
                                             ((p->Hq / p->Hkv + 1) / 2);
  const int64_t n_ctas = head_tiles * a.n_qtiles;
  if (n_ctas > 0x7FFFFFFF) return fail(SSA_ERR_UNSUPPORTED, "too many query tiles");
  const cudaError_t e =
      p->D == 64 ? launch_attend_t<64>(tq, tk, tv, a, static_cast<int>(n_ctas), stream)
                 : launch_attend_t<128>(tq, tk, tv, a, static_cast<int>(n_ctas), stream);
  if (e != cudaSuccess) return cuda_fail(e, "attend_kernel launch");
  return SSA_OK;
}

// ------------------------------------------------ second-cumulant routing
int64_t cum_features(const ssa_params* p) { return p->D + static_cast<int64_t>(p->D) * (p->D + 1) / 2; }

template <int D>
cudaError_t launch_cum_features_t(const ssa::CumFeatArgs& a, cudaStream_t stream) {
  const size_t smem = ssa::cumulant_features_smem<D>(a.block);
  cudaError_t e = cudaFuncSetAttribute(ssa::cumulant_features_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  ssa::cumulant_features_kernel<D><<<static_cast<unsigned>(a.n_blocks), ssa::kCumThreads, smem,
                                     stream>>>(a);
  return cudaGetLastError();
}

ssa_status launch_cum_features(const ssa_params* p, const void* x, int32_t H, int32_t block,
                               int32_t queries, float* out, cudaStream_t stream) {
  ssa::CumFeatArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.out = out;
  a.n_blocks = static_cast<int64_t>(p->B) * H * (p->N / block);
  a.block = block;
  a.queries = queries;
  a.half_beta = 0.5f * p->beta;
  if (a.n_blocks > 0x7FFFFFFF) return fail(SSA_ERR_UNSUPPORTED, "too many blocks");
  if (a.n_blocks == 0) return SSA_OK;
  const cudaError_t e = p->D == 64 ? launch_cum_features_t<64>(a, stream)
                                   : launch_cum_features_t<128>(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cumulant_features_kernel launch");
  return SSA_OK;
}

ssa_status launch_cum_route(const ssa_params* p, const float* qf, const float* kf, float* scores,
                            int32_t* idx, int32_t* cnt, cudaStream_t stream) {
  ssa::CumScoreArgs sa;
  sa.qf = qf;
  sa.kf = kf;
  sa.scores = scores;
  sa.Hq = p->Hq;
  sa.Hkv = p->Hkv;
  sa.NQB = p->N / p->block_q;
  sa.NB = p->N / p->block_k;
  sa.Bq = p->block_q;
  sa.Bk = p->block_k;
  sa.causal = p->causal;
  sa.n_row_tiles = (sa.NQB + ssa::kCumTile - 1) / ssa::kCumTile;
  sa.n_cand_tiles = (sa.NB + ssa::kCumTile - 1) / ssa::kCumTile;
  cudaError_t e;
  if (p->top_k > 0) {
    const int64_t gx = static_cast<int64_t>(sa.n_row_tiles) * sa.n_cand_tiles;
    const int64_t gy = static_cast<int64_t>(p->B) * p->Hq;
    if (gx > 0x7FFFFFFF || gy > 65535) return fail(SSA_ERR_UNSUPPORTED, "score grid too large");
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    if (p->D == 64)
      ssa::cumulant_scores_kernel<64><<<grid, ssa::kCumThreads, 0, stream>>>(sa);
    else
      ssa::cumulant_scores_kernel<128><<<grid, ssa::kCumThreads, 0, stream>>>(sa);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "cumulant_scores_kernel launch");
  }
  ssa::CumSelectArgs c;
  c.scores = scores;
  c.idx = idx;
  c.cnt = cnt;
  c.NQB = sa.NQB;
  c.NB = sa.NB;
  c.Bq = p->block_q;
  c.Bk = p->block_k;
  c.top_k = p->top_k;
  c.causal = p->causal;
  c.n_rows = static_cast<int64_t>(p->B) * p->Hq * sa.NQB;
  const int64_t grid = (c.n_rows + 7) / 8;
  if (grid > 0x7FFFFFFF) return fail(SSA_ERR_UNSUPPORTED, "too many query blocks");
  const unsigned g = static_cast<unsigned>(grid);
  if (p->top_k <= 8)
    ssa::cumulant_select_kernel<8><<<g, ssa::kCumThreads, 0, stream>>>(c);
  else if (p->top_k <= 16)
    ssa::cumulant_select_kernel<16><<<g, ssa::kCumThreads, 0, stream>>>(c);
  else if (p->top_k <= 32)
    ssa::cumulant_select_kernel<32><<<g, ssa::kCumThreads, 0, stream>>>(c);
  else
    ssa::cumulant_select_kernel<64><<<g, ssa::kCumThreads, 0, stream>>>(c);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "cumulant_select_kernel launch");
  return SSA_OK;
}

ssa_status launch_consensus(const ssa_params* p, const int32_t* idx, const int32_t* cnt,
                            int32_t* idx_kv, int32_t* cnt_kv, cudaStream_t stream) {
  ssa::ConsensusArgs a;
  a.idx = idx;
  a.cnt = cnt;
  a.idx_kv = idx_kv;
  a.cnt_kv = cnt_kv;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.NQB = p->N / p->block_q;
  a.NB = p->N / p->block_k;
  a.top_k = p->top_k;
  a.n_rows = static_cast<int64_t>(p->B) * p->Hkv * a.NQB;
  const int64_t grid = (a.n_rows + ssa::kConsWarps - 1) / ssa::kConsWarps;
  if (grid > 0x7FFFFFFF) return fail(SSA_ERR_UNSUPPORTED, "too many query blocks");
  int P = 32;
  while (P < (p->Hq / p->Hkv) * p->top_k) P <<= 1;
  const unsigned gr = static_cast<unsigned>(grid);
  switch (P) {
    case 32: ssa::consensus_kernel<1><<<gr, ssa::kConsThreads, 0, stream>>>(a); break;
    case 64: ssa::consensus_kernel<2><<<gr, ssa::kConsThreads, 0, stream>>>(a); break;
    case 128: ssa::consensus_kernel<4><<<gr, ssa::kConsThreads, 0, stream>>>(a); break;
    case 256: ssa::consensus_kernel<8><<<gr, ssa::kConsThreads, 0, stream>>>(a); break;
    default: ssa::consensus_kernel<16><<<gr, ssa::kConsThreads, 0, stream>>>(a); break;
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "consensus_kernel launch");
  return SSA_OK;
}

// Workspace of ssa_forward: K and Q summaries, the per-head routed lists and
// counts, and (consensus routing only) the per-group lists and counts.
struct WsLayout {
  size_t ksum, qsum, idx, cnt, idx_kv, cnt_kv, qf, kf, sc, ksum2, sup_idx, sup_cnt, kimg, total;
};

WsLayout ws_layout(const ssa_params* p) {
  WsLayout w;
  const size_t nb = p->N / p->block_k, nqb = p->N / p->block_q;
  const size_t ks = static_cast<size_t>(p->B) * p->Hkv * nb * p->D * sizeof(float);
  const size_t qs = static_cast<size_t>(p->B) * p->Hq * nqb * p->D * sizeof(float);
  const size_t ix = static_cast<size_t>(p->B) * p->Hq * nqb * p->top_k * sizeof(int32_t);
  const size_t cn = static_cast<size_t>(p->B) * p->Hq * nqb * sizeof(int32_t);
  const size_t g = static_cast<size_t>(p->Hq / p->Hkv);
  const size_t ixk = p->consensus ? ix / g : 0, cnk = p->consensus ? cn / g : 0;
  w.ksum = 0;
  w.qsum = align256(ks);
  w.idx = w.qsum + align256(qs);
  w.cnt = w.idx + align256(ix);
  w.idx_kv = w.cnt + align256(cn);
  w.cnt_kv = w.idx_kv + align256(ixk);
  // second-cumulant routing: query and key features, and the score matrix
  const bool cum = p->beta != 0.0f;
  const size_t F = static_cast<size_t>(cum_features(p));
  const size_t qfb = cum ? static_cast<size_t>(p->B) * p->Hq * nqb * F * sizeof(float) : 0;
  const size_t kfb = cum ? static_cast<size_t>(p->B) * p->Hkv * nb * F * sizeof(float) : 0;
  const size_t scb = cum ? static_cast<size_t>(p->B) * p->Hq * nqb * nb * sizeof(float) : 0;
  w.qf = w.cnt_kv + align256(cnk);
  w.kf = w.qf + align256(qfb);
  w.sc = w.kf + align256(kfb);
  // two-level routing: super-block summaries and the kept super-blocks
  const bool tree = p->tree_fanout > 0;
  const size_t ns = tree ? nb / p->tree_fanout : 0;
  const size_t k2b = static_cast<size_t>(p->B) * p->Hkv * ns * p->D * sizeof(float);
  const size_t s2b = tree ? static_cast<size_t>(p->B) * p->Hq * nqb * p->tree_beam * sizeof(int32_t) : 0;
  const size_t c2b = tree ? cn : 0;
  w.ksum2 = w.sc + align256(scb);
  w.sup_idx = w.ksum2 + align256(k2b);
  w.sup_cnt = w.sup_idx + align256(s2b);
  // flat routing in the tensor-core form: the pre-split key image
  const size_t imgb = (!cum && !tree) ? route_img_bytes(p, nullptr) : 0;
  w.kimg = w.sup_cnt + align256(c2b);
  w.total = w.kimg + imgb;
  return w;
}

// ------------------------------------------------------------------ decode
int decode_km(int32_t top_k) { return top_k <= 8 ? 8 : top_k <= 16 ? 16 : top_k <= 32 ? 32 : 64; }

size_t decode_ws_bytes(const ssa_params* p) {
  const size_t heads = static_cast<size_t>(p->B) * p->Hq;
  return align256(heads * ssa::kDecMaxSplits * decode_km(p->top_k) * sizeof(uint64_t)) +
         align256(heads * ssa::kDecMaxSplits * (p->D + 2) * sizeof(float)) +
         align256(heads * sizeof(uint32_t));
}

ssa_status validate_decode(const ssa_params* p) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (!p->causal) return fail(SSA_ERR_INVALID_ARG, "decode is causal (causal must be 1)");
  if (p->consensus) return fail(SSA_ERR_UNSUPPORTED, "decode routes per head (consensus must be 0)");
  if (p->beta != 0.0f) return fail(SSA_ERR_UNSUPPORTED, "decode ranks by block means (beta must be 0)");
  if (p->tree_fanout != 0)
    return fail(SSA_ERR_UNSUPPORTED, "decode routes over the flat block list (tree_fanout must be 0)");
  if (static_cast<int64_t>(p->B) * p->Hq > 65535)
    return fail(SSA_ERR_UNSUPPORTED, "decode needs B * Hq <= 65535");
  return SSA_OK;
}

template <int D, int KM>
cudaError_t launch_decode_t(const ssa::DecodeArgs& a, int B, cudaStream_t stream) {
  const size_t rs = ssa::decode_route_smem<D>(a.Hq / a.Hkv, a.cands_per_split);
  cudaError_t e = cudaFuncSetAttribute(ssa::decode_route_kernel<D, KM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(rs));
  if (e != cudaSuccess) return e;
  ssa::decode_route_kernel<D, KM><<<dim3(a.S, B * a.Hkv), ssa::kDecThreads, rs, stream>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t as = ssa::decode_attend_smem<D>();
  e = cudaFuncSetAttribute(ssa::decode_attend_kernel<D, KM>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(as));
  if (e != cudaSuccess) return e;
  ssa::decode_attend_kernel<D, KM><<<dim3(a.KS, B * a.Hq), ssa::kDecThreads, as, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_d(const ssa::DecodeArgs& a, int B, cudaStream_t stream) {
  switch (decode_km(a.top_k)) {
    case 8: return launch_decode_t<D, 8>(a, B, stream);
    case 16: return launch_decode_t<D, 16>(a, B, stream);
    case 32: return launch_decode_t<D, 32>(a, B, stream);
    default: return launch_decode_t<D, 64>(a, B, stream);
  }
}

}  // namespace

extern "C" {

size_t ssa_workspace_size(const ssa_params* p) {
  if (validate(p) != SSA_OK) return 0;
  return ws_layout(p).total;
}

ssa_status ssa_block_summary(const ssa_params* p, const void* x, int32_t H, int32_t block,
                             float* out, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (x == nullptr || out == nullptr) return fail(SSA_ERR_INVALID_ARG, "x and out must be non-NULL");
  if (!aligned16(x) || !aligned16(out))
    return fail(SSA_ERR_INVALID_ARG, "x and out must be 16-byte aligned");
  if (H < 1) return fail(SSA_ERR_INVALID_ARG, "H must be positive");
  if (!pow2_in(block, 1, 1 << 20) || p->N % block != 0)
    return fail(SSA_ERR_INVALID_ARG, "block must be a power of two dividing N");
  s = launch_pool(p, x, H, block, out, nullptr, 0, 0, nullptr, static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_route(const ssa_params* p, const float* qsum, const float* ksum, int32_t* idx,
                     int32_t* cnt, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (p->beta != 0.0f)
    return fail(SSA_ERR_INVALID_ARG,
                "beta != 0: route with ssa_route_features and ssa_route_cumulant");
  if (qsum == nullptr || ksum == nullptr || cnt == nullptr || (p->top_k > 0 && idx == nullptr))
    return fail(SSA_ERR_INVALID_ARG, "qsum, ksum, cnt (and idx when top_k > 0) must be non-NULL");
  if (!aligned16(qsum) || !aligned16(ksum) || !aligned16(cnt) || (idx && !aligned16(idx)))
    return fail(SSA_ERR_INVALID_ARG, "routing buffers must be 16-byte aligned");
  s = launch_route(p, qsum, ksum, idx, cnt, static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

size_t ssa_route_workspace_size(const ssa_params* p) {
  if (validate(p) != SSA_OK || p->beta != 0.0f) return 0;
  return route_img_bytes(p, nullptr);
}

ssa_status ssa_route_with_workspace(const ssa_params* p, const float* qsum, const float* ksum,
                                    int32_t* idx, int32_t* cnt, void* workspace,
                                    size_t workspace_bytes, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (p->beta != 0.0f)
    return fail(SSA_ERR_INVALID_ARG,
                "beta != 0: route with ssa_route_features and ssa_route_cumulant");
  if (qsum == nullptr || ksum == nullptr || cnt == nullptr || (p->top_k > 0 && idx == nullptr))
    return fail(SSA_ERR_INVALID_ARG, "qsum, ksum, cnt (and idx when top_k > 0) must be non-NULL");
  if (!aligned16(qsum) || !aligned16(ksum) || !aligned16(cnt) || (idx && !aligned16(idx)))
    return fail(SSA_ERR_INVALID_ARG, "routing buffers must be 16-byte aligned");
  const size_t need = route_img_bytes(p, nullptr);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(SSA_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  s = launch_route(p, qsum, ksum, idx, cnt, static_cast<cudaStream_t>(stream),
                   need > 0 ? static_cast<uint8_t*>(workspace) : nullptr);
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_tree_summary(const ssa_params* p, const float* ksum, float* ksum2,
                            ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (p->tree_fanout < 1) return fail(SSA_ERR_INVALID_ARG, "tree_fanout must be >= 1");
  if (ksum == nullptr || ksum2 == nullptr)
    return fail(SSA_ERR_INVALID_ARG, "ksum and ksum2 must be non-NULL");
  if (!aligned16(ksum) || !aligned16(ksum2))
    return fail(SSA_ERR_INVALID_ARG, "ksum and ksum2 must be 16-byte aligned");
  s = launch_tree_pool(p, ksum, ksum2, static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_route_tree(const ssa_params* p, const float* qsum, const float* ksum,
                          const float* ksum2, int32_t* sup_idx, int32_t* sup_cnt, int32_t* idx,
                          int32_t* cnt, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (p->tree_fanout < 1) return fail(SSA_ERR_INVALID_ARG, "tree_fanout must be >= 1");
  if (!qsum || !ksum || !ksum2 || !sup_idx || !sup_cnt || !cnt || (p->top_k > 0 && !idx))
    return fail(SSA_ERR_INVALID_ARG,
                "qsum, ksum, ksum2, sup_idx, sup_cnt, cnt (and idx when top_k > 0) must be non-NULL");
  if (!aligned16(qsum) || !aligned16(ksum) || !aligned16(ksum2) || !aligned16(sup_idx) ||
      !aligned16(sup_cnt) || !aligned16(cnt) || (idx && !aligned16(idx)))
    return fail(SSA_ERR_INVALID_ARG, "routing buffers must be 16-byte aligned");
  s = launch_route_tree(p, qsum, ksum, ksum2, sup_idx, sup_cnt, idx, cnt,
                        static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_route_consensus(const ssa_params* p, const int32_t* idx, const int32_t* cnt,
                               int32_t* idx_kv, int32_t* cnt_kv, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if ((p->Hq / p->Hkv) * p->top_k > ssa::kConsMaxVotes)
    return fail(SSA_ERR_UNSUPPORTED, "consensus routing needs (Hq / Hkv) * top_k <= %d",
                ssa::kConsMaxVotes);
  if (cnt == nullptr || cnt_kv == nullptr || (p->top_k > 0 && (idx == nullptr || idx_kv == nullptr)))
    return fail(SSA_ERR_INVALID_ARG, "cnt, cnt_kv (and idx, idx_kv when top_k > 0) must be non-NULL");
  if (!aligned16(cnt) || !aligned16(cnt_kv) || (idx && !aligned16(idx)) ||
      (idx_kv && !aligned16(idx_kv)))
    return fail(SSA_ERR_INVALID_ARG, "routing buffers must be 16-byte aligned");
  s = launch_consensus(p, idx, cnt, idx_kv, cnt_kv, static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_route_features(const ssa_params* p, const void* x, int32_t H, int32_t block,
                              int32_t queries, float* out, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (x == nullptr || out == nullptr) return fail(SSA_ERR_INVALID_ARG, "x and out must be non-NULL");
  if (!aligned16(x) || !aligned16(out))
    return fail(SSA_ERR_INVALID_ARG, "x and out must be 16-byte aligned");
  if (H < 1) return fail(SSA_ERR_INVALID_ARG, "H must be positive");
  if (queries != 0 && queries != 1) return fail(SSA_ERR_INVALID_ARG, "queries must be 0 or 1");
  if (!pow2_in(block, 1, 128) || p->N % block != 0)
    return fail(SSA_ERR_INVALID_ARG, "block must be a power of two <= 128 dividing N");
  s = launch_cum_features(p, x, H, block, queries, out, static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_route_cumulant(const ssa_params* p, const float* qfeat, const float* kfeat,
                              float* scores, int32_t* idx, int32_t* cnt, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (!qfeat || !kfeat || !scores || !cnt || (p->top_k > 0 && !idx))
    return fail(SSA_ERR_INVALID_ARG,
                "qfeat, kfeat, scores, cnt (and idx when top_k > 0) must be non-NULL");
  if (!aligned16(qfeat) || !aligned16(kfeat) || !aligned16(scores) || !aligned16(cnt) ||
      (idx && !aligned16(idx)))
    return fail(SSA_ERR_INVALID_ARG, "routing buffers must be 16-byte aligned");
  s = launch_cum_route(p, qfeat, kfeat, scores, idx, cnt, static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_attend(const ssa_params* p, const void* q, const void* k, const void* v,
                      const int32_t* idx, const int32_t* cnt, void* o, float* lse,
                      ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (!q || !k || !v || !o || !cnt || (p->top_k > 0 && !idx))
    return fail(SSA_ERR_INVALID_ARG, "q, k, v, o, cnt (and idx when top_k > 0) must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return fail(SSA_ERR_INVALID_ARG, "q, k, v, o and lse must be 16-byte aligned");
  s = launch_attend(p, q, k, v, idx, cnt, o, lse, static_cast<cudaStream_t>(stream));
  return s == SSA_OK ? ok() : s;
}

ssa_status ssa_forward(const ssa_params* p, const void* q, const void* k, const void* v, void* o,
                       float* lse, int32_t* idx_out, int32_t* cnt_out, void* workspace,
                       size_t workspace_bytes, ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (!q || !k || !v || !o) return fail(SSA_ERR_INVALID_ARG, "q, k, v, o must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)) ||
      (idx_out && !aligned16(idx_out)) || (cnt_out && !aligned16(cnt_out)))
    return fail(SSA_ERR_INVALID_ARG, "all buffers must be 16-byte aligned");
  const WsLayout w = ws_layout(p);
  if (workspace == nullptr || workspace_bytes < w.total)
    return fail(SSA_ERR_WORKSPACE, "workspace needs %zu bytes", w.total);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* ksum = reinterpret_cast<float*>(ws + w.ksum);
  float* qsum = reinterpret_cast<float*>(ws + w.qsum);
  // the lists attend reads: per head, or per KV group with consensus routing;
  // the caller's idx_out / cnt_out receive them when given
  int32_t* idx_h = reinterpret_cast<int32_t*>(ws + w.idx);
  int32_t* cnt_h = reinterpret_cast<int32_t*>(ws + w.cnt);
  int32_t* idx_a = p->consensus ? reinterpret_cast<int32_t*>(ws + w.idx_kv) : idx_h;
  int32_t* cnt_a = p->consensus ? reinterpret_cast<int32_t*>(ws + w.cnt_kv) : cnt_h;
  if (idx_out) idx_a = idx_out;
  if (cnt_out) cnt_a = cnt_out;
  if (!p->consensus) {
    idx_h = idx_a;
    cnt_h = cnt_a;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->beta != 0.0f) {
    float* qf = reinterpret_cast<float*>(ws + w.qf);
    float* kf = reinterpret_cast<float*>(ws + w.kf);
    float* sc = reinterpret_cast<float*>(ws + w.sc);
    if ((s = launch_cum_features(p, k, p->Hkv, p->block_k, 0, kf, st)) != SSA_OK) return s;
    if ((s = launch_cum_features(p, q, p->Hq, p->block_q, 1, qf, st)) != SSA_OK) return s;
    if ((s = launch_cum_route(p, qf, kf, sc, idx_h, cnt_h, st)) != SSA_OK) return s;
  } else {
    if ((s = launch_pool(p, k, p->Hkv, p->block_k, ksum, q, p->Hq, p->block_q, qsum, st)) != SSA_OK)
      return s;
    if (p->tree_fanout > 0) {
      float* ksum2 = reinterpret_cast<float*>(ws + w.ksum2);
      int32_t* sup_idx = reinterpret_cast<int32_t*>(ws + w.sup_idx);
      int32_t* sup_cnt = reinterpret_cast<int32_t*>(ws + w.sup_cnt);
      if ((s = launch_tree_pool(p, ksum, ksum2, st)) != SSA_OK) return s;
      if ((s = launch_route_tree(p, qsum, ksum, ksum2, sup_idx, sup_cnt, idx_h, cnt_h, st)) !=
          SSA_OK)
        return s;
    } else if ((s = launch_route(p, qsum, ksum, idx_h, cnt_h, st, ws + w.kimg)) != SSA_OK) {
      return s;
    }
  }
  if (p->consensus && (s = launch_consensus(p, idx_h, cnt_h, idx_a, cnt_a, st)) != SSA_OK)
    return s;
  if ((s = launch_attend(p, q, k, v, idx_a, cnt_a, o, lse, st)) != SSA_OK) return s;
  return ok();
}

// Device address of the static scratch on the current device.  It is looked
// up once per device and context: the first call on a device does the
// lookup, and so does the first call after the device's context was made
// anew (after cudaDeviceReset the module is loaded again and the array may
// sit at another address).  Contexts are told apart by the driver's context
// ID, which is unique for the life of the process.
std::mutex g_static_mu;
constexpr int kMaxDevices = 256;
void* g_static_ptr[kMaxDevices] = {};
unsigned long long g_static_ctx[kMaxDevices] = {};
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// ID of the context current on this thread (0 if there is none yet)
ssa_status current_context_id(unsigned long long* id) {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  if (g_ctx_current == nullptr || g_ctx_id == nullptr)
    return fail(SSA_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId are unavailable (no CUDA driver?)");
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return fail(SSA_ERR_CUDA, "cuCtxGetCurrent failed");
  *id = 0;
  if (ctx != nullptr && g_ctx_id(ctx, id) != CUDA_SUCCESS)
    return fail(SSA_ERR_CUDA, "cuCtxGetId failed");
  return SSA_OK;
}

ssa_status static_scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  unsigned long long ctx = 0;
  ssa_status s = current_context_id(&ctx);
  if (s != SSA_OK) return s;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr || ctx == 0 || ctx != g_static_ctx[dev]) {
    void* ptr = nullptr;
    // with this device current; makes its primary context current when no
    // context is yet
    e = cudaGetSymbolAddress(&ptr, ssa::g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    if ((s = current_context_id(&ctx)) != SSA_OK) return s;
    g_static_ptr[dev] = ptr;
    g_static_ctx[dev] = ctx;
  }
  *out = g_static_ptr[dev];
  return SSA_OK;
}

ssa_status ssa_forward_static(const ssa_params* p, const void* q, const void* k, const void* v,
                              void* o, float* lse, int32_t* idx_out, int32_t* cnt_out,
                              ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  const size_t need = ws_layout(p).total;
  if (need > ssa::kStaticScratchBytes)
    return fail(SSA_ERR_WORKSPACE,
                "this shape needs %zu bytes of scratch; the built-in scratch holds %zu bytes "
                "(use ssa_forward with a caller workspace)",
                need, ssa::kStaticScratchBytes);
  void* scratch = nullptr;
  if ((s = static_scratch_address(&scratch)) != SSA_OK) return s;
  // Every buffer in the scratch is fully written by the kernels before it is
  // read (summaries by the pool kernel, lists and counts by the router), so
  // nothing has to be cleared between calls.
  return ssa_forward(p, q, k, v, o, lse, idx_out, cnt_out, scratch, ssa::kStaticScratchBytes,
                     stream);
}

size_t ssa_backward_workspace_size(const ssa_params* p) {
  if (validate(p) != SSA_OK) return 0;
  return bwd_ws_bytes(p);
}

ssa_status ssa_attend_backward(const ssa_params* p, const void* q, const void* k, const void* v,
                               const void* o, const float* lse, const void* d_o,
                               const int32_t* idx, const int32_t* cnt, float* dq, float* dk,
                               float* dv, void* workspace, size_t workspace_bytes,
                               ssa_stream_t stream) {
  ssa_status s = validate(p);
  if (s != SSA_OK) return s;
  if (!q || !k || !v || !o || !lse || !d_o || !cnt || !dq || !dk || !dv || (p->top_k > 0 && !idx))
    return fail(SSA_ERR_INVALID_ARG,
                "q, k, v, o, lse, d_o, cnt, dq, dk, dv (and idx when top_k > 0) must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(d_o) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(SSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const size_t need = bwd_ws_bytes(p);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(SSA_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  ssa::BwdArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.o = static_cast<const __nv_bfloat16*>(o);
  a.d_o = static_cast<const __nv_bfloat16*>(d_o);
  a.lse = lse;
  a.idx = idx;
  a.cnt = cnt;
  a.delta = static_cast<float*>(workspace);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.N = p->N;
  a.Bq = p->block_q;
  a.Bk = p->block_k;
  a.top_k = p->top_k;
  a.window = p->window;
  a.causal = p->causal;
  a.list_heads = p->consensus ? p->Hkv : p->Hq;
  a.NQB = p->N / p->block_q;
  a.NB = p->N / p->block_k;
  a.RT = std::min(p->block_q, p->D == 64 ? ssa::bwd_rows<64>() : ssa::bwd_rows<128>());
  a.CK = std::min(p->block_k, p->D == 64 ? ssa::bwd_keys<64>() : ssa::bwd_keys<128>());
  a.scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->D));
  if (use_simt_backward()) {
    // CUDA-core form: dk / dv are accumulated with atomics, so clear them
    const size_t kv_bytes = static_cast<size_t>(p->B) * p->Hkv * p->N * p->D * sizeof(float);
    e = cudaMemsetAsync(dk, 0, kv_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "clear dk / dv");
    e = p->D == 64 ? launch_backward_d<64>(a, p->B, st) : launch_backward_d<128>(a, p->B, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return ok();
  }

  // tensor-core form: delta, the list transpose, the query-major dq kernel
  // and the key-major dk / dv kernel
  const BwdWs w = bwd_ws_layout(p);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* map = reinterpret_cast<uint32_t*>(ws + w.map);
  e = cudaMemsetAsync(map, 0, w.map_bytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "clear the list transpose");
  if ((s = get_encoder()) != SSA_OK) return s;
  const int64_t hq = static_cast<int64_t>(p->B) * p->Hq, hkv = static_cast<int64_t>(p->B) * p->Hkv;
  const uint32_t kv_rows = static_cast<uint32_t>(p->block_k < 64 ? p->block_k : 64);
  CUtensorMap maps[8];
  if ((s = make_map(&maps[0], q, hq, p->N, p->D, ssa::kAtQT)) != SSA_OK ||
      (s = make_map(&maps[1], d_o, hq, p->N, p->D, ssa::kAtQT)) != SSA_OK ||
      (s = make_map(&maps[2], k, hkv, p->N, p->D, kv_rows)) != SSA_OK ||
      (s = make_map(&maps[3], v, hkv, p->N, p->D, kv_rows)) != SSA_OK ||
      (s = make_map(&maps[4], q, hq, p->N, p->D, ssa::kBkQC)) != SSA_OK ||
      (s = make_map(&maps[5], d_o, hq, p->N, p->D, ssa::kBkQC)) != SSA_OK ||
      (s = make_map(&maps[6], k, hkv, p->N, p->D, ssa::kBkKT)) != SSA_OK ||
      (s = make_map(&maps[7], v, hkv, p->N, p->D, ssa::kBkKT)) != SSA_OK)
    return s;
  ssa::BwdTcArgs t;
  t.at.idx = idx;
  t.at.cnt = cnt;
  t.at.o = nullptr;
  t.at.lse = nullptr;
  t.at.Hq = p->Hq;
  t.at.Hkv = p->Hkv;
  t.at.N = p->N;
  t.at.NQB = p->N / p->block_q;
  t.at.NB = p->N / p->block_k;
  t.at.Bq = p->block_q;
  t.at.Bk = p->block_k;
  t.at.top_k = p->top_k;
  t.at.window = p->window;
  t.at.causal = p->causal;
  t.at.idx_heads = p->consensus ? p->Hkv : p->Hq;
  t.at.pack = 1;
  t.at.n_qtiles = (p->N + ssa::kAtQT - 1) / ssa::kAtQT;
  t.at.scale_log2 = a.scale * 1.4426950408889634f;
  t.at.timeout_ns = timeout_ns(p);
  t.lse = lse;
  t.delta = a.delta;
  t.delta_w = a.delta;
  t.lse2 = reinterpret_cast<float*>(ws + w.lse2);
  t.o = static_cast<const __nv_bfloat16*>(o);
  t.d_o = static_cast<const __nv_bfloat16*>(d_o);
  t.dq = dq;
  t.dk = dk;
  t.dv = dv;
  t.map = map;
  t.map_w = map;
  t.n_ktiles = w.n_ktiles;
  t.map_words = w.map_words;
  t.B = p->B;
  t.part_dk = p->Hq > p->Hkv ? reinterpret_cast<float*>(ws + w.part_dk) : nullptr;
  t.part_dv = p->Hq > p->Hkv ? reinterpret_cast<float*>(ws + w.part_dv) : nullptr;
  t.scale = a.scale;
  const int64_t rows = static_cast<int64_t>(p->B) * p->Hq * p->N;
  if (p->D == 64)
    ssa::bwd_prep_kernel<64><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(t, rows);
  else
    ssa::bwd_prep_kernel<128><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(t, rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_prep_kernel launch");
  if (p->top_k > 0) {
    const int64_t slots = static_cast<int64_t>(p->B) * t.at.idx_heads * t.at.NQB * p->top_k;
    ssa::bwd_map_kernel<<<static_cast<unsigned>((slots + 255) / 256), 256, 0, st>>>(t, slots);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bwd_map_kernel launch");
  }
  const int64_t n_qctas = hq * t.at.n_qtiles;
  if (n_qctas > 0x7FFFFFFF || hq * w.n_ktiles > 0x7FFFFFFF)
    return fail(SSA_ERR_UNSUPPORTED, "too many tiles");
  e = p->D == 64 ? launch_backward_tc_d<64>(maps, t, p->B, p->Hkv, n_qctas, st)
                 : launch_backward_tc_d<128>(maps, t, p->B, p->Hkv, n_qctas, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  return ok();
}

size_t ssa_decode_workspace_size(const ssa_params* p) {
  if (validate_decode(p) != SSA_OK) return 0;
  return decode_ws_bytes(p);
}

ssa_status ssa_decode(const ssa_params* p, const void* q, const void* k_cache, const void* v_cache,
                      int32_t n_ctx, float* ksum_cache, void* o, float* lse, int32_t* idx_out,
                      int32_t* cnt_out, void* workspace, size_t workspace_bytes,
                      ssa_stream_t stream) {
  ssa_status s = validate_decode(p);
  if (s != SSA_OK) return s;
  if (!q || !k_cache || !v_cache || !ksum_cache || !o)
    return fail(SSA_ERR_INVALID_ARG, "q, k_cache, v_cache, ksum_cache and o must be non-NULL");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(ksum_cache) ||
      !aligned16(o) || (lse && !aligned16(lse)) || (idx_out && !aligned16(idx_out)) ||
      (cnt_out && !aligned16(cnt_out)))
    return fail(SSA_ERR_INVALID_ARG, "all buffers must be 16-byte aligned");
  if (n_ctx < 1 || n_ctx > p->N)
    return fail(SSA_ERR_INVALID_ARG, "n_ctx must be in 1..N (the cache capacity)");
  const size_t need = decode_ws_bytes(p);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(SSA_ERR_WORKSPACE, "decode workspace needs %zu bytes", need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  ssa::DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k_cache);
  a.v = static_cast<const __nv_bfloat16*>(v_cache);
  a.ksum = ksum_cache;
  const size_t heads = static_cast<size_t>(p->B) * p->Hq;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.part_keys = reinterpret_cast<uint64_t*>(ws);
  const size_t keys_bytes = align256(heads * ssa::kDecMaxSplits * decode_km(p->top_k) * sizeof(uint64_t));
  a.part_attn = reinterpret_cast<float*>(ws + keys_bytes);
  a.done = reinterpret_cast<uint32_t*>(
      ws + keys_bytes + align256(heads * ssa::kDecMaxSplits * (p->D + 2) * sizeof(float)));
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.idx = idx_out;
  a.cnt = cnt_out;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.Ncap = p->N;
  a.Bk = p->block_k;
  a.top_k = p->top_k;
  a.window = p->window;
  a.i = n_ctx - 1;
  a.nb = a.i / p->block_k;
  // about two CTAs per SM in each phase; a route split scans >= 32 blocks
  // and a key split >= 128 keys (the attend kernel's warps take 32 keys a
  // step; measured: 256-key minimum 42.4 us, 128-key 39.2 us per step on the
  // 8K-token, 64-head needle cache; unchanged at 1M and 32K tokens)
  const int64_t want_s = (2 * 148 + static_cast<int64_t>(p->B) * p->Hkv - 1) /
                         (static_cast<int64_t>(p->B) * p->Hkv);
  int64_t S = std::min<int64_t>(std::min<int64_t>(ssa::kDecMaxSplits, want_s), (a.nb + 31) / 32);
  S = std::max<int64_t>(S, 1);
  a.cands_per_split = static_cast<int32_t>(std::max<int64_t>(1, (a.nb + S - 1) / S));
  const size_t route_smem = p->D == 64 ? ssa::decode_route_smem<64>(p->Hq / p->Hkv, a.cands_per_split)
                                       : ssa::decode_route_smem<128>(p->Hq / p->Hkv, a.cands_per_split);
  if (route_smem > 200 * 1024)
    return fail(SSA_ERR_UNSUPPORTED, "decode: too many key blocks per routing split for shared memory");
  a.S = static_cast<int32_t>(S);
  const int64_t lmax = static_cast<int64_t>(p->top_k) * p->block_k + p->window;
  const int64_t want_ks = (2 * 148 + static_cast<int64_t>(heads) - 1) / static_cast<int64_t>(heads);
  int64_t KS = std::min<int64_t>(std::min<int64_t>(ssa::kDecMaxSplits, want_ks), (lmax + 127) / 128);
  a.KS = static_cast<int32_t>(std::max<int64_t>(KS, 1));
  const float scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->D));
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = p->D == 64 ? launch_decode_d<64>(a, p->B, st) : launch_decode_d<128>(a, p->B, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode kernels launch");
  return ok();
}

ssa_status ssa_check_error(ssa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t flags = 0, site = 0;
  if ((e = cudaMemcpyFromSymbol(&flags, ssa::g_err_flags, sizeof(flags))) != cudaSuccess)
    return cuda_fail(e, "read error word");
  if ((e = cudaMemcpyFromSymbol(&site, ssa::g_err_site, sizeof(site))) != cudaSuccess)
    return cuda_fail(e, "read error site");
  const uint32_t zero = 0;
  if ((e = cudaMemcpyToSymbol(ssa::g_err_flags, &zero, sizeof(zero))) != cudaSuccess)
    return cuda_fail(e, "clear error word");
  if ((e = cudaMemcpyToSymbol(ssa::g_err_site, &zero, sizeof(zero))) != cudaSuccess)
    return cuda_fail(e, "clear error site");
  if (flags & ssa::kErrTimeout)
    return fail(SSA_ERR_TIMEOUT, "a device-side wait ran out (site %u)", site);
  if (flags & ssa::kErrCheck)
    return fail(SSA_ERR_DEVICE_CHECK, "a device-side check failed (site %u)", site);
  return ok();
}

ssa_status ssa_probe_wait_timeout(int32_t timeout_us, ssa_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 10000000)
    return fail(SSA_ERR_INVALID_ARG, "timeout_us must be in 1..10^7");
  ssa::probe_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "probe_wait_kernel launch");
  return ok();
}

ssa_status ssa_probe_ex2_rate(int32_t n_ctas, int32_t iters, float* sink,
                              ssa_stream_t stream) {
  if (n_ctas < 1 || n_ctas > (1 << 20) || iters < 1 || iters > (1 << 24) || sink == nullptr)
    return fail(SSA_ERR_INVALID_ARG, "n_ctas in 1..2^20, iters in 1..2^24, sink non-NULL");
  ssa::ex2_rate_kernel<<<n_ctas, 256, 0, static_cast<cudaStream_t>(stream)>>>(iters, sink);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "ex2_rate_kernel launch");
  return ok();
}

const char* ssa_status_string(ssa_status s) {
  switch (s) {
    case SSA_OK: return "ok";
    case SSA_ERR_INVALID_ARG: return "invalid argument";
    case SSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SSA_ERR_WORKSPACE: return "workspace too small";
    case SSA_ERR_CUDA: return "CUDA error";
    case SSA_ERR_TIMEOUT: return "device wait timed out";
    case SSA_ERR_DEVICE_CHECK: return "device check failed";
  }
  return "unknown status";
}

const char* ssa_last_error_message(void) { return g_msg.c_str(); }

int32_t ssa_version(void) { return kVersion; }

}  // extern "C"
