// K1: block summaries (mean pooling).
//
// jonsmirl/ssa README, "Algorithm and complexity": each key block c is
// summarised by its mean key mu_c; the query side is summarised the same way
// at the query block size.  out[bh, c, :] = (1/block) * sum_t x[bh, c*block+t, :].
//
// HBM-bound streaming read.  One warp owns one block (see the kernel); the
// sum runs in fp32 and the 1/block factor (a power of two) is exact.  K and Q
// summaries are one launch: the grid covers both jobs back to back.
#pragma once

#include "common.cuh"

namespace ssa {

struct PoolJob {
  const uint4* x;      // bf16 [rows, D] viewed as 16-byte vectors
  float* out;          // fp32 [rows / block, D]
  int64_t n_blocks;    // B * H * (N / block)
  int32_t block;       // rows per block (power of two)
  float inv_block;
};

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] += __uint_as_float(w[i] << 16);
    a[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One warp per block: lane = (row phase rs, 16-byte column group g) with
// G = D/8 groups and RS = 32/G row phases, so one warp instruction reads RS
// consecutive rows = RS*D*2 contiguous bytes.  Each lane sums rows rs, rs+RS,
// ... in fp32; the RS partial sums are combined by shuffles.
template <int D>
__global__ void __launch_bounds__(256) block_mean_kernel(PoolJob j0, PoolJob j1, int64_t split) {
  constexpr int G = D / 8;    // 16-byte vectors per row
  constexpr int RS = 32 / G;  // rows read together by one warp instruction
  const int64_t wglobal = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const bool first = wglobal < split;
  const int64_t blk = first ? wglobal : wglobal - split;
  const uint4* x = first ? j0.x : j1.x;
  float* out = first ? j0.out : j1.out;
  const int64_t n_blocks = first ? j0.n_blocks : j1.n_blocks;
  const int block = first ? j0.block : j1.block;
  const float inv = first ? j0.inv_block : j1.inv_block;
  if (blk >= n_blocks) return;  // warp-uniform

  const int g = lane % G, rs = lane / G;
  const uint4* src = x + blk * block * G + g;
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int r = rs;
  for (; r + 7 * RS < block; r += 8 * RS) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) u[k] = ldg_stream(src + static_cast<int64_t>(r + k * RS) * G);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc_bf16x8(a, u[k]);
  }
  for (; r < block; r += RS) acc_bf16x8(a, ldg_stream(src + static_cast<int64_t>(r) * G));
#pragma unroll
  for (int off = G; off < 32; off <<= 1)
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] += __shfl_xor_sync(0xffffffffu, a[k], off);
  if (rs == 0) {
    // Non-finite inputs are outside the method's domain: a NaN or infinite
    // summary would give NaN routing scores, which rank nowhere.  Report it
    // through the error word (the summary is still written).
    bool finite = true;
#pragma unroll
    for (int k = 0; k < 8; ++k) finite = finite && isfinite(a[k]);
    if (!finite) record_error(kErrCheck, kSitePool);
    float4* dst = reinterpret_cast<float4*>(out + blk * D + g * 8);
    dst[0] = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
    dst[1] = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
  }
}

}  // namespace ssa
