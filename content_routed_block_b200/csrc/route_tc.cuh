// K2 (tensor-core form): routing scores on tcgen05 with a proven error bound,
// then an exact fp32 top-k.
//
// jonsmirl/ssa README, "Algorithm and complexity": block c is scored by
// <q, mu_c> (the second-cumulant weight beta is 0 here) and the top_k
// admissible blocks of each query block are kept; ties go to the lower block
// index.  The ranking must be decided on fp32 scores.  Scoring every
// (query block, key block) pair in fp32 FMA costs NQB*NB*D*2 flops, which is
// 240 GFLOP at a million tokens, so this kernel ranks in two passes:
//
//  pass 1  bf16 tensor-core scores sa_c (M = 128 query blocks, N = 256 or 128
//          key blocks per MMA, fp32 accumulation in TMEM).  With bf16
//          rounding of both operands (unit roundoff u = 2^-9) every score obeys
//          |sa_c - s_c| <= (2u + u^2 + accumulation) ||qbar|| ||mu_c||
//          < 2^-7 ||qbar|| ||mu_c|| =: E_c.  Each row keeps the k largest
//          lower bounds sa_c - E_c; L is the k-th of them.
//  pass 2  the same tensor-core scores again; every candidate whose upper
//          bound sa_c + E_c reaches L is rescored exactly in fp32 (sequential
//          FMA over d, the same arithmetic as the fp32 kernel) and offered to
//          the row's exact top-k list (64-bit keys: orderable score bits << 32
//          | ~block).  At least k candidates have s_c >= L, so every member of
//          the true top-k has an upper bound >= L and is rescored: the result
//          equals the fp32 top-k exactly.  (The filter is widened by
//          2^-16 ||qbar|| max_c ||mu_c||, which covers the fp32 rounding of the
//          rescored values themselves, at most ~2^-18 of the same product.)
//
// One CTA owns 128 query blocks of one (b, head) (thread r = row r = TMEM
// lane r for the epilogue).  All 256 threads convert each fp32 key-summary
// tile to bf16 in the 128-byte-swizzled K-major layout the MMA reads and
// compute its row norms; one thread issues the MMAs; threads 0-127 run the
// per-row bound test straight out of TMEM.
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace ssa {

constexpr int kRtcRows = 128;
constexpr int kRtcThreads = 256;
constexpr float kRtcEps = 0.0078125f;  // 2^-7

template <int D>
struct RtcLayout {
  static constexpr int NT = (D == 64) ? 256 : 128;    // key blocks per MMA (N)
  static constexpr uint32_t HALF_Q = kRtcRows * 128;  // one 64-column bf16 half of the Q tile
  static constexpr uint32_t Q_BYTES = kRtcRows * D * 2;
  static constexpr uint32_t HALF_K = NT * 128;
  static constexpr uint32_t K_BYTES = NT * D * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_QF = OFF_K + K_BYTES;          // fp32 [D][128] query summaries
  static constexpr uint32_t OFF_NRM = OFF_QF + D * kRtcRows * 4;  // fp32 [NT] key-summary norms
  static constexpr uint32_t OFF_BAR = OFF_NRM + NT * 4;
  static constexpr uint32_t USED = OFF_BAR + 32;
  static constexpr uint32_t SMEM_BYTES = USED + 1024;
  static constexpr uint32_t TMEM_COLS = NT;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// byte offset of 16-byte chunk g (of D/8) of row r in a 128B-swizzled,
// K-major bf16 tile of `rows` rows (64-column halves stacked)
__device__ __forceinline__ uint32_t sw128_offset(int r, int g, uint32_t half_bytes) {
  return static_cast<uint32_t>(g >> 3) * half_bytes + static_cast<uint32_t>(r) * 128u +
         static_cast<uint32_t>(((g & 7) ^ (r & 7)) << 4);
}

// convert 8 fp32 to 8 bf16 (RNE) packed in a uint4; also accumulate squares
__device__ __forceinline__ uint4 cvt8_bf16(const float4& a, const float4& b, float& sq) {
  sq = fmaf(a.x, a.x, sq); sq = fmaf(a.y, a.y, sq); sq = fmaf(a.z, a.z, sq); sq = fmaf(a.w, a.w, sq);
  sq = fmaf(b.x, b.x, sq); sq = fmaf(b.y, b.y, sq); sq = fmaf(b.z, b.z, sq); sq = fmaf(b.w, b.w, sq);
  return make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                    pack_bf16x2(b.z, b.w));
}

// insert v into a descending array (the smallest falls off the end)
template <int KM, typename T>
__device__ __forceinline__ void sorted_insert(T (&arr)[KM], T v) {
#pragma unroll
  for (int j = KM - 1; j > 0; --j) arr[j] = (v > arr[j - 1]) ? arr[j - 1] : (v > arr[j] ? v : arr[j]);
  arr[0] = v > arr[0] ? v : arr[0];
}

template <int D, int KM>
__global__ void __launch_bounds__(kRtcThreads, (KM <= 16 && D == 64) ? 2 : 1)
    route_tc_kernel(const RouteArgs a) {
  using Lay = RtcLayout<D>;
  constexpr int NT = Lay::NT;
  constexpr uint32_t IDESC = idesc_bf16_f32(kRtcRows, NT, false, false);
  extern __shared__ uint8_t rtc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(rtc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  float* qf = reinterpret_cast<float*>(smem + Lay::OFF_QF);     // [D][128]
  float* nrm = reinterpret_cast<float*>(smem + Lay::OFF_NRM);   // [NT]
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_BAR + 8);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int bkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int rt = a.causal ? (a.n_row_tiles - 1 - static_cast<int>(blockIdx.x))
                          : static_cast<int>(blockIdx.x);
  const int qb0 = rt * kRtcRows;
  const int qb_last = min(qb0 + kRtcRows - 1, a.NQB - 1);
  const int lim_max =
      a.top_k == 0 ? 0
      : a.causal   ? min(a.NB, static_cast<int>((static_cast<int64_t>(qb_last) * a.Bq) / a.Bk))
                   : a.NB;
  const int n_tiles = (lim_max + NT - 1) / NT;
  const float* qsrc = a.qsum + static_cast<int64_t>(bh) * a.NQB * D;
  const float* ksrc = a.ksum + static_cast<int64_t>(bkv) * a.NB * D;

  if (tid == 0) {
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  // query summaries: bf16 swizzled (MMA A operand) and fp32 transposed
  {
    constexpr int TPR = kRtcThreads / kRtcRows;   // 2 threads per row
    constexpr int CPT = (D / 8) / TPR;            // 16-byte chunks per thread
    const int r = tid / TPR, part = tid % TPR;
    const bool ok = qb0 + r < a.NQB;
    const float* src = qsrc + static_cast<int64_t>(qb0 + r) * D;
    float sq = 0.f;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int g = part * CPT + c;
      float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
      if (ok) {
        v0 = *reinterpret_cast<const float4*>(src + g * 8);
        v1 = *reinterpret_cast<const float4*>(src + g * 8 + 4);
      }
      *reinterpret_cast<uint4*>(smem + Lay::OFF_Q + sw128_offset(r, g, Lay::HALF_Q)) =
          cvt8_bf16(v0, v1, sq);
      const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[(g * 8 + e) * kRtcRows + r] = vv[e];
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // per-row state (threads 0..127)
  const int r = tid;
  const bool is_row = tid < kRtcRows;
  const int qb = qb0 + r;
  int lim = 0;
  float e_row = 0.f;
  if (is_row && qb < a.NQB) {
    lim = a.causal ? min(a.NB, static_cast<int>((static_cast<int64_t>(qb) * a.Bq) / a.Bk)) : a.NB;
    float sq = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) sq = fmaf(qf[d * kRtcRows + r], qf[d * kRtcRows + r], sq);
    // bound with a little slack for the fp32 norms themselves
    e_row = kRtcEps * sqrtf(sq) * 1.001f;
  }
  const int k = a.top_k;
  const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  uint32_t phase = 0;

  // one tile: convert key summaries, MMA, then `visit(col, score)` per column
  auto run_tile = [&](int tile, auto&& visit) {
    const int c0 = tile * NT;
    {
      constexpr int TPR = kRtcThreads / NT;          // 1 (D=64) or 2 (D=128) threads per row
      constexpr int CPT = (D / 8) / TPR;
      const int cr = tid / TPR, part = tid % TPR;
      const bool ok = c0 + cr < a.NB;
      const float* src = ksrc + static_cast<int64_t>(c0 + cr) * D;
      float sq = 0.f;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int g = part * CPT + c;
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
        if (ok) {
          v0 = *reinterpret_cast<const float4*>(src + g * 8);
          v1 = *reinterpret_cast<const float4*>(src + g * 8 + 4);
        }
        *reinterpret_cast<uint4*>(smem + Lay::OFF_K + sw128_offset(cr, g, Lay::HALF_K)) =
            cvt8_bf16(v0, v1, sq);
      }
      if (TPR == 2) sq += __shfl_xor_sync(0xffffffffu, sq, 1);
      if (part == 0) nrm[cr] = sqrtf(sq) * 1.001f;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == kRtcRows) {  // warp 4, lane 0
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t qa = sbase + Lay::OFF_Q + (kk / 4) * Lay::HALF_Q + (kk % 4) * 32;
        const uint32_t kb = sbase + Lay::OFF_K + (kk / 4) * Lay::HALF_K + (kk % 4) * 32;
        mma_ss(tmem, sdesc_sw128(qa, 16, 1024), sdesc_sw128(kb, 16, 1024), IDESC,
               kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    if (is_row) {
      // the MMA completes in bounded time; the wait is bounded anyway
      mbar_wait(bar_mma, phase, a.timeout_ns, nullptr, kSiteMma);
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < NT / 32; ++cc) {
        uint32_t sv[32];
        tmem_ld32(trow + cc * 32, sv);
        tmem_ld_wait(sv);
        const int cb = c0 + cc * 32;
        if (cb < lim) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cb + j < lim) visit(cb + j, __uint_as_float(sv[j]), nrm[cc * 32 + j]);
        }
      }
    }
    phase ^= 1u;
    tc_fence_before();
    __syncthreads();
  };

  // pass 1: the k-th largest lower bound.  The array holds KM slots; the
  // first KM - k are +inf sentinels, so slot KM-1 is the k-th real entry.
  float L = -INFINITY;
  float nmax = 0.f;
  {
    float lb[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) lb[j] = (j < KM - k) ? INFINITY : -INFINITY;
    for (int tile = 0; tile < n_tiles; ++tile) {
      run_tile(tile, [&](int, float sa, float nc) {
        nmax = fmaxf(nmax, nc);
        const float v = fmaf(-e_row, nc, sa);
        if (v > lb[KM - 1]) sorted_insert<KM>(lb, v);
      });
    }
    // widen by 2^-16 ||qbar|| max ||mu|| (e_row carries 2^-7 ||qbar||)
    L = lb[KM - 1] - e_row * nmax * 0.0078125f;
  }

  // pass 2: exact fp32 rescoring of every candidate whose upper bound reaches L
  uint64_t keys[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) keys[j] = (j < KM - k) ? ~0ull : 0ull;
  for (int tile = 0; tile < n_tiles; ++tile) {
    run_tile(tile, [&](int c, float sa, float nc) {
      if (fmaf(e_row, nc, sa) >= L) {
        const float4* mu = reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(c) * D);
        float acc = 0.f;
#pragma unroll 4
        for (int d4 = 0; d4 < D / 4; ++d4) {
          const float4 m = mu[d4];
          acc = fmaf(qf[(d4 * 4 + 0) * kRtcRows + r], m.x, acc);
          acc = fmaf(qf[(d4 * 4 + 1) * kRtcRows + r], m.y, acc);
          acc = fmaf(qf[(d4 * 4 + 2) * kRtcRows + r], m.z, acc);
          acc = fmaf(qf[(d4 * 4 + 3) * kRtcRows + r], m.w, acc);
        }
        const uint64_t key = route_key(acc, c);
        if (key > keys[KM - 1]) sorted_insert<KM>(keys, key);
      }
    });
  }

  // output: the real entries, ascending by block index
  if (is_row && qb < a.NQB) {
    int sel[KM];
    int n = 0;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      const bool real = (j >= KM - k) && keys[j] != 0ull;
      sel[j] = real ? static_cast<int>(~static_cast<uint32_t>(keys[j] & 0xFFFFFFFFull)) : 0x7FFFFFFF;
      n += real ? 1 : 0;
    }
    // insertion sort, ascending (KM <= 64, per thread)
#pragma unroll
    for (int x = 1; x < KM; ++x) {
#pragma unroll
      for (int y = x; y > 0; --y) {
        const int lo = min(sel[y - 1], sel[y]), hi = max(sel[y - 1], sel[y]);
        sel[y - 1] = lo;
        sel[y] = hi;
      }
    }
    int32_t* dst = a.idx + (static_cast<int64_t>(bh) * a.NQB + qb) * k;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < k) dst[j] = j < n ? sel[j] : -1;
    a.cnt[static_cast<int64_t>(bh) * a.NQB + qb] = n;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace ssa
