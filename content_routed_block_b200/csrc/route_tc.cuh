// K2 (tensor-core form): routing scores on tcgen05 with a proven error bound,
// then an exact fp32 top-k.
//
// jonsmirl/ssa README, "Algorithm and complexity": block c is scored by
// <q, mu_c> (the second-cumulant weight beta is 0 here) and the top_k
// admissible blocks of each query block are kept; ties go to the lower block
// index.  The ranking is decided on fp32 scores.  Scoring every (query block,
// key block) pair with fp32 FMAs costs NQB*NB*D*2 flops (240 GFLOP at a
// million tokens), so this kernel ranks in two passes over tensor-core scores:
//
//  scores  each fp32 summary x is split into bf16 parts x = x_hi + x_lo + r:
//          x_hi = bf16(x), x_lo = bf16(x - x_hi) (the difference is exact in
//          fp32).  bf16 rounds to nearest with an 8-bit significand, so with
//          u = 2^-8: |x - x_hi| <= u|x|, |x_lo| <= u(1+u)|x|, |r| <= u^2 |x|
//          (for |x| >= 2^-118; below that the parts' absolute errors are
//          under 2^-134).  sa_c = q_hi.mu_hi + q_hi.mu_lo + q_lo.mu_hi is three
//          MMAs into one fp32 TMEM accumulator (M = 128 query blocks, N = 128
//          key blocks).  Error of sa_c against s_c, the fp32 score the FMA
//          router computes (sequential fmaf over d), in units of
//          S = sum_d |q_d mu_d| <= ||qbar|| ||mu_c||:
//            dropped terms q_lo.mu_lo + q_hi.r + r.mu_hi + O(u^3):
//              <= u^2 (3 + 6u) S = 4.61e-5 S;
//            the tensor core's fp32 accumulation of the 3D exact bf16
//              products, assumed only faithful (each addition within one
//              fp32 ulp, 2^-23 relative, i.e. truncation allowed):
//              <= 3D 2^-23 (1 + 4u) S = 2.33e-5 S (D = 64), 4.65e-5 S (128);
//            the fp32 score itself (sequential fmaf, round to nearest):
//              <= D 2^-24 S = 0.38e-5 S (D = 64), 0.76e-5 S (128).
//          Total 7.3e-5 S (D = 64) and 1.00e-4 S (D = 128).  The kernel uses
//          E_c = eps ||qbar|| ||mu_c|| with eps = 2^-12 (D = 64) or 2^-11
//          (D = 128), margins of 3.3x and 4.9x over those bounds (1.001 on
//          each fp32 norm covers the norms' own rounding).
//  pass 1  L = the k-th largest of the per-32-column maxima of the lower
//          bounds sa_c - E_c.  Each maximum is the lower bound of a distinct
//          candidate, so at least k candidates have s_c >= L.
//  pass 2  every candidate whose upper bound sa_c + E_c reaches the filter is
//          queued per row in shared memory; a warp's queues are rescored
//          exactly in fp32 together (sequential FMA over d, the arithmetic of
//          the fp32 kernel) and offered to the row's exact top-k list (64-bit
//          keys: orderable score bits << 32 | ~block).  The filter starts at L
//          and rises to the current exact k-th score once k are known.  Every
//          member of the true top-k passes the filter, so the result equals
//          the fp32 top-k exactly.  (The filter is also lowered by
//          eps/2 ||qbar|| max_c ||mu_c||, which covers the fp32 rounding of
//          the bounds sa_c - E_c themselves, at most an ulp of the score.)
//
// One CTA owns 128 query blocks of one (b, head): thread r = row r = TMEM
// lane r runs the per-row tests straight out of TMEM, while the next
// key-summary tiles are staged and their MMAs issued: from the key image that
// rtc_split_kernel writes once per launch (one producer thread, bulk copies),
// or, without scratch, split by four stager warps in the kernel.
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace ssa {

constexpr int kRtcRows = 128;
constexpr int kRtcThreads = 256;          // in-kernel split: 4 row warps + 4 stager warps
constexpr int kRtcThreadsPre = 160;       // pre-split image: 4 row warps + 1 producer warp
constexpr int kRtcNT = 128;               // key blocks per MMA (N)
// error-bound factor of the split tensor-core scores (see above)
template <int D>
__host__ __device__ constexpr float rtc_eps() { return D == 64 ? 2.4414062e-4f : 4.8828125e-4f; }
constexpr int kRtcCap = 32;               // queued candidates per row before a flush

template <int D>
struct RtcLayout {
  static constexpr int NT = kRtcNT;
  static constexpr int KSTAGES = 2;                   // key-summary tiles in flight
  static constexpr uint32_t HALF_Q = kRtcRows * 128;  // one 64-column bf16 half of a Q tile
  static constexpr uint32_t Q_BYTES = kRtcRows * D * 2;
  static constexpr uint32_t HALF_K = NT * 128;
  static constexpr uint32_t K_BYTES = NT * D * 2;
  static constexpr uint32_t OFF_QH = 0;
  static constexpr uint32_t OFF_QL = OFF_QH + Q_BYTES;
  static constexpr uint32_t OFF_K = OFF_QL + Q_BYTES;              // stage s: hi, then lo
  static constexpr uint32_t OFF_NRM = OFF_K + KSTAGES * 2 * K_BYTES;  // fp32 [KSTAGES][NT]
  static constexpr uint32_t OFF_LIST = OFF_NRM + KSTAGES * NT * 4;    // uint16 [kRtcCap][128]
  static constexpr uint32_t OFF_BAR = OFF_LIST + kRtcCap * kRtcRows * 2;
  // acc_full[2] | acc_empty[2] | TMEM base (+ pad) | kload[2] | nrm_full[2]
  static constexpr uint32_t USED = OFF_BAR + 72;
  // one tile of the pre-split image: hi then lo, each laid out as a stage
  static constexpr uint32_t IMG_TILE = 2 * K_BYTES;
  static constexpr uint32_t SMEM_BYTES = USED + 1024;
  static constexpr uint32_t TMEM_COLS = KSTAGES * NT;             // two accumulators
  static __device__ __forceinline__ uint32_t kh(int st) { return OFF_K + st * 2 * K_BYTES; }
  static __device__ __forceinline__ uint32_t kl(int st) { return OFF_K + st * 2 * K_BYTES + K_BYTES; }
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// byte offset of 16-byte chunk g (of D/8) of row r in a 128B-swizzled,
// K-major bf16 tile (64-column halves stacked)
__device__ __forceinline__ uint32_t sw128_offset(int r, int g, uint32_t half_bytes) {
  return static_cast<uint32_t>(g >> 3) * half_bytes + static_cast<uint32_t>(r) * 128u +
         static_cast<uint32_t>(((g & 7) ^ (r & 7)) << 4);
}

// split 8 fp32 into bf16 hi and lo parts (both round to nearest even);
// accumulate the squares of the fp32 values
__device__ __forceinline__ void split8_bf16(const float4& a, const float4& b, uint4& hi, uint4& lo,
                                            float& sq) {
  const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 hv = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    const float r0 = v[2 * i] - __bfloat162float(hv.x);
    const float r1 = v[2 * i + 1] - __bfloat162float(hv.y);
    const __nv_bfloat162 lv = __floats2bfloat162_rn(r0, r1);
    h[i] = *reinterpret_cast<const uint32_t*>(&hv);
    l[i] = *reinterpret_cast<const uint32_t*>(&lv);
    sq = fmaf(v[2 * i], v[2 * i], sq);
    sq = fmaf(v[2 * i + 1], v[2 * i + 1], sq);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// insert v into a descending array (the smallest falls off the end)
template <int KM, typename T>
__device__ __forceinline__ void sorted_insert(T (&arr)[KM], T v) {
#pragma unroll
  for (int j = KM - 1; j > 0; --j) arr[j] = (v > arr[j - 1]) ? arr[j - 1] : (v > arr[j] ? v : arr[j]);
  arr[0] = v > arr[0] ? v : arr[0];
}

// The key summaries' MMA image, once per launch instead of once per CTA and
// tile: tile t of KV head bkv holds rows c = 128 t .. 128 t + 127 as the bf16
// hi parts then the lo parts, each in the shared-memory layout of a stage
// (128B-swizzled, K-major), and their norms sqrt(sum mu^2) * 1.001.  Rows past
// NB are zero.  D/8 lanes per row, one 16-byte chunk each.
template <int D>
__global__ void __launch_bounds__(256) rtc_split_kernel(const float* ksum, uint8_t* img, float* nrm,
                                                        int32_t NB, int32_t k_tiles,
                                                        int64_t n_rows) {
  using Lay = RtcLayout<D>;
  constexpr int G = D / 8;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = t / G;        // (bkv, tile, r) flattened
  const int g = static_cast<int>(t % G);
  if (row >= n_rows) return;        // whole warps: n_rows * G is a multiple of 32
  const int64_t per_head = static_cast<int64_t>(k_tiles) * kRtcNT;
  const int64_t bkv = row / per_head;
  const int c = static_cast<int>(row - bkv * per_head);
  const int tile = c / kRtcNT, r = c % kRtcNT;
  float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
  if (c < NB) {
    const float* src = ksum + (bkv * NB + c) * D + g * 8;
    v0 = *reinterpret_cast<const float4*>(src);
    v1 = *reinterpret_cast<const float4*>(src + 4);
  }
  uint4 hi, lo;
  float sq = 0.f;
  split8_bf16(v0, v1, hi, lo, sq);
  uint8_t* base = img + (bkv * k_tiles + tile) * static_cast<int64_t>(Lay::IMG_TILE);
  *reinterpret_cast<uint4*>(base + sw128_offset(r, g, Lay::HALF_K)) = hi;
  *reinterpret_cast<uint4*>(base + Lay::K_BYTES + sw128_offset(r, g, Lay::HALF_K)) = lo;
#pragma unroll
  for (int off = 1; off < G; off <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  if (g == 0) nrm[(bkv * k_tiles + tile) * kRtcNT + r] = sqrtf(sq) * 1.001f;
}

// Warp roles: warps 0-3 are the rows (thread r = query block qb0 + r = TMEM
// lane r) and scan every tile's scores.  PRE (160 threads): thread 128 copies
// each tile's pre-split image and norms into one of two stages and issues its
// three MMAs into one of two TMEM accumulators.  Otherwise (256 threads)
// warps 4-7 stage the tiles themselves (eight lanes per key block: load,
// split into bf16 hi / lo, norm) and thread 128 issues the MMAs.  The tiles of
// both passes form one stream, so the staging of the next tile overlaps the
// scan of the current one.  Barriers: acc_full[b] (MMAs of a tile into
// accumulator b done), acc_empty[b] (the rows have read accumulator b and the
// norms of stage b), and with PRE kload[b] / nrm_full[b] (the stage's image
// and norms have landed).
template <int D, int KM, bool PRE>
__global__ void __launch_bounds__(PRE ? kRtcThreadsPre : kRtcThreads, (D == 64 && KM <= 16) ? 2 : 1)
    route_tc_kernel(const RouteArgs a) {
  constexpr int THREADS = PRE ? kRtcThreadsPre : kRtcThreads;
  using Lay = RtcLayout<D>;
  constexpr int NT = Lay::NT;
  constexpr uint32_t IDESC = idesc_bf16_f32(kRtcRows, NT, false, false);
  extern __shared__ uint8_t rtc_smem_raw[];
  // 1024-byte aligned start, as an offset into the shared array (not through an
  // integer cast, which would drop the shared address space from every pointer
  // derived from it and turn their loads into generic ones)
  uint8_t* smem = rtc_smem_raw + ((1024u - (smem_u32(rtc_smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float* nrm = reinterpret_cast<float*>(smem + Lay::OFF_NRM);   // [2][NT]
  uint16_t* qlist = reinterpret_cast<uint16_t*>(smem + Lay::OFF_LIST);
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);       // [2]
  uint64_t* bar_empty = bar_full + 2;                                          // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_BAR + 32);
  uint64_t* bar_kload = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR + 40);  // [2]
  uint64_t* nrm_full = bar_kload + 2;                                           // [2]
  constexpr bool presplit = PRE;   // a.kimg holds the key image

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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 4);   // one arrival per row warp
      mbar_init(&bar_kload[i], 1);
      mbar_init(&nrm_full[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  // query summaries: bf16 hi / lo (MMA A operands), TPR threads per row
  if (tid < kRtcRows * (THREADS / kRtcRows)) {
    constexpr int TPR = THREADS / kRtcRows;
    constexpr int CPT = (D / 8) / TPR;
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
      uint4 hi, lo;
      split8_bf16(v0, v1, hi, lo, sq);
      *reinterpret_cast<uint4*>(smem + Lay::OFF_QH + sw128_offset(r, g, Lay::HALF_Q)) = hi;
      *reinterpret_cast<uint4*>(smem + Lay::OFF_QL + sw128_offset(r, g, Lay::HALF_Q)) = lo;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = 2 * n_tiles;     // pass 1 tiles, then pass 2 tiles

  if (warp >= 4) {
    // ------------------------------------------------ key-summary producers
    const int lane = tid & 31;
    // the descriptors of the Q parts and of stage 0's key parts; the other
    // operands are these plus a shared-memory offset (>> 4 in the low field)
    const uint64_t dq_hi = sdesc_sw128(sbase + Lay::OFF_QH, 16, 1024);
    const uint64_t dq_lo = sdesc_sw128(sbase + Lay::OFF_QL, 16, 1024);
    const uint64_t dk0 = sdesc_sw128(sbase + Lay::kh(0), 16, 1024);
    // the tile's three MMAs (q_hi k_hi, q_hi k_lo, q_lo k_hi) into accumulator st
    auto issue_mmas = [&](int st) {
      const uint64_t dk_st = dk0 + ((st * 2 * Lay::K_BYTES) >> 4);
      const uint64_t da[3] = {dq_hi, dq_hi, dq_lo};
      const uint64_t db[3] = {dk_st, dk_st + (Lay::K_BYTES >> 4), dk_st};
#pragma unroll
      for (int term = 0; term < 3; ++term) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t qoff = ((kk / 4) * Lay::HALF_Q + (kk % 4) * 32) >> 4;
          const uint64_t koff = ((kk / 4) * Lay::HALF_K + (kk % 4) * 32) >> 4;
          mma_ss(tmem + st * NT, da[term] + qoff, db[term] + koff, IDESC,
                 (term > 0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit(&bar_full[st]);
    };
    if constexpr (PRE) {
      // ------------------------------------- pre-split image: one producer
      // thread copies a tile's image and norms into stage st (untiled bulk
      // copies) once the rows have released it, and issues its MMAs.
      if (tid == kRtcRows) {
        const uint8_t* img = a.kimg + static_cast<int64_t>(bkv) * a.k_tiles * Lay::IMG_TILE;
        const float* kn = a.knrm + static_cast<int64_t>(bkv) * a.k_tiles * NT;
        for (int t = 0; t < total; ++t) {
          const int st = t & 1, tile = t % n_tiles;
          if (t >= 2) mbar_wait(&bar_empty[st], ((t - 2) >> 1) & 1, a.timeout_ns, nullptr, kSiteMma);
          mbar_arrive_expect_tx(&bar_kload[st], Lay::IMG_TILE);
          bulk_load(smem + Lay::kh(st), img + static_cast<int64_t>(tile) * Lay::IMG_TILE,
                    Lay::IMG_TILE, &bar_kload[st]);
          mbar_arrive_expect_tx(&nrm_full[st], NT * 4);
          bulk_load(nrm + st * NT, kn + static_cast<int64_t>(tile) * NT, NT * 4, &nrm_full[st]);
          mbar_wait(&bar_kload[st], (t >> 1) & 1, a.timeout_ns, nullptr, kSiteMma);
          tc_fence_after();
          issue_mmas(st);
        }
        // every copy is waited for before the final barrier: the images
        // here, the norms by the rows
      }
      __syncwarp();   // warp 4 converges before the final barrier
    } else {
      // ------------------- otherwise the four stager warps split the tiles:
      // warp w stages key rows 32(w-4) .. +31, four rows per step: lane =
      // (row of the four, 16-byte bf16 chunk g), so one load instruction
      // covers four consecutive rows (one contiguous span for D = 64)
      const int g0 = lane & 7, rsub = lane >> 3;
      const int rbase = (warp - 4) * 32 + rsub;
      constexpr int RB = D == 64 ? 8 : 4;      // rows of a batch, all loads in flight
      constexpr int HH = D / 64;               // 64-column halves of a row
      for (int t = 0; t < total; ++t) {
        const int st = t & 1;
        const int c0 = (t % n_tiles) * NT;
#pragma unroll 1
        for (int i0 = 0; i0 < 8; i0 += RB) {
          float4 va[RB][HH], vb[RB][HH];
#pragma unroll
          for (int i = 0; i < RB; ++i) {
            const int row = rbase + (i0 + i) * 4;
            const bool ok = c0 + row < a.NB;
            const float* src = ksrc + static_cast<int64_t>(c0 + row) * D;
#pragma unroll
            for (int hh = 0; hh < HH; ++hh) {
              const int g = hh * 8 + g0;
              va[i][hh] = ok ? *reinterpret_cast<const float4*>(src + g * 8) : make_float4(0.f, 0.f, 0.f, 0.f);
              vb[i][hh] = ok ? *reinterpret_cast<const float4*>(src + g * 8 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
          // the stage is rewritten only after the rows have read it (the
          // loads above are already in flight)
          if (i0 == 0 && t >= 2) mbar_wait(&bar_empty[st], ((t - 2) >> 1) & 1, a.timeout_ns, nullptr, kSiteMma);
#pragma unroll
          for (int i = 0; i < RB; ++i) {
            const int row = rbase + (i0 + i) * 4;
            float sq = 0.f;
#pragma unroll
            for (int hh = 0; hh < HH; ++hh) {
              const int g = hh * 8 + g0;
              uint4 hi, lo;
              split8_bf16(va[i][hh], vb[i][hh], hi, lo, sq);
              *reinterpret_cast<uint4*>(smem + Lay::kh(st) + sw128_offset(row, g, Lay::HALF_K)) = hi;
              *reinterpret_cast<uint4*>(smem + Lay::kl(st) + sw128_offset(row, g, Lay::HALF_K)) = lo;
            }
            // the row's sum of squares over its 8 (or 16) chunks: the
            // summation order differs from a sequential one by far less than
            // the 1.001 slack
            sq += __shfl_xor_sync(0xffffffffu, sq, 1);
            sq += __shfl_xor_sync(0xffffffffu, sq, 2);
            sq += __shfl_xor_sync(0xffffffffu, sq, 4);
            if (g0 == 0) nrm[st * NT + row] = sqrtf(sq) * 1.001f;
          }
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");   // the stagers only
        if (tid == kRtcRows) {
          tc_fence_after();
          issue_mmas(st);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ rows
    const int r = tid;
    const int qb = qb0 + r;
    const bool row_valid = qb < a.NQB;
    const float* qrow = qsrc + static_cast<int64_t>(row_valid ? qb : qb0) * D;
    int lim = 0;
    float e_row = 0.f;
    if (row_valid) {
      lim = a.causal ? min(a.NB, static_cast<int>((static_cast<int64_t>(qb) * a.Bq) / a.Bk)) : a.NB;
      float sq = 0.f;
#pragma unroll
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 v = reinterpret_cast<const float4*>(qrow)[d4];
        sq = fmaf(v.x, v.x, sq);
        sq = fmaf(v.y, v.y, sq);
        sq = fmaf(v.z, v.z, sq);
        sq = fmaf(v.w, v.w, sq);
      }
      e_row = rtc_eps<D>() * sqrtf(sq) * 1.001f;  // slack for the fp32 norms themselves
    }
    const int k = a.top_k;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);

    // scan tile t of the stream: for every 32-column group `group(cb, scores,
    // norms, full)` (full: every column of the group is admissible for this
    // row), then hand the accumulator and the stage's norms back
    auto scan_tile = [&](int t, auto&& group) {
      const int st = t & 1;
      mbar_wait(&bar_full[st], (t >> 1) & 1, a.timeout_ns, nullptr, kSiteMma);
      // the pre-split norms come by bulk copy: observe its completion here too
      const int ns = st;
      if (presplit) mbar_wait(&nrm_full[st], (t >> 1) & 1, a.timeout_ns, nullptr, kSiteMma);
      tc_fence_after();
      const int c0 = (t % n_tiles) * NT;
      if constexpr (PRE) {
        // the next group's TMEM load is in flight while this group is tested
        uint32_t sv0[32], sv1[32];
        tmem_ld32(trow + st * NT, sv0);
        tmem_ld_wait(sv0);
#pragma unroll
        for (int cc = 0; cc < NT / 32; ++cc) {
          uint32_t(&cur)[32] = (cc & 1) ? sv1 : sv0;
          uint32_t(&nxt)[32] = (cc & 1) ? sv0 : sv1;
          if (cc + 1 < NT / 32) tmem_ld32(trow + st * NT + (cc + 1) * 32, nxt);
          const int cb = c0 + cc * 32;
          group(cb, cur, nrm + ns * NT + cc * 32, cb + 32 <= lim);
          if (cc + 1 < NT / 32) tmem_ld_wait(nxt);
        }
      } else {
#pragma unroll 1
        for (int cc = 0; cc < NT / 32; ++cc) {
          uint32_t sv[32];
          tmem_ld32(trow + st * NT + cc * 32, sv);
          tmem_ld_wait(sv);
          const int cb = c0 + cc * 32;
          group(cb, sv, nrm + ns * NT + cc * 32, cb + 32 <= lim);
        }
      }
      tc_fence_before();
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&bar_empty[st]);
    };

    // pass 1: L = k-th largest per-group maximum of the lower bounds (the
    // first KM - k slots of lb are +inf sentinels, so slot KM-1 is the k-th)
    float L = -INFINITY;
    float nmax = 0.f;
    {
      float lb[KM];
#pragma unroll
      for (int j = 0; j < KM; ++j) lb[j] = (j < KM - k) ? INFINITY : -INFINITY;
      for (int t = 0; t < n_tiles; ++t) {
        scan_tile(t, [&](int cb, const uint32_t (&sv)[32], const float* nc, bool full) {
          // (the vote comes before any lane leaves: full implies cb < lim)
          const bool warp_full = __all_sync(0xffffffffu, full);
          if (cb >= lim) return;
          // branch-free: inadmissible columns count as -inf (and norm 0);
          // four partial maxima keep the dependent chain short (max is exact)
          const float4* nc4 = reinterpret_cast<const float4*>(nc);
          float gmax, gn;
          if (warp_full) {
            // the usual case: three-input maxima, no per-column test
            float gm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            float gq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j4 = 0; j4 < 8; j4 += 2) {
              const float4 na = nc4[j4], nb = nc4[j4 + 1];
              const float nn[8] = {na.x, na.y, na.z, na.w, nb.x, nb.y, nb.z, nb.w};
              float lbv[8];
#pragma unroll
              for (int u = 0; u < 8; ++u)
                lbv[u] = fmaf(-e_row, nn[u], __uint_as_float(sv[4 * j4 + u]));
              gm[0] = fmax3(gm[0], lbv[0], lbv[1]);
              gm[1] = fmax3(gm[1], lbv[2], lbv[3]);
              gm[2] = fmax3(gm[2], lbv[4], lbv[5]);
              gm[3] = fmax3(gm[3], lbv[6], lbv[7]);
              gq[0] = fmax3(gq[0], nn[0], nn[1]);
              gq[1] = fmax3(gq[1], nn[2], nn[3]);
              gq[2] = fmax3(gq[2], nn[4], nn[5]);
              gq[3] = fmax3(gq[3], nn[6], nn[7]);
            }
            gmax = fmaxf(fmaxf(gm[0], gm[1]), fmaxf(gm[2], gm[3]));
            gn = fmaxf(fmaxf(gq[0], gq[1]), fmaxf(gq[2], gq[3]));
          } else {
            const int nadm = full ? 32 : lim - cb;
            float gm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            float gq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 n4 = nc4[j4];
              const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const bool adm = 4 * j4 + u < nadm;
                const float lbv = fmaf(-e_row, nn[u], __uint_as_float(sv[4 * j4 + u]));
                gm[u] = fmaxf(gm[u], adm ? lbv : -INFINITY);
                gq[u] = fmaxf(gq[u], adm ? nn[u] : 0.f);
              }
            }
            gmax = fmaxf(fmaxf(gm[0], gm[1]), fmaxf(gm[2], gm[3]));
            gn = fmaxf(fmaxf(gq[0], gq[1]), fmaxf(gq[2], gq[3]));
          }
          nmax = fmaxf(nmax, gn);
          if (gmax > lb[KM - 1]) sorted_insert<KM>(lb, gmax);
        });
      }
      L = lb[KM - 1];
    }

    // pass 2: queue every candidate whose upper bound reaches the filter and
    // rescore the queues exactly in fp32, a warp's rows together
    uint64_t keys[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) keys[j] = (j < KM - k) ? ~0ull : 0ull;
    const float slack = e_row * nmax * 0.5f;  // >= (eps / 2) ||qbar|| max ||mu||
    float filt = L - slack;
    int nq = 0;
    // the exact fp32 scores of up to four candidates: per candidate a
    // sequential fmaf over d (the FMA router's arithmetic); the four share
    // each load of the row's query summary
    auto rescore4 = [&](const int (&c)[4], const bool (&h)[4], float (&s)[4]) {
      const float4* qv = reinterpret_cast<const float4*>(qrow);
      const float4* mu[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        mu[u] = reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(c[u]) * D);
        s[u] = 0.f;
      }
#pragma unroll 2
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 q = qv[d4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (h[u]) {
            const float4 m = mu[u][d4];
            s[u] = fmaf(q.x, m.x, s[u]);
            s[u] = fmaf(q.y, m.y, s[u]);
            s[u] = fmaf(q.z, m.z, s[u]);
            s[u] = fmaf(q.w, m.w, s[u]);
          }
        }
      }
    };
    auto flush = [&]() {
      int rounds = nq;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        rounds = max(rounds, __shfl_xor_sync(0xffffffffu, rounds, off));
      for (int t = 0; t < rounds; t += 4) {
        int c[4];
        bool h[4];
        float sc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          h[u] = t + u < nq;
          c[u] = h[u] ? qlist[(t + u) * kRtcRows + r] : 0;
        }
        rescore4(c, h, sc);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (h[u]) {
            const uint64_t key = route_key(sc[u], c[u]);
            if (key > keys[KM - 1]) sorted_insert<KM>(keys, key);
          }
        }
      }
      nq = 0;
      // once k exact candidates are known, the k-th exact score bounds the rest
      if (keys[KM - 1] != 0ull && keys[KM - 1] != ~0ull)
        filt = fmaxf(filt, key_score(keys[KM - 1]) - slack);
    };
    for (int t = n_tiles; t < total; ++t) {
      scan_tile(t, [&](int cb, const uint32_t (&sv)[32], const float* nc, bool full) {
        // branch-free: a bit per column whose upper bound reaches the filter,
        // then the inadmissible columns cut off
        // (few groups hold a candidate: the maximum upper bound is taken
        // first, with three-input maxima, and the bits only where it passes)
        uint32_t m = 0u;
        if (cb < lim) {
          const float4* nc4 = reinterpret_cast<const float4*>(nc);
          float ub[32];
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 n4 = nc4[j4];
            ub[4 * j4 + 0] = fmaf(e_row, n4.x, __uint_as_float(sv[4 * j4 + 0]));
            ub[4 * j4 + 1] = fmaf(e_row, n4.y, __uint_as_float(sv[4 * j4 + 1]));
            ub[4 * j4 + 2] = fmaf(e_row, n4.z, __uint_as_float(sv[4 * j4 + 2]));
            ub[4 * j4 + 3] = fmaf(e_row, n4.w, __uint_as_float(sv[4 * j4 + 3]));
          }
          float um[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            um[0] = fmax3(um[0], ub[j], ub[j + 1]);
            um[1] = fmax3(um[1], ub[j + 2], ub[j + 3]);
            um[2] = fmax3(um[2], ub[j + 4], ub[j + 5]);
            um[3] = fmax3(um[3], ub[j + 6], ub[j + 7]);
          }
          if (fmaxf(fmaxf(um[0], um[1]), fmaxf(um[2], um[3])) >= filt) {
#pragma unroll
            for (int j = 0; j < 32; ++j) m |= static_cast<uint32_t>(ub[j] >= filt) << j;
            if (!full) m &= (1u << (lim - cb)) - 1u;   // 0 < lim - cb < 32 here
          }
        }
        // flush (warp-uniform) only when a queue would overflow
        if (__any_sync(0xffffffffu, nq + __popc(m) > kRtcCap)) flush();
        while (m) {
          const int j = __ffs(m) - 1;
          m &= m - 1;
          qlist[nq * kRtcRows + r] = static_cast<uint16_t>(cb + j);
          ++nq;
        }
      });
    }
    flush();

    // output: the real entries, ascending by block index
    if (row_valid) {
      int sel[KM];
      int n = 0;
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        const bool real = (j >= KM - k) && keys[j] != 0ull;
        sel[j] = real ? static_cast<int>(~static_cast<uint32_t>(keys[j] & 0xFFFFFFFFull)) : 0x7FFFFFFF;
        n += real ? 1 : 0;
      }
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace ssa
