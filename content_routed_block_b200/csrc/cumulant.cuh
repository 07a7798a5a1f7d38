// Routing with SSA's second-cumulant score.
//
// jonsmirl/ssa README, "Algorithm and complexity": block c is scored by
// r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q, mu_c the block's mean key and
// Sigma_c its second cumulant.  A query block scores by the mean of its
// queries' scores, s_c = <qbar, mu_c> + (beta/2) tr(Sigma_c Q2), Q2 the mean of
// q_i q_i^T over the block (the quadratic term is linear in q q^T, as the
// first is in q).  With the feature vectors
//   keys     psi_c = [mu_c | vech(Sigma_c)]
//   queries  phi   = [qbar | (beta/2) w . vech(Q2)],  w = 1 on the diagonal,
//                                                     2 off it
// (vech = upper triangle d <= e, row by row) the score is one dot product of
// length F = D + D(D+1)/2: 2144 for D = 64.  Three kernels:
//  * cumulant_features_kernel: one CTA per block builds psi or phi in fp32
//    (the keys are centred on their mean before the outer products, which
//    keeps the covariance accurate when the mean is large);
//  * cumulant_scores_kernel: fp32 SIMT GEMM S = Phi Psi^T per (b, head),
//    64 x 64 tiles, only tiles that hold admissible pairs;
//  * cumulant_select_kernel: one warp per query block; every lane keeps the
//    top KM keys of its strided candidates in registers (the 64-bit keys of
//    route.cuh: score desc, index asc), and five shuffle bitonic merges leave
//    the row's top KM in every lane.
// The fp32 scores are a different rounding of the fp64 definition than the
// plain router's, so indices agree with the oracle except at its counted
// near-ties, like the rest of the routing.
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace ssa {

template <int D>
__host__ __device__ constexpr int cumulant_features() { return D + D * (D + 1) / 2; }

constexpr int kCumThreads = 256;
constexpr int kCumTile = 64;   // rows and candidates per score tile
constexpr int kCumK = 32;      // features per K step of the score GEMM

struct CumFeatArgs {
  const __nv_bfloat16* x;  // [rows, D] (B * H * N rows)
  float* out;              // [B * H * N / block, F]
  int64_t n_blocks;
  int32_t block;
  int32_t queries;         // 0: keys (mean, covariance); 1: queries (mean, weighted moment)
  float half_beta;         // beta / 2 (queries only)
};

// One CTA per block; dynamic shared memory holds the block as fp32 [block][D]
// and its mean.  The D x D outer-product sum is computed on 4 x 4 register
// tiles of the upper triangle (tile rows ti <= tile columns tj): per row t of
// the block a thread reads two float4 and does 16 FMAs.
template <int D>
__host__ __device__ constexpr size_t cumulant_features_smem(int block) {
  return static_cast<size_t>(block) * D * 4 + D * 4;
}

template <int D>
__global__ void __launch_bounds__(kCumThreads) cumulant_features_kernel(const CumFeatArgs a) {
  constexpr int F = cumulant_features<D>();
  constexpr int T = D / 4;                  // tiles per side
  constexpr int NT = T * (T + 1) / 2;       // upper-triangular tiles
  extern __shared__ __align__(16) float cum_x[];
  float* mean = cum_x + a.block * D;        // [D]
  const int64_t blk = blockIdx.x;
  if (blk >= a.n_blocks) return;
  const int tid = threadIdx.x;
  const __nv_bfloat16* src = a.x + blk * a.block * D;
  for (int i = tid; i < a.block * D; i += kCumThreads) cum_x[i] = __bfloat162float(src[i]);
  __syncthreads();
  const float inv = 1.0f / static_cast<float>(a.block);  // exact: block is a power of two
  if (tid < D) {
    float s = 0.f;
    for (int t = 0; t < a.block; ++t) s += cum_x[t * D + tid];
    mean[tid] = s * inv;
  }
  __syncthreads();
  float* dst = a.out + blk * F;
  if (tid < D) dst[tid] = mean[tid];
  if (!a.queries) {
    // centre the keys: Sigma = (1/block) sum (x - mu)(x - mu)^T
    for (int i = tid; i < a.block * D; i += kCumThreads) cum_x[i] -= mean[i % D];
    __syncthreads();
  }
  for (int u = tid; u < NT; u += kCumThreads) {
    // tile u -> (ti, tj), ti <= tj: row ti of the tile triangle starts at
    // ti*T - ti(ti-1)/2
    int ti = 0, off = 0;
    while (off + (T - ti) <= u) {
      off += T - ti;
      ++ti;
    }
    const int tj = ti + (u - off);
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int t = 0; t < a.block; ++t) {
      const float4 xa = *reinterpret_cast<const float4*>(cum_x + t * D + 4 * ti);
      const float4 xb = *reinterpret_cast<const float4*>(cum_x + t * D + 4 * tj);
      const float va[4] = {xa.x, xa.y, xa.z, xa.w};
      const float vb[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(va[i], vb[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int d = 4 * ti + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = 4 * tj + j;
        if (d > e) continue;  // lower half of a diagonal tile
        float v = acc[i][j] * inv;
        if (a.queries) v *= a.half_beta * (d == e ? 1.f : 2.f);
        dst[D + d * D - d * (d - 1) / 2 + (e - d)] = v;
      }
    }
  }
}

struct CumScoreArgs {
  const float* qf;   // [B*Hq, NQB, F]
  const float* kf;   // [B*Hkv, NB, F]
  float* scores;     // [B*Hq, NQB, NB]
  int32_t Hq, Hkv, NQB, NB, Bq, Bk, causal;
  int32_t n_row_tiles, n_cand_tiles;
};

// this thread's share of one K step: rows / candidates i / 8 of the tile,
// features f0 + 4 (i % 8) .. + 3, for i = tid and tid + 256
template <int F>
__device__ __forceinline__ void cum_load_step(float4 (&pa)[2], float4 (&pb)[2], const float* qsrc,
                                              const float* ksrc, int qb0, int c0, int NQB, int NB,
                                              int f0, int tid) {
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int i = tid + kCumThreads * j;
    const int r = i / (kCumK / 4), f4 = i % (kCumK / 4);
    pa[j] = (qb0 + r < NQB)
                ? *reinterpret_cast<const float4*>(qsrc + static_cast<int64_t>(qb0 + r) * F + f0 + f4 * 4)
                : make_float4(0.f, 0.f, 0.f, 0.f);
    pb[j] = (c0 + r < NB)
                ? *reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(c0 + r) * F + f0 + f4 * 4)
                : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// S = Phi Psi^T on 64 x 64 tiles; 256 threads, 4 x 4 outputs each; the next
// K step's operands go global -> registers while the current one is used
template <int D>
__global__ void __launch_bounds__(kCumThreads) cumulant_scores_kernel(const CumScoreArgs a) {
  constexpr int F = cumulant_features<D>();
  static_assert(F % kCumK == 0, "feature length must be a multiple of the K step");
  constexpr int LD = kCumTile + 4;
  __shared__ __align__(16) float As[kCumK][LD];  // query features, [f][row]
  __shared__ __align__(16) float Bs[kCumK][LD];  // key features,   [f][cand]
  const int bh = blockIdx.y;
  const int rt = blockIdx.x / a.n_cand_tiles, ct = blockIdx.x % a.n_cand_tiles;
  const int qb0 = rt * kCumTile, c0 = ct * kCumTile;
  const int qb_last = min(qb0 + kCumTile - 1, a.NQB - 1);
  const int lim_max =
      a.causal ? min(a.NB, static_cast<int>((static_cast<int64_t>(qb_last) * a.Bq) / a.Bk)) : a.NB;
  if (c0 >= lim_max) return;  // no admissible pair in this tile
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int bkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const float* qsrc = a.qf + static_cast<int64_t>(bh) * a.NQB * F;
  const float* ksrc = a.kf + static_cast<int64_t>(bkv) * a.NB * F;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;

  // loads: 64 rows x 32 features = 512 float4 per operand, 2 per thread
  float4 pa[2], pb[2];
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  cum_load_step<F>(pa, pb, qsrc, ksrc, qb0, c0, a.NQB, a.NB, 0, tid);
  for (int f0 = 0; f0 < F; f0 += kCumK) {
    __syncthreads();  // the previous step's reads of As / Bs are done
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int i = tid + kCumThreads * j;
      const int r = i / (kCumK / 4), f4 = i % (kCumK / 4);
      As[f4 * 4 + 0][r] = pa[j].x; As[f4 * 4 + 1][r] = pa[j].y;
      As[f4 * 4 + 2][r] = pa[j].z; As[f4 * 4 + 3][r] = pa[j].w;
      Bs[f4 * 4 + 0][r] = pb[j].x; Bs[f4 * 4 + 1][r] = pb[j].y;
      Bs[f4 * 4 + 2][r] = pb[j].z; Bs[f4 * 4 + 3][r] = pb[j].w;
    }
    __syncthreads();
    if (f0 + kCumK < F) cum_load_step<F>(pa, pb, qsrc, ksrc, qb0, c0, a.NQB, a.NB, f0 + kCumK, tid);
#pragma unroll
    for (int f = 0; f < kCumK; ++f) {
      const float4 qa = *reinterpret_cast<const float4*>(&As[f][ty * 4]);
      const float4 kb = *reinterpret_cast<const float4*>(&Bs[f][tx * 4]);
      const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
      const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qb = qb0 + ty * 4 + i;
    if (qb >= a.NQB) continue;
    float* dst = a.scores + (static_cast<int64_t>(bh) * a.NQB + qb) * a.NB + c0 + tx * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (c0 + tx * 4 + j < a.NB) dst[j] = acc[i][j];
  }
}

struct CumSelectArgs {
  const float* scores;  // [B*Hq, NQB, NB]
  int32_t* idx;         // [B*Hq, NQB, top_k]
  int32_t* cnt;         // [B*Hq, NQB]
  int32_t NQB, NB, Bq, Bk, top_k, causal;
  int64_t n_rows;       // B * Hq * NQB
};

template <int KM>
__global__ void __launch_bounds__(kCumThreads) cumulant_select_kernel(const CumSelectArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (kCumThreads / 32) + (threadIdx.x >> 5);
  if (row >= a.n_rows) return;  // warp-uniform
  const int qb = static_cast<int>(row % a.NQB);
  const int lim =
      a.top_k == 0 ? 0
      : a.causal   ? min(a.NB, static_cast<int>((static_cast<int64_t>(qb) * a.Bq) / a.Bk))
                   : a.NB;
  const float* s = a.scores + row * a.NB;
  uint64_t keys[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) keys[j] = 0ull;
  float thr_f = -INFINITY;
  for (int c = lane; c < lim; c += 32) {
    const float v = s[c];
    if (v >= thr_f) {
      const uint64_t key = route_key(v, c);
      if (key > keys[KM - 1]) {
        route_sorted_insert<KM>(keys, key);
        if (keys[KM - 1] != 0ull) thr_f = key_score(keys[KM - 1]);
      }
    }
  }
#pragma unroll
  for (int mask = 1; mask < 32; mask <<= 1) route_merge_partner<KM>(keys, mask);
  if (lane == 0) {
    const int k = a.top_k;
    int sel[KM];
    int n = 0;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      const bool real = j < k && keys[j] != 0ull;
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
    if (k > 0) {
      int32_t* dst = a.idx + row * k;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j < k) dst[j] = j < n ? sel[j] : -1;
    }
    a.cnt[row] = n;
  }
}

}  // namespace ssa
