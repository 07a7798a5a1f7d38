// K2d: two-level (fixed-beam tree) routing.
//
// jonsmirl/ssa README, "Algorithm and complexity": a hierarchical router with
// fixed block size and budget approaches linear routing work on benign
// geometry, where a flat router scores every admissible block (the measured
// tree uses fanout 16); "Mathematical status": fixed-beam routing is not an
// exact selector.  Super-block S covers key blocks S*F .. S*F+F-1 and is
// summarised by the mean of its keys.  A query block keeps its best `beam`
// complete admissible super-blocks and then its top_k blocks among their
// children and the frontier (the admissible blocks past the last complete
// admissible super-block).  Both levels order by (score descending, block
// index ascending).
//
// Three launches per route:
//  * tree_pool_kernel: super-block means from the block means (each block
//    has Bk keys, so the mean of the F child means is the mean of the F*Bk
//    keys).  One thread per (super-block, 4 columns), F float4 loads.
//  * the upper level is the flat router (route.cuh) run on the super-block
//    summaries with block F*Bk and top_k = beam: its admissibility rule
//    (S+1)*F*Bk <= qb*Bq is exactly "S is complete and admissible".
//  * tree_select_kernel: one warp per query block.  Lane l scores candidates
//    l, l+32, ... (fp32 dot products, the block summary read as float4) and
//    keeps its top KM in registers as route.cuh's 64-bit keys; five shuffle
//    merges leave the row's top KM in every lane.  The CTA's eight warps
//    take eight consecutive query blocks of one head, whose kept
//    super-blocks mostly coincide, so the children's summaries are re-read
//    from L1.
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace ssa {

constexpr int kTreeThreads = 256;
constexpr int kTreeWarps = kTreeThreads / 32;
constexpr int kTreeMaxBeam = 64;

struct TreePoolArgs {
  const float* ksum;  // [B*Hkv, NB, D] block means
  float* ksum2;       // [B*Hkv, NS, D] super-block means (out)
  int64_t n_nodes;    // B * Hkv * NS
  int32_t NB, NS, F;
  float inv_f;        // 1 / F (exact: F is a power of two)
};

template <int D>
__global__ void __launch_bounds__(256) tree_pool_kernel(const TreePoolArgs a) {
  constexpr int C4 = D / 4;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t node = t / C4;
  if (node >= a.n_nodes) return;
  const int c4 = static_cast<int>(t % C4);
  const int64_t bkv = node / a.NS;
  const int s = static_cast<int>(node % a.NS);
  const float4* src =
      reinterpret_cast<const float4*>(a.ksum + (bkv * a.NB + static_cast<int64_t>(s) * a.F) * D) +
      c4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < a.F; ++j) {
    const float4 v = __ldg(src + static_cast<int64_t>(j) * C4);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  acc.x *= a.inv_f;
  acc.y *= a.inv_f;
  acc.z *= a.inv_f;
  acc.w *= a.inv_f;
  reinterpret_cast<float4*>(a.ksum2 + node * D)[c4] = acc;
}

struct TreeSelectArgs {
  const float* qsum;       // [B*Hq, NQB, D]
  const float* ksum;       // [B*Hkv, NB, D]
  const int32_t* sup_idx;  // [B*Hq, NQB, beam] kept super-blocks, ascending, -1 padded
  const int32_t* sup_cnt;  // [B*Hq, NQB]
  int32_t* idx;            // [B*Hq, NQB, top_k] (out)
  int32_t* cnt;            // [B*Hq, NQB] (out)
  int32_t Hq, Hkv, NQB, NB, Bq, Bk, top_k, causal;
  int32_t log2_f, beam;
  int64_t n_rows;          // B * Hq * NQB
};

template <int D, int KM>
__global__ void __launch_bounds__(kTreeThreads) tree_select_kernel(const TreeSelectArgs a) {
  __shared__ __align__(16) float qs[kTreeWarps][D];
  __shared__ int32_t sup_s[kTreeWarps][kTreeMaxBeam];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kTreeWarps + warp;
  if (row >= a.n_rows) return;  // warp-uniform
  const int qb = static_cast<int>(row % a.NQB);
  const int64_t bh = row / a.NQB;
  const int b = static_cast<int>(bh / a.Hq), h = static_cast<int>(bh % a.Hq);
  const int64_t bkv = static_cast<int64_t>(b) * a.Hkv + h / (a.Hq / a.Hkv);
  const int F = 1 << a.log2_f;
  // admissible blocks 0 .. n_adm-1; complete admissible super-blocks 0 .. ns-1
  const int n_adm =
      a.causal ? min(a.NB, static_cast<int>((static_cast<int64_t>(qb) * a.Bq) / a.Bk)) : a.NB;
  const int ns = n_adm >> a.log2_f;

  for (int d = lane; d < D; d += 32) qs[warp][d] = a.qsum[row * D + d];
  int n2 = a.sup_cnt[row];
  if (n2 < 0 || n2 > min(a.beam, ns)) {
    record_error(kErrCheck, kSiteTree);
    n2 = min(max(n2, 0), min(a.beam, ns));
  }
  // a kept super-block must be complete, admissible and above its
  // predecessor; a bad entry is reported and contributes no candidates
  for (int j = lane; j < n2; j += 32) {
    int s = a.sup_idx[row * a.beam + j];
    const int prev = j > 0 ? a.sup_idx[row * a.beam + j - 1] : -1;
    if (s < 0 || s >= ns || s <= prev) {
      record_error(kErrCheck, kSiteTree);
      s = -1;
    }
    sup_s[warp][j] = s;
  }
  __syncwarp();

  const int n_kids = n2 << a.log2_f;
  const int n_cand = a.top_k == 0 ? 0 : n_kids + (n_adm - (ns << a.log2_f));
  const float* kbase = a.ksum + bkv * a.NB * D;
  const float4* q4 = reinterpret_cast<const float4*>(qs[warp]);
  uint64_t keys[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) keys[j] = 0ull;
  float thr_f = -INFINITY;
  for (int e = lane; e < n_cand; e += 32) {
    int c;
    if (e < n_kids) {
      const int s = sup_s[warp][e >> a.log2_f];
      if (s < 0) continue;
      c = (s << a.log2_f) + (e & (F - 1));
    } else {
      c = (ns << a.log2_f) + (e - n_kids);
    }
    const float4* k4 = reinterpret_cast<const float4*>(kbase + static_cast<int64_t>(c) * D);
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int i = 0; i < D / 4; i += 2) {
      const float4 x0 = __ldg(k4 + i), y0 = q4[i];
      const float4 x1 = __ldg(k4 + i + 1), y1 = q4[i + 1];
      acc0 = fmaf(x0.x, y0.x, acc0);
      acc0 = fmaf(x0.y, y0.y, acc0);
      acc0 = fmaf(x0.z, y0.z, acc0);
      acc0 = fmaf(x0.w, y0.w, acc0);
      acc1 = fmaf(x1.x, y1.x, acc1);
      acc1 = fmaf(x1.y, y1.y, acc1);
      acc1 = fmaf(x1.z, y1.z, acc1);
      acc1 = fmaf(x1.w, y1.w, acc1);
    }
    const float v = acc0 + acc1;
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

  // every lane now holds the row's top KM keys, best first; lane j writes
  // the j-th smallest selected block index (rank by counting)
  const int k = a.top_k;
  int n = 0;
#pragma unroll
  for (int j = 0; j < KM; ++j) n += (j < k && keys[j] != 0ull) ? 1 : 0;
  if (k > 0) {
    int32_t* dst = a.idx + row * k;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (j >= n) continue;
      const int cj = static_cast<int>(~static_cast<uint32_t>(keys[j] & 0xFFFFFFFFull));
      // rank of block cj among the n selected blocks
      int rank = 0;
#pragma unroll
      for (int i = 0; i < KM; ++i)
        if (i < n && static_cast<int>(~static_cast<uint32_t>(keys[i] & 0xFFFFFFFFull)) < cj) ++rank;
      if ((j & 31) == lane) dst[rank] = cj;
    }
    for (int j = n + lane; j < k; j += 32) dst[j] = -1;
  }
  if (lane == 0) a.cnt[row] = n;
}

}  // namespace ssa
