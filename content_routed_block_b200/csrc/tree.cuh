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
//  * tree_select_kernel: one warp per query block.  Candidates go 32 at a
//    time, 16 per half-warp: each candidate's summary row is read coalesced
//    (16 lanes x float4), 16 independent loads per lane, and a shuffle
//    reduce-scatter leaves lane l with candidate e0 + l's fp32 score, which
//    it keeps in its register top-KM list (route.cuh's 64-bit keys).  The
//    k-th largest lane maximum bounds the row's k-th key from below; the few
//    list entries above it are sorted by the warp (butterfly merges of the
//    lane lists when more than 64 survive, or k > 32).  The CTA's eight warps take eight consecutive query
//    blocks of one head, whose kept super-blocks mostly coincide, so the
//    children's summaries are re-read from L1.
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
  __shared__ uint64_t surv[kTreeWarps][64];
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
  // candidate e -> key block (-1: a child of a rejected super-block)
  auto block_of = [&](int e) -> int {
    if (e >= n_kids) return (ns << a.log2_f) + (e - n_kids);
    const int s = sup_s[warp][e >> a.log2_f];
    return s < 0 ? -1 : (s << a.log2_f) + (e & (F - 1));
  };
  // Candidates go 32 at a time, 16 per half-warp: lane hl of half h reads
  // columns 4hl .. 4hl+3 (+64 i) of the rows of candidates e0 + 16h + j,
  // j = 0..15 (each row read coalesced by the half-warp, all 16 loads
  // independent), and forms 16 partial dot products with its slice of qbar.
  // A reduce-scatter over the half-warp (8 + 4 + 2 + 1 shuffles) then leaves
  // lane hl holding the full product of candidate j = hl, i.e. lane l holds
  // candidate e0 + l.
  constexpr int QV = D / 64;
  const int half = lane >> 4, hl = lane & 15;
  float4 qv[QV];
#pragma unroll
  for (int i = 0; i < QV; ++i) qv[i] = reinterpret_cast<const float4*>(qs[warp])[hl + 16 * i];
  uint64_t keys[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) keys[j] = 0ull;
  float thr_f = -INFINITY;
  // With F >= 16 a half's 16 candidates (e0 + 16h is a multiple of 16, and
  // so are n_kids and every super-block's first child) are 16 consecutive
  // blocks of one kept super-block, or of the frontier: one base row serves
  // all of them.  Smaller fanouts map every candidate separately.
  const bool contiguous = F >= 16;
  for (int e0 = 0; e0 < n_cand; e0 += 32) {  // warp-uniform
    float p[16];
    if (contiguous) {
      const int eh = e0 + 16 * half;
      const int nh = min(16, n_cand - eh);   // candidates of this half (may be <= 0)
      const int c0 = nh > 0 ? block_of(eh) : -1;
      const float4* k4 =
          reinterpret_cast<const float4*>(kbase + static_cast<int64_t>(max(c0, 0)) * D) + hl;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float part = 0.f;
        if (c0 >= 0 && j < nh) {
#pragma unroll
          for (int i = 0; i < QV; ++i) {
            const float4 x = __ldg(k4 + j * (D / 4) + 16 * i);
            part = fmaf(x.x, qv[i].x, part);
            part = fmaf(x.y, qv[i].y, part);
            part = fmaf(x.z, qv[i].z, part);
            part = fmaf(x.w, qv[i].w, part);
          }
        }
        p[j] = part;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int e = e0 + 16 * half + j;
        const int c = e < n_cand ? block_of(e) : -1;
        float part = 0.f;
        if (c >= 0) {
          const float4* k4 =
              reinterpret_cast<const float4*>(kbase + static_cast<int64_t>(c) * D) + hl;
#pragma unroll
          for (int i = 0; i < QV; ++i) {
            const float4 x = __ldg(k4 + 16 * i);
            part = fmaf(x.x, qv[i].x, part);
            part = fmaf(x.y, qv[i].y, part);
            part = fmaf(x.z, qv[i].z, part);
            part = fmaf(x.w, qv[i].w, part);
          }
        }
        p[j] = part;
      }
    }
    // reduce-scatter: at offset m a lane keeps the half of its candidates
    // whose bit m matches its own lane bit and adds its partner's partials
#pragma unroll
    for (int m = 8; m > 0; m >>= 1) {
      const bool up = (hl & m) != 0;
#pragma unroll
      for (int i = 0; i < m; ++i) {
        const float send = up ? p[i] : p[i + m];
        const float keep = up ? p[i + m] : p[i];
        p[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
      }
    }
    const float mine = p[0];
    const int e = e0 + lane;
    const int c = e < n_cand ? block_of(e) : -1;
    if (c >= 0 && mine >= thr_f) {
      const uint64_t key = route_key(mine, c);
      if (key > keys[KM - 1]) {
        route_sorted_insert<KM>(keys, key);
        if (keys[KM - 1] != 0ull) thr_f = key_score(keys[KM - 1]);
      }
    }
  }
  const int k = a.top_k;
  int n = 0;
  if (KM <= 32) {
    // The row's top k from the 32 lane lists.  The k-th largest lane maximum
    // T is a lower bound on the row's k-th key (k lanes hold a key >= T), so
    // only list entries >= T can be selected.  When at most 64 survive they
    // are sorted directly (two warp sorts and a bitonic merge keep the top
    // 32); otherwise five butterfly merges of the lane lists.  Either way
    // lane j ends with the row's j-th best key (0 = none).
    uint64_t best = 0ull;
    bool done = false;
    if (k > 0) {
      const uint64_t lane_max = warp_sort_desc(keys[0], lane);
      const uint64_t T = __shfl_sync(0xffffffffu, lane_max, k - 1);
      if (T != 0ull) {
        int mine = 0;
#pragma unroll
        for (int j = 0; j < KM; ++j) mine += keys[j] >= T ? 1 : 0;
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (total <= 64) {  // warp-uniform
          uint64_t* buf = surv[warp];
          const int pos = incl - mine;  // the lane's survivors are its first `mine` entries
#pragma unroll
          for (int j = 0; j < KM; ++j)
            if (j < mine) buf[pos + j] = keys[j];
          __syncwarp();
          uint64_t v0 = lane < total ? buf[lane] : 0ull;
          uint64_t v1 = lane + 32 < total ? buf[lane + 32] : 0ull;
          __syncwarp();
          v0 = warp_sort_desc(v0, lane);
          v1 = warp_sort_desc(v1, lane);
          uint64_t r = umax64(v0, __shfl_sync(0xffffffffu, v1, 31 - lane));
#pragma unroll
          for (int j = 16; j > 0; j >>= 1) {
            const uint64_t y = __shfl_xor_sync(0xffffffffu, r, j);
            r = (lane & j) ? umin64(r, y) : umax64(r, y);
          }
          best = r;
          done = true;
        }
      }
    }
    if (!done) {
#pragma unroll
      for (int mask = 1; mask < 32; mask <<= 1) route_merge_partner<KM>(keys, mask);
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j == lane) best = keys[j];
    }
    n = __popc(__ballot_sync(0xffffffffu, lane < k && best != 0ull));
    if (k > 0) {
      // the selected blocks ascending: sort (2^32 - 1 - block) descending
      uint64_t key = lane < n ? 0xFFFFFFFFull - (~static_cast<uint32_t>(best & 0xFFFFFFFFull)) : 0ull;
      key = warp_sort_desc(key, lane);
      if (lane < k) a.idx[row * k + lane] = lane < n ? static_cast<int>(0xFFFFFFFFull - key) : -1;
    }
  } else {
#pragma unroll
    for (int mask = 1; mask < 32; mask <<= 1) route_merge_partner<KM>(keys, mask);
    // every lane holds the row's top KM keys, best first; rank by counting
#pragma unroll
    for (int j = 0; j < KM; ++j) n += (j < k && keys[j] != 0ull) ? 1 : 0;
    if (k > 0) {
      int32_t* dst = a.idx + row * k;
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        if (j >= n) continue;
        const int cj = static_cast<int>(~static_cast<uint32_t>(keys[j] & 0xFFFFFFFFull));
        int rank = 0;
#pragma unroll
        for (int i = 0; i < KM; ++i)
          if (i < n && static_cast<int>(~static_cast<uint32_t>(keys[i] & 0xFFFFFFFFull)) < cj)
            ++rank;
        if ((j & 31) == lane) dst[rank] = cj;
      }
      for (int j = n + lane; j < k; j += 32) dst[j] = -1;
    }
  }
  if (lane == 0) a.cnt[row] = n;
}

}  // namespace ssa
