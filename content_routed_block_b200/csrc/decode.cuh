// Decode: one new query per head against the cached keys.
//
// jonsmirl/ssa README, introduction and "Algorithm and complexity", for a
// single query: the query at position i = n_ctx - 1 is its own query block;
// it scores the completed key blocks (c+1)*Bk <= i by <q, mu_c>, keeps the
// top_k (score desc, index asc), and reads exact softmax over the routed
// blocks' keys united with the window i - W < j <= i, cut at i.
//
// B200 design (flash-decoding with routing in front; two launches):
//  * decode_route_kernel: grid (candidate splits, b * KV head).  One warp per
//    query head of the group (the group's block means are read once per CTA
//    and hit L1 for the other heads); lanes take strided candidates and keep
//    a register top-KM list each, merged by shuffle bitonic merges; lane 0
//    writes the split's KM keys.  The split holding the newest admissible
//    block (i / Bk - 1) first recomputes that block's mean from the key cache
//    into the summary cache, so a caller only has to keep the cache valid for
//    the blocks before it.
//  * decode_attend_kernel: grid (key splits, b * head).  Merges the splits'
//    keys into the top_k, lays the key set out as the routed blocks' keys
//    below the window followed by the window, and runs an online softmax in
//    the exp2 domain over its share: 32 keys per warp step with lanes = keys
//    for q.k, then lanes = dims for p.v.  Writes a partial (m, l, o); the
//    last split of a head to finish (counted atomically; the route kernel
//    zeroes the counts) merges the partials and writes O (bf16) and the
//    natural-log LSE.
// The work is memory-bound: the block means of the admissible blocks
// (A * D * 4 bytes per KV head) and the gathered K/V rows (k*Bk + W rows per
// head).
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace ssa {

constexpr int kDecThreads = 256;
constexpr int kDecMaxSplits = 128;
constexpr int kDecSurvivors = 64;   // keys a fast selection sorts (two per lane)

// bitonic sort of 64 keys, element e = lane + 32 h (x0: h = 0, x1: h = 1),
// descending over e: both halves sorted, the second reversed (the 64 form a
// bitonic sequence), one exchange at distance 32, then each half merged
__device__ __forceinline__ void warp_sort64_desc(uint64_t& x0, uint64_t& x1, int lane) {
  x0 = warp_sort_desc(x0, lane);
  x1 = warp_sort_desc(x1, lane);
  const uint64_t r1 = __shfl_sync(0xffffffffu, x1, 31 - lane);
  uint64_t a = umax64(x0, r1), b = umin64(x0, r1);
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t ya = __shfl_xor_sync(0xffffffffu, a, j);
    const uint64_t yb = __shfl_xor_sync(0xffffffffu, b, j);
    const bool low = (lane & j) == 0;
    a = low ? umax64(a, ya) : umin64(a, ya);
    b = low ? umax64(b, yb) : umin64(b, yb);
  }
  x0 = a;
  x1 = b;
}

struct DecodeArgs {
  const __nv_bfloat16* q;   // [B*Hq, D]
  const __nv_bfloat16* k;   // [B*Hkv, Ncap, D]
  const __nv_bfloat16* v;   // [B*Hkv, Ncap, D]
  float* ksum;              // [B*Hkv, Ncap/Bk, D] (in / out)
  uint64_t* part_keys;      // [B*Hq, S, KM]
  float* part_attn;         // [B*Hq, KS, D + 2]: m, l, o
  uint32_t* done;           // [B*Hq] key splits finished (zeroed by the route kernel)
  __nv_bfloat16* o;         // [B*Hq, D]
  float* lse;               // [B*Hq] or null
  int32_t* idx;             // [B*Hq, top_k] or null
  int32_t* cnt;             // [B*Hq] or null
  int32_t Hq, Hkv, Ncap, Bk, top_k, window;
  int32_t i;                // query position (n_ctx - 1)
  int32_t nb;               // admissible blocks: i / Bk
  int32_t S, cands_per_split, KS;
  float scale_log2;
};

// dynamic shared memory of decode_route_kernel: the group's queries and the
// split's scores for every head of the group
template <int D>
__host__ __device__ constexpr size_t decode_route_smem(int g, int cands) {
  return static_cast<size_t>(g) * D * 4 + static_cast<size_t>(g) * cands * 4;
}

template <int D, int KM>
__global__ void __launch_bounds__(kDecThreads, (KM <= 16) ? 2 : 1) decode_route_kernel(const DecodeArgs a) {
  constexpr int LPR = D / 4;        // lanes per block-mean row (one float4 each)
  constexpr int RPI = 32 / LPR;     // rows per warp step
  constexpr int NW = kDecThreads / 32;
  extern __shared__ __align__(16) float dec_smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, bkv = blockIdx.y;
  const int g = a.Hq / a.Hkv;
  const int b = bkv / a.Hkv, kv = bkv % a.Hkv;
  const int c0 = s * a.cands_per_split, c1 = min(a.nb, c0 + a.cands_per_split);
  const int nc = max(0, c1 - c0);
  float* qs = dec_smem;                       // [g][D]
  float* sc = dec_smem + g * D;               // [g][cands_per_split]
  if (s == 0 && tid < g) a.done[static_cast<int64_t>(b) * a.Hq + kv * g + tid] = 0u;
  float* ksum = a.ksum + static_cast<int64_t>(bkv) * (a.Ncap / a.Bk) * D;
  // the newest admissible block's mean (its last key is i - 1 or earlier):
  // thread t sums rows t / D, t / D + 256 / D, ... of column t % D (the loads
  // are independent and unrolled), then D threads add the row phases
  const int c_new = a.nb - 1;
  if (c_new >= c0 && c_new < c1) {  // uniform over the CTA
    constexpr int RPH = kDecThreads / D;
    __shared__ float red[RPH][D];
    const int d = tid % D, rp = tid / D;
    const __nv_bfloat16* src = a.k + (static_cast<int64_t>(bkv) * a.Ncap + c_new * a.Bk) * D + d;
    float acc = 0.f;
#pragma unroll 8
    for (int t = rp; t < a.Bk; t += RPH) acc += __bfloat162float(src[static_cast<int64_t>(t) * D]);
    red[rp][d] = acc;
    __syncthreads();
    if (tid < D) {
      float sum = 0.f;
#pragma unroll
      for (int r = 0; r < RPH; ++r) sum += red[r][tid];
      ksum[static_cast<int64_t>(c_new) * D + tid] = sum * (1.0f / static_cast<float>(a.Bk));
    }
  }
  for (int e = tid; e < g * D; e += kDecThreads)
    qs[e] = __bfloat162float(a.q[(static_cast<int64_t>(b) * a.Hq + kv * g) * D + e]);
  __syncthreads();

  // 1. scores of every head for the split's candidates: a row is read once,
  //    coalesced (LPR lanes x float4), and dotted with all g queries
  //    (four rows' loads are issued before any is used)
  constexpr int UN = 4;
  const int sub = lane / LPR, part = lane % LPR;
  for (int r0 = warp * RPI * UN; r0 < nc; r0 += NW * RPI * UN) {
    float4 m[UN];
#pragma unroll
    for (int u = 0; u < UN; ++u) {
      const int r = r0 + u * RPI + sub;
      m[u] = r < nc ? reinterpret_cast<const float4*>(ksum + static_cast<int64_t>(c0 + r) * D)[part]
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < UN; ++u) {
      const int r = r0 + u * RPI + sub;
      for (int j = 0; j < g; ++j) {
        const float4 qv = reinterpret_cast<const float4*>(qs + j * D)[part];
        float acc = qv.x * m[u].x;
        acc = fmaf(qv.y, m[u].y, acc);
        acc = fmaf(qv.z, m[u].z, acc);
        acc = fmaf(qv.w, m[u].w, acc);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (r < nc && part == 0) sc[j * a.cands_per_split + r] = acc;
      }
    }
  }
  __syncthreads();

  // 2. per head, the top KM of the split: a lower bound L from the lanes'
  //    maxima (the KM-th largest of them is reached by >= KM candidates).
  //    The candidates at or above L hold the top KM; when at most 64 do, the
  //    warp compacts them and sorts them (the usual case), otherwise they go
  //    through per-lane register lists and shuffle merges
  __shared__ uint64_t surv[NW][kDecSurvivors];
  for (int j = warp; j < g; j += NW) {
    const int bh = b * a.Hq + kv * g + j;
    const float* sj = sc + j * a.cands_per_split;
    float lmax = -INFINITY;
    for (int r = lane; r < nc; r += 32) lmax = fmaxf(lmax, sj[r]);
    float L = -INFINITY;
    if (KM <= 32) {
      // descending bitonic sort of the 32 lane maxima
      float x = lmax;
#pragma unroll
      for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
          const float y = __shfl_xor_sync(0xffffffffu, x, jj);
          const bool desc_block = (lane & k) == 0;
          const bool low = (lane & jj) == 0;
          x = (low == desc_block) ? fmaxf(x, y) : fminf(x, y);
        }
      }
      L = __shfl_sync(0xffffffffu, x, KM - 1);
    }
    uint64_t* dst = a.part_keys + (static_cast<int64_t>(bh) * a.S + s) * KM;
    if (KM <= 32 && a.top_k > 0) {
      int nsv = 0;
      for (int r0 = 0; r0 < nc; r0 += 32) {
        const int r = r0 + lane;
        const float v = r < nc ? sj[r] : 0.f;
        const bool take = r < nc && v >= L;
        const uint32_t bal = __ballot_sync(0xffffffffu, take);
        const int pos = nsv + __popc(bal & ((1u << lane) - 1u));
        if (take && pos < kDecSurvivors) surv[warp][pos] = route_key(v, c0 + r);
        nsv += __popc(bal);
      }
      __syncwarp();
      if (nsv <= kDecSurvivors) {
        uint64_t x0 = lane < nsv ? surv[warp][lane] : 0ull;
        if (nsv <= 32) {
          x0 = warp_sort_desc(x0, lane);
        } else {
          uint64_t x1 = lane + 32 < nsv ? surv[warp][lane + 32] : 0ull;
          warp_sort64_desc(x0, x1, lane);
        }
        __syncwarp();
        if (lane < KM) dst[lane] = x0;   // zeros past the split's candidates
        continue;
      }
      __syncwarp();
    }
    uint64_t keys[KM];
#pragma unroll
    for (int e = 0; e < KM; ++e) keys[e] = 0ull;
    if (a.top_k > 0) {
      for (int r = lane; r < nc; r += 32) {
        const float v = sj[r];
        if (v >= L) {
          const uint64_t key = route_key(v, c0 + r);
          if (key > keys[KM - 1]) route_sorted_insert<KM>(keys, key);
        }
      }
    }
#pragma unroll
    for (int mask = 1; mask < 32; mask <<= 1) route_merge_partner<KM>(keys, mask);
    if (lane == 0) {
#pragma unroll
      for (int e = 0; e < KM; ++e) dst[e] = keys[e];
    }
  }
}

template <int D, int KM>
__global__ void __launch_bounds__(kDecThreads) decode_attend_kernel(const DecodeArgs a) {
  constexpr int NW = kDecThreads / 32;
  constexpr int DL = D / 32;  // dims per lane in the p.v step
  extern __shared__ __align__(16) uint4 dec_vstage[];  // [NW][32 keys][D/8]: a warp's V rows
  __shared__ __align__(16) float qs[D];
  __shared__ int sel[64];
  __shared__ int seg_off[65];
  __shared__ int n_sel_s;
  __shared__ float wm[NW], wl[NW];
  __shared__ __align__(16) float wo[NW][D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int x = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int bkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int i = a.i;
  const int lo = max(0, i - a.window + 1);

  for (int d = tid; d < D; d += kDecThreads) qs[d] = __bfloat162float(a.q[static_cast<int64_t>(bh) * D + d]);
  // 1. the top_k of the splits' keys, listed ascending.  Each split's list is
  //    sorted descending, so L = the largest of the splits' top_k-th keys is
  //    reached by top_k keys of one split: the selection lies among the keys
  //    >= L, and only in the first top_k entries of each list.  When at most
  //    64 keys pass (the usual case) the whole CTA collects them and warp 0
  //    sorts them; otherwise warp 0 merges the lists.
  __shared__ uint64_t surv[kDecSurvivors];
  __shared__ uint64_t wmax[NW];
  __shared__ int n_surv;
  bool fast = false;
  if constexpr (KM <= 32) {
    if (a.top_k > 0) {
      const uint64_t* lists = a.part_keys + static_cast<int64_t>(bh) * a.S * KM;
      uint64_t kth = 0ull;
      for (int sp = tid; sp < a.S; sp += kDecThreads) kth = umax64(kth, lists[sp * KM + a.top_k - 1]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) kth = umax64(kth, __shfl_xor_sync(0xffffffffu, kth, off));
      if (lane == 0) wmax[warp] = kth;
      if (tid == 0) n_surv = 0;
      __syncthreads();
      uint64_t L = wmax[0];
#pragma unroll
      for (int w = 1; w < NW; ++w) L = umax64(L, wmax[w]);
      const int total = a.S * a.top_k;
      for (int e = tid; e < total; e += kDecThreads) {
        const int sp = e / a.top_k, jj = e - sp * a.top_k;
        const uint64_t key = lists[sp * KM + jj];
        if (key != 0ull && key >= L) {
          const int pos = atomicAdd(&n_surv, 1);
          if (pos < kDecSurvivors) surv[pos] = key;
        }
      }
      __syncthreads();
      fast = n_surv <= kDecSurvivors;
    } else {
      fast = true;   // nothing is routed
    }
  }
  if (warp == 0) {
    uint64_t keys[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) keys[j] = 0ull;
    uint64_t mine = 0ull;
    int n = 0;
    if (fast) {
      const int ns = a.top_k > 0 ? n_surv : 0;
      uint64_t x0 = lane < ns ? surv[lane] : 0ull;
      if (ns <= 32) {
        x0 = warp_sort_desc(x0, lane);
      } else {
        uint64_t x1 = lane + 32 < ns ? surv[lane + 32] : 0ull;
        warp_sort64_desc(x0, x1, lane);
      }
      mine = (lane < a.top_k) ? x0 : 0ull;
      n = __popc(__ballot_sync(0xffffffffu, mine != 0ull));
    } else {
      // lane l folds splits l, l + 32, ... (each sorted descending) into its
      // list with in-register bitonic merges; the shuffle merges then keep
      // the top KM of all of them
      for (int sp = lane; sp < a.S; sp += 32) {
        const uint64_t* src = a.part_keys + (static_cast<int64_t>(bh) * a.S + sp) * KM;
        uint64_t other[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j) other[j] = src[j];
        route_merge_lists<KM>(keys, other);
      }
#pragma unroll
      for (int mask = 1; mask < 32; mask <<= 1) route_merge_partner<KM>(keys, mask);
      // every lane now holds the top KM; lane j takes entry j (j < top_k)
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        const bool real = j < a.top_k && keys[j] != 0ull;
        n += real ? 1 : 0;
        if (j == lane) mine = real ? keys[j] : 0ull;
      }
    }
    if constexpr (KM <= 32) {
      // the warp sorts the selected block indices ascending and scans the
      // far-segment lengths (the part of each routed block below the window)
      int c = mine != 0ull ? static_cast<int>(~static_cast<uint32_t>(mine & 0xFFFFFFFFull)) : 0x7FFFFFFF;
#pragma unroll
      for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
          const int y = __shfl_xor_sync(0xffffffffu, c, jj);
          const bool asc = (lane & k) == 0;
          const bool low = (lane & jj) == 0;
          c = (low == asc) ? min(c, y) : max(c, y);
        }
      }
      // KM <= 32 here: lanes 0..n-1 hold the selection ascending
      const int start = c * a.Bk;
      int len = lane < n ? max(0, min(start + a.Bk, lo) - start) : 0;
      int incl = len;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (lane < n) {
        sel[lane] = c;
        seg_off[lane] = incl - len;
      }
      if (lane == n - 1 || (n == 0 && lane == 0)) {
        seg_off[n] = n ? incl : 0;
        n_sel_s = n;
      }
      if (x == 0) {
        if (a.cnt != nullptr && lane == 0) a.cnt[bh] = n;
        if (a.idx != nullptr && lane < a.top_k) a.idx[static_cast<int64_t>(bh) * a.top_k + lane] = lane < n ? c : -1;
      }
    } else if (lane == 0) {
      // top_k > 32: one lane lists the selection
      int v[KM];
      int n = 0;
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        const bool real = j < a.top_k && keys[j] != 0ull;
        v[j] = real ? static_cast<int>(~static_cast<uint32_t>(keys[j] & 0xFFFFFFFFull)) : 0x7FFFFFFF;
        n += real ? 1 : 0;
      }
#pragma unroll
      for (int p = 1; p < KM; ++p) {
#pragma unroll
        for (int y = p; y > 0; --y) {
          const int l0 = min(v[y - 1], v[y]), h0 = max(v[y - 1], v[y]);
          v[y - 1] = l0;
          v[y] = h0;
        }
      }
      int off = 0;
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        if (j < n) {
          sel[j] = v[j];
          seg_off[j] = off;
          const int start = v[j] * a.Bk;
          off += max(0, min(start + a.Bk, lo) - start);
        }
      }
      seg_off[n] = off;
      n_sel_s = n;
      if (x == 0) {
        if (a.cnt != nullptr) a.cnt[bh] = n;
        if (a.idx != nullptr) {
#pragma unroll
          for (int j = 0; j < KM; ++j)
            if (j < a.top_k) a.idx[static_cast<int64_t>(bh) * a.top_k + j] = j < n ? v[j] : -1;
        }
      }
    }
  }
  __syncthreads();
  const int n_sel = n_sel_s;
  const int far_total = seg_off[n_sel];
  const int L = far_total + (i - lo + 1);
  const int p0 = static_cast<int>((static_cast<int64_t>(L) * x) / a.KS);
  const int p1 = static_cast<int>((static_cast<int64_t>(L) * (x + 1)) / a.KS);

  // 2. online softmax over key positions p0..p1-1 (lanes = keys for q.k)
  const __nv_bfloat16* kb = a.k + static_cast<int64_t>(bkv) * a.Ncap * D;
  const __nv_bfloat16* vb = a.v + static_cast<int64_t>(bkv) * a.Ncap * D;
  float m = -INFINITY, l = 0.f;
  float o[DL];
#pragma unroll
  for (int d = 0; d < DL; ++d) o[d] = 0.f;
  for (int base = p0 + warp * 32; base < p1; base += NW * 32) {
    const int pos = base + lane;
    const bool valid = pos < p1;
    int j = 0;
    if (valid) {
      if (pos < far_total) {
        int seg = 0;
        while (seg + 1 < n_sel && seg_off[seg + 1] <= pos) ++seg;
        j = sel[seg] * a.Bk + (pos - seg_off[seg]);
      } else {
        j = lo + (pos - far_total);
      }
    }
    float sc = -INFINITY;
    uint4* vst = dec_vstage + (warp * 32 + lane) * (D / 8);
    if (valid) {
      // this lane's V row goes to the warp's stage now, so that all 32 rows
      // are in flight at once
      const uint4* vr = reinterpret_cast<const uint4*>(vb + static_cast<int64_t>(j) * D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) vst[c] = vr[c];
      const uint4* kr = reinterpret_cast<const uint4*>(kb + static_cast<int64_t>(j) * D);
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 u = kr[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          acc = fmaf(qs[8 * c + 2 * t], __uint_as_float(w[t] << 16), acc);
          acc = fmaf(qs[8 * c + 2 * t + 1], __uint_as_float(w[t] & 0xFFFF0000u), acc);
        }
      }
      sc = acc * a.scale_log2;
    }
    float bm = sc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
    const float m_new = fmaxf(m, bm);
    const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
    const float pk = valid ? exp2f(sc - m_new) : 0.f;
    float ps = pk;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * alpha + ps;
#pragma unroll
    for (int d = 0; d < DL; ++d) o[d] *= alpha;
    m = m_new;
    // p.v with lanes = dims from the staged rows: key t, dims lane + 32 d
    __syncwarp();
    const int nk = min(32, p1 - base);
    const __nv_bfloat16* vs = reinterpret_cast<const __nv_bfloat16*>(dec_vstage + warp * 32 * (D / 8));
    for (int t = 0; t < nk; ++t) {
      const float pt = __shfl_sync(0xffffffffu, pk, t);
#pragma unroll
      for (int d = 0; d < DL; ++d) o[d] = fmaf(pt, __bfloat162float(vs[t * D + lane + 32 * d]), o[d]);
    }
    __syncwarp();  // the stage is rewritten by the next step
  }
  // 3. combine the warps, write the split's partial
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int d = 0; d < DL; ++d) wo[warp][lane + 32 * d] = o[d];
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w]);
    float Lsum = 0.f;
    float oo[DL];
#pragma unroll
    for (int d = 0; d < DL; ++d) oo[d] = 0.f;
    for (int w = 0; w < NW; ++w) {
      const float f = (wm[w] == -INFINITY) ? 0.f : exp2f(wm[w] - M);
      Lsum += wl[w] * f;
#pragma unroll
      for (int d = 0; d < DL; ++d) oo[d] += wo[w][lane + 32 * d] * f;
    }
    float* dst = a.part_attn + (static_cast<int64_t>(bh) * a.KS + x) * (D + 2);
    if (lane == 0) {
      dst[0] = M;
      dst[1] = Lsum;
    }
#pragma unroll
    for (int d = 0; d < DL; ++d) dst[2 + lane + 32 * d] = oo[d];
    // 4. the last key split of this head to finish merges all splits'
    // partials and writes O and the LSE: each split's partial is visible
    // device-wide before its count, and the last one sees every count
    __threadfence();
    __syncwarp();
    uint32_t prev = 0;
    if (lane == 0) prev = atomicAdd(&a.done[bh], 1u);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev == static_cast<uint32_t>(a.KS - 1)) {
      __threadfence();
      const volatile float* src = a.part_attn + static_cast<int64_t>(bh) * a.KS * (D + 2);
      float Mx = -INFINITY;
      for (int y = 0; y < a.KS; ++y) Mx = fmaxf(Mx, src[y * (D + 2)]);
      float L = 0.f;
      float acc[DL];
#pragma unroll
      for (int d = 0; d < DL; ++d) acc[d] = 0.f;
      for (int y = 0; y < a.KS; ++y) {
        const float my = src[y * (D + 2)];
        const float f = (my == -INFINITY) ? 0.f : exp2f(my - Mx);
        L += src[y * (D + 2) + 1] * f;
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[d] += src[y * (D + 2) + 2 + lane + 32 * d] * f;
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
      for (int d = 0; d < DL; ++d)
        a.o[static_cast<int64_t>(bh) * D + lane + 32 * d] = __float2bfloat16_rn(acc[d] * inv);
      if (lane == 0 && a.lse != nullptr)
        a.lse[bh] = L > 0.f ? (Mx + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
    }
  }
}

template <int D>
__host__ __device__ constexpr size_t decode_attend_smem() {
  return static_cast<size_t>(kDecThreads / 32) * 32 * D * 2;
}

}  // namespace ssa
