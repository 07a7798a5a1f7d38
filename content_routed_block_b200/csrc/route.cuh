// K2: routing -- block scores and top-k per query block.
//
// jonsmirl/ssa README, "Algorithm and complexity": block c is scored by
// r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q; here beta = 0 (mean pooling
// only) and q is the query block's mean.  Each query block keeps the top_k
// admissible blocks; ties go to the lower block index (an explicit
// deterministic order; the same page notes that without a margin a
// deterministic index order is needed to name one top set).  The selected
// blocks are written in ascending order, padded with -1, with their count.
//
// Two selection schemes share the scoring below: route_rows_kernel (top_k <=
// 32, at the end of this file) keeps a per-thread register list; the
// warp-list route_kernel serves 32 < top_k <= 64.
//
// Design (sm_100a):
//  * One CTA owns 64 consecutive query blocks of one (b, head) and streams
//    the key summaries of its KV head in tiles of 64 blocks through shared
//    memory, so each summary tile is read once per 64 query blocks.  Scores
//    are fp32 FMA dot products (a 4x4 register tile per thread): fp32 keeps
//    the ranking exact up to ~1e-6 relative, which tensor-core bf16/tf32
//    products would not.
//  * Causal row tiles have triangular work; the grid visits the heaviest
//    (last) tiles first.
//  * Each warp owns 8 query-block rows and keeps each row's running top list
//    in registers as 64-bit keys (orderable score bits << 32 | ~block), so
//    "score descending, index ascending" is one unsigned compare and every
//    key is distinct.  A new batch of 32 candidates is filtered by a ballot
//    against the current k-th key; a few survivors are inserted by a warp
//    shift, many are sorted with a register bitonic network (shuffles) and
//    merged into the list with a bitonic merge.
#pragma once

#include "common.cuh"

namespace ssa {

constexpr int kRouteCands = 64;    // key blocks per summary tile
constexpr int kRouteThreads = 256;

struct RouteArgs {
  const float* qsum;   // [B*Hq, NQB, D]
  const float* ksum;   // [B*Hkv, NB, D]
  int32_t* idx;        // [B*Hq, NQB, top_k]
  int32_t* cnt;        // [B*Hq, NQB]
  int32_t Hq, Hkv, NQB, NB, Bq, Bk, top_k, causal;
  int32_t n_row_tiles;
  uint64_t timeout_ns;
  // tensor-core form only: the key summaries already split into their bf16
  // MMA image (rtc_split_kernel), or null to split them in the kernel
  const uint8_t* kimg = nullptr;   // [B*Hkv, k_tiles, 2 * 128 * D * 2]
  const float* knrm = nullptr;     // [B*Hkv, k_tiles * 128]
  int32_t k_tiles = 0;
};

// orderable 64-bit key: larger key <=> (higher score, then lower index)
__device__ __forceinline__ uint64_t route_key(float s, int c) {
  s = (s == 0.0f) ? 0.0f : s;  // -0 and +0 are the same score
  const uint32_t u = __float_as_uint(s);
  const uint32_t hi = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(hi) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(c));
}

// the score a key was made from (inverse of route_key's orderable mapping)
__device__ __forceinline__ float key_score(uint64_t key) {
  const uint32_t hi = static_cast<uint32_t>(key >> 32);
  return __uint_as_float((hi & 0x80000000u) ? (hi & 0x7FFFFFFFu) : ~hi);
}

__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t umin64(uint64_t a, uint64_t b) { return a < b ? a : b; }

// bitonic sort of one key per lane, descending over lanes
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t x, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint64_t y = __shfl_xor_sync(0xffffffffu, x, j);
      const bool desc_block = (lane & k) == 0;
      const bool low = (lane & j) == 0;
      x = (low == desc_block) ? umax64(x, y) : umin64(x, y);
    }
  }
  return x;
}

// list element e = lane + 32*r, sorted descending over e
template <int R>
__device__ __forceinline__ uint64_t list_get(const uint64_t (&v)[R], int e) {
  uint64_t src = v[0];
#pragma unroll
  for (int r = 1; r < R; ++r)
    if ((e >> 5) == r) src = v[r];
  return __shfl_sync(0xffffffffu, src, e & 31);
}

// insert one key (same value in every lane) that beats the current k-th key
template <int R>
__device__ __forceinline__ void list_insert(uint64_t (&v)[R], uint64_t y, int lane) {
  int pos = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) pos += __popc(__ballot_sync(0xffffffffu, v[r] > y));
  uint64_t carry = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    uint64_t up = __shfl_up_sync(0xffffffffu, v[r], 1);
    const uint64_t last = __shfl_sync(0xffffffffu, v[r], 31);
    if (lane == 0) up = carry;
    const int e = lane + 32 * r;
    v[r] = (e < pos) ? v[r] : (e == pos ? y : up);
    carry = last;
  }
}

// merge 32 keys sorted descending (one per lane) into the list, keeping the
// top 32*R: max against the reversed batch makes a bitonic sequence, which a
// bitonic merge sorts
template <int R>
__device__ __forceinline__ void list_merge(uint64_t (&v)[R], uint64_t sorted, int lane) {
  const uint64_t rev = __shfl_sync(0xffffffffu, sorted, 31 - lane);
  v[R - 1] = umax64(v[R - 1], rev);
  if (R == 2) {
    const uint64_t a = v[0], b = v[R - 1];
    v[0] = umax64(a, b);
    v[R - 1] = umin64(a, b);
  }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const bool low = (lane & j) == 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint64_t y = __shfl_xor_sync(0xffffffffu, v[r], j);
      v[r] = low ? umax64(v[r], y) : umin64(v[r], y);
    }
  }
}

// offer one candidate key per lane (0 = no candidate)
template <int R>
__device__ __forceinline__ void list_offer(uint64_t (&v)[R], uint64_t& thr, uint64_t x, int k,
                                           int lane) {
  const bool pass = x > thr;
  uint32_t m = __ballot_sync(0xffffffffu, pass);
  if (m == 0) return;
  if (__popc(m) <= 4) {
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      const uint64_t y = __shfl_sync(0xffffffffu, x, src);
      if (y > thr) {
        list_insert<R>(v, y, lane);
        thr = list_get<R>(v, k - 1);
      }
    }
  } else {
    const uint64_t s = warp_sort_desc(pass ? x : 0ull, lane);
    list_merge<R>(v, s, lane);
    thr = list_get<R>(v, k - 1);
  }
}

// ascending bitonic sort of 32*R ints spread as e = lane + 32*r
template <int R>
__device__ __forceinline__ void warp_sort_asc_i32(int (&a)[R], int lane) {
#pragma unroll
  for (int k = 2; k <= 32 * R; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
        // only when R == 2 and k == 64: the whole sequence is one ascending block
        const int x0 = a[0], x1 = a[R - 1];
        a[0] = min(x0, x1);
        a[R - 1] = max(x0, x1);
      } else {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int e = lane + 32 * r;
          const int y = __shfl_xor_sync(0xffffffffu, a[r], j);
          const bool asc = (e & k) == 0;
          const bool low = (lane & j) == 0;
          a[r] = (low == asc) ? min(a[r], y) : max(a[r], y);
        }
      }
    }
  }
}

// shared-memory bytes of route_kernel<D, R, RT>
template <int D, int R, int RT>
__host__ __device__ constexpr size_t route_smem_bytes() {
  return static_cast<size_t>(D * RT + D * kRouteCands + RT * (kRouteCands + 1)) * 4 +
         static_cast<size_t>(RT) * (32 * R + 1) * 8 + static_cast<size_t>(RT) * 4;
}

// admissible key blocks of query block qb: 0 .. limit-1
__device__ __forceinline__ int route_row_limit(const RouteArgs& a, int qb) {
  return a.causal ? min(a.NB, static_cast<int>((static_cast<int64_t>(qb) * a.Bq) / a.Bk)) : a.NB;
}

// this thread's share of the key-summary tile starting at block c0: float4
// j of the thread is element i = tid + 256 j, i.e. block c0 + i % 64,
// columns 4 (i / 64) .. 4 (i / 64) + 3
template <int D, int NPRE>
__device__ __forceinline__ void route_load_tile(float4 (&pre)[NPRE], const float* ksrc, int c0,
                                                int NB, int tid) {
#pragma unroll
  for (int j = 0; j < NPRE; ++j) {
    const int i = tid + kRouteThreads * j;
    const int c = i % kRouteCands, d4 = i / kRouteCands;
    pre[j] = (c0 + c < NB)
                 ? *reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(c0 + c) * D + d4 * 4)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// RT query blocks per CTA (64, or 16 when 64 would leave SMs idle)
template <int D, int R, int RT>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteArgs a) {
  constexpr int kRouteRows = RT;
  constexpr int SC_LD = kRouteCands + 1;
  constexpr int ROWS_PER_WARP = kRouteRows / (kRouteThreads / 32);
  constexpr int RPT = kRouteRows / 16;      // score rows per thread
  constexpr int NPRE = (kRouteCands * D / 4) / kRouteThreads;  // float4 per thread per tile
  extern __shared__ __align__(16) float rsm[];
  float* qsT = rsm;                         // [D][RT]   query summaries, transposed
  float* ksT = qsT + D * kRouteRows;        // [D][64]   key summaries, transposed
  float* sc = ksT + D * kRouteCands;        // [RT][65]  score tile
  // per-row top lists (element e = lane + 32 r of row `row` at
  // lst[(row * R + r) * 32 + lane], descending), the k-th key, and its score
  uint64_t* lst = reinterpret_cast<uint64_t*>(sc + kRouteRows * SC_LD);
  uint64_t* thr_s = lst + kRouteRows * R * 32;
  float* thrf_s = reinterpret_cast<float*>(thr_s + kRouteRows);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int bkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int rt = a.causal ? (a.n_row_tiles - 1 - static_cast<int>(blockIdx.x))
                          : static_cast<int>(blockIdx.x);
  const int qb0 = rt * kRouteRows;
  const int qb_last = min(qb0 + kRouteRows - 1, a.NQB - 1);
  const int lim_max = a.top_k == 0 ? 0 : route_row_limit(a, qb_last);
  const int n_tiles = (lim_max + kRouteCands - 1) / kRouteCands;

  const float* qsrc = a.qsum + static_cast<int64_t>(bh) * a.NQB * D;
  const float* ksrc = a.ksum + static_cast<int64_t>(bkv) * a.NB * D;

  // key-summary tiles go global -> registers one tile ahead, then registers
  // -> shared memory (transposed) at the top of the next iteration, so the
  // L2 latency of tile t+1 hides behind the scoring and selection of tile t
  float4 pre[NPRE];
  if (n_tiles > 0) route_load_tile<D, NPRE>(pre, ksrc, 0, a.NB, tid);

  // query summaries of this row tile, transposed (consecutive threads take
  // consecutive rows so the shared-memory stores do not conflict)
  for (int i = tid; i < kRouteRows * (D / 4); i += kRouteThreads) {
    const int r = i % kRouteRows, d4 = i / kRouteRows;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qb0 + r < a.NQB)
      v = *reinterpret_cast<const float4*>(qsrc + static_cast<int64_t>(qb0 + r) * D + d4 * 4);
    qsT[(d4 * 4 + 0) * kRouteRows + r] = v.x;
    qsT[(d4 * 4 + 1) * kRouteRows + r] = v.y;
    qsT[(d4 * 4 + 2) * kRouteRows + r] = v.z;
    qsT[(d4 * 4 + 3) * kRouteRows + r] = v.w;
  }
  for (int i = tid; i < kRouteRows * R * 32; i += kRouteThreads) lst[i] = 0ull;
  for (int i = tid; i < kRouteRows; i += kRouteThreads) {
    thr_s[i] = 0ull;
    thrf_s[i] = -INFINITY;
  }

  const int ty = tid / 16, tx = tid % 16;
  for (int tile = 0; tile < n_tiles; ++tile) {
    const int c0 = tile * kRouteCands;
#pragma unroll
    for (int j = 0; j < NPRE; ++j) {
      const int i = tid + kRouteThreads * j;
      const int c = i % kRouteCands, d4 = i / kRouteCands;
      ksT[(d4 * 4 + 0) * kRouteCands + c] = pre[j].x;
      ksT[(d4 * 4 + 1) * kRouteCands + c] = pre[j].y;
      ksT[(d4 * 4 + 2) * kRouteCands + c] = pre[j].z;
      ksT[(d4 * 4 + 3) * kRouteCands + c] = pre[j].w;
    }
    // the tile is staged, and every warp has finished the previous tile's
    // selection (it read the score tile that is about to be overwritten)
    __syncthreads();
    if (tile + 1 < n_tiles) route_load_tile<D, NPRE>(pre, ksrc, c0 + kRouteCands, a.NB, tid);

    float acc[RPT][4];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float4 kb = *reinterpret_cast<const float4*>(ksT + d * kRouteCands + tx * 4);
      const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
      float qv[RPT];
      if constexpr (RPT == 4) {
        const float4 qa = *reinterpret_cast<const float4*>(qsT + d * kRouteRows + ty * 4);
        qv[0] = qa.x; qv[1] = qa.y; qv[2] = qa.z; qv[3] = qa.w;
      } else {
#pragma unroll
        for (int i = 0; i < RPT; ++i) qv[i] = qsT[d * kRouteRows + ty * RPT + i];
      }
#pragma unroll
      for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) sc[(ty * RPT + i) * SC_LD + tx * 4 + j] = acc[i][j];
    __syncthreads();

    // selection: a row's 64 candidates are first compared, as floats, with
    // the score of its current k-th key; only when one reaches it is the
    // row's list brought into registers and the candidates offered as
    // 64-bit keys (an equal score is settled there by the block index)
#pragma unroll 1
    for (int rr = 0; rr < ROWS_PER_WARP; ++rr) {
      const int row = warp * ROWS_PER_WARP + rr;
      const int qb = qb0 + row;
      if (qb >= a.NQB) continue;
      const int lim = route_row_limit(a, qb);
      if (c0 >= lim) continue;
      const float tf = thrf_s[row];
      const int ca = c0 + lane, cb = c0 + 32 + lane;
      const float sa = sc[row * SC_LD + lane], sb = sc[row * SC_LD + 32 + lane];
      const bool pa = ca < lim && sa >= tf;
      const bool pb = cb < lim && sb >= tf;
      if (!__any_sync(0xffffffffu, pa || pb)) continue;
      uint64_t v[R];
#pragma unroll
      for (int r = 0; r < R; ++r) v[r] = lst[(row * R + r) * 32 + lane];
      uint64_t thr = thr_s[row];
      list_offer<R>(v, thr, pa ? route_key(sa, ca) : 0ull, a.top_k, lane);
      list_offer<R>(v, thr, pb ? route_key(sb, cb) : 0ull, a.top_k, lane);
#pragma unroll
      for (int r = 0; r < R; ++r) lst[(row * R + r) * 32 + lane] = v[r];
      __syncwarp();
      if (lane == 0) {
        thr_s[row] = thr;
        thrf_s[row] = thr != 0ull ? key_score(thr) : -INFINITY;
      }
      __syncwarp();
    }
  }

  // epilogue: the first top_k keys, as block indices in ascending order
#pragma unroll 1
  for (int rr = 0; rr < ROWS_PER_WARP; ++rr) {
    const int row = warp * ROWS_PER_WARP + rr;
    const int qb = qb0 + row;
    if (qb >= a.NQB) continue;
    int vals[R];
    int n_valid = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = lane + 32 * r;
      const uint64_t key = lst[(row * R + r) * 32 + lane];
      const bool ok = e < a.top_k && key != 0ull;
      vals[r] = ok ? static_cast<int>(~static_cast<uint32_t>(key & 0xFFFFFFFFull)) : 0x7FFFFFFF;
      n_valid += __popc(__ballot_sync(0xffffffffu, ok));
    }
    warp_sort_asc_i32<R>(vals, lane);
    int32_t* dst = a.idx + (static_cast<int64_t>(bh) * a.NQB + qb) * a.top_k;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = lane + 32 * r;
      if (e < a.top_k) dst[e] = e < n_valid ? vals[r] : -1;
    }
    if (lane == 0) a.cnt[static_cast<int64_t>(bh) * a.NQB + qb] = n_valid;
  }
}

// ---------------------------------------------------------------------------
// Thread-per-row form (top_k <= 32).  The same tiles and the same fp32 scores
// (sequential FMA over d) as route_kernel, but the selection is per thread:
// row r of the tile is split among TPR = 256 / RT consecutive threads, each
// of which keeps the top KM (>= top_k) keys of its candidates in registers,
// sorted descending.  A candidate first meets a float filter (its score
// against the score of the thread's KM-th key); only a survivor becomes a
// 64-bit key and is inserted.  At the end the TPR lists of a row are merged
// pairwise with shuffles (bitonic merge of two sorted lists keeps the top
// KM of their union), so every thread of the row holds the row's top KM.
// ---------------------------------------------------------------------------
template <int D, int KM, int RT>
__host__ __device__ constexpr size_t route_rows_smem_bytes() {
  return static_cast<size_t>(D * RT + D * kRouteCands + RT * (kRouteCands + kRouteThreads / RT)) * 4;
}

// insert v into a descending array (the smallest falls off the end)
template <int KM>
__device__ __forceinline__ void route_sorted_insert(uint64_t (&arr)[KM], uint64_t v) {
#pragma unroll
  for (int j = KM - 1; j > 0; --j) arr[j] = (v > arr[j - 1]) ? arr[j - 1] : (v > arr[j] ? v : arr[j]);
  arr[0] = v > arr[0] ? v : arr[0];
}

// keep in `a` the top KM of a U b, where a and b are sorted descending and b
// is the list of lane ^ mask: max(a[i], b[KM-1-i]) is a bitonic sequence
// holding the top KM, which a bitonic clean-up sorts descending
template <int KM>
__device__ __forceinline__ void route_merge_partner(uint64_t (&a)[KM], int mask) {
  uint64_t b[KM];
#pragma unroll
  for (int i = 0; i < KM; ++i) b[i] = __shfl_xor_sync(0xffffffffu, a[i], mask);
#pragma unroll
  for (int i = 0; i < KM; ++i) a[i] = umax64(a[i], b[KM - 1 - i]);
#pragma unroll
  for (int j = KM / 2; j > 0; j >>= 1) {
#pragma unroll
    for (int i = 0; i < KM; ++i) {
      if ((i & j) == 0) {
        const uint64_t x = a[i], y = a[i + j];
        a[i] = umax64(x, y);
        a[i + j] = umin64(x, y);
      }
    }
  }
}

// keep in `a` the top KM of a U b, both sorted descending (b in registers)
template <int KM>
__device__ __forceinline__ void route_merge_lists(uint64_t (&a)[KM], const uint64_t (&b)[KM]) {
#pragma unroll
  for (int i = 0; i < KM; ++i) a[i] = umax64(a[i], b[KM - 1 - i]);
#pragma unroll
  for (int j = KM / 2; j > 0; j >>= 1) {
#pragma unroll
    for (int i = 0; i < KM; ++i) {
      if ((i & j) == 0) {
        const uint64_t x = a[i], y = a[i + j];
        a[i] = umax64(x, y);
        a[i + j] = umin64(x, y);
      }
    }
  }
}

template <int D, int KM, int RT>
__global__ void __launch_bounds__(kRouteThreads) route_rows_kernel(const RouteArgs a) {
  constexpr int TPR = kRouteThreads / RT;           // threads per row
  constexpr int CPT = kRouteCands / TPR;            // candidates per thread per tile
  constexpr int SC_LD = kRouteCands + TPR;          // each thread's span padded by one
  constexpr int RPT = RT / 16;                      // score rows per thread (FMA tile)
  constexpr int NPRE = (kRouteCands * D / 4) / kRouteThreads;
  static_assert(TPR >= 2 && TPR <= 16 && CPT <= 32, "tile shape");
  extern __shared__ __align__(16) float rsm[];
  float* qsT = rsm;                   // [D][RT]
  float* ksT = qsT + D * RT;          // [D][64]
  float* sc = ksT + D * kRouteCands;  // [RT][SC_LD]: candidate c of the tile at
                                      // (c / CPT) * (CPT + 1) + c % CPT

  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int bkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int rt = a.causal ? (a.n_row_tiles - 1 - static_cast<int>(blockIdx.x))
                          : static_cast<int>(blockIdx.x);
  const int qb0 = rt * RT;
  const int qb_last = min(qb0 + RT - 1, a.NQB - 1);
  const int lim_max = a.top_k == 0 ? 0 : route_row_limit(a, qb_last);
  const int n_tiles = (lim_max + kRouteCands - 1) / kRouteCands;
  const float* qsrc = a.qsum + static_cast<int64_t>(bh) * a.NQB * D;
  const float* ksrc = a.ksum + static_cast<int64_t>(bkv) * a.NB * D;

  float4 pre[NPRE];
  if (n_tiles > 0) route_load_tile<D, NPRE>(pre, ksrc, 0, a.NB, tid);
  for (int i = tid; i < RT * (D / 4); i += kRouteThreads) {
    const int r = i % RT, d4 = i / RT;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qb0 + r < a.NQB)
      v = *reinterpret_cast<const float4*>(qsrc + static_cast<int64_t>(qb0 + r) * D + d4 * 4);
    qsT[(d4 * 4 + 0) * RT + r] = v.x;
    qsT[(d4 * 4 + 1) * RT + r] = v.y;
    qsT[(d4 * 4 + 2) * RT + r] = v.z;
    qsT[(d4 * 4 + 3) * RT + r] = v.w;
  }

  // selection state of this thread: row `row`, candidates part * CPT ..
  const int row = tid / TPR, part = tid % TPR;
  const int qb = qb0 + row;
  const int lim = (qb < a.NQB && a.top_k > 0) ? route_row_limit(a, qb) : 0;
  uint64_t keys[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) keys[j] = 0ull;
  float thr_f = -INFINITY;  // score of keys[KM-1] once the list is full

  const int ty = tid / 16, tx = tid % 16;
  for (int tile = 0; tile < n_tiles; ++tile) {
    const int c0 = tile * kRouteCands;
#pragma unroll
    for (int j = 0; j < NPRE; ++j) {
      const int i = tid + kRouteThreads * j;
      const int c = i % kRouteCands, d4 = i / kRouteCands;
      ksT[(d4 * 4 + 0) * kRouteCands + c] = pre[j].x;
      ksT[(d4 * 4 + 1) * kRouteCands + c] = pre[j].y;
      ksT[(d4 * 4 + 2) * kRouteCands + c] = pre[j].z;
      ksT[(d4 * 4 + 3) * kRouteCands + c] = pre[j].w;
    }
    __syncthreads();
    if (tile + 1 < n_tiles) route_load_tile<D, NPRE>(pre, ksrc, c0 + kRouteCands, a.NB, tid);

    float acc[RPT][4];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
      const float4 kb = *reinterpret_cast<const float4*>(ksT + d * kRouteCands + tx * 4);
      const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
      float qv[RPT];
      if constexpr (RPT % 4 == 0) {
#pragma unroll
        for (int i4 = 0; i4 < RPT / 4; ++i4) {
          const float4 qa = *reinterpret_cast<const float4*>(qsT + d * RT + ty * RPT + i4 * 4);
          qv[i4 * 4 + 0] = qa.x; qv[i4 * 4 + 1] = qa.y; qv[i4 * 4 + 2] = qa.z; qv[i4 * 4 + 3] = qa.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < RPT; ++i) qv[i] = qsT[d * RT + ty * RPT + i];
      }
#pragma unroll
      for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
    }
    {
      const int cl = tx * 4;  // 4 candidates in one thread span (CPT >= 4)
      const int pos = (cl / CPT) * (CPT + 1) + cl % CPT;
#pragma unroll
      for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[(ty * RPT + i) * SC_LD + pos + j] = acc[i][j];
    }
    __syncthreads();

    // selection over this thread's CPT candidates
    const int cb = c0 + part * CPT;
    if (cb < lim) {
      const float* srow = sc + row * SC_LD + part * (CPT + 1);
      uint32_t m = 0u;
#pragma unroll
      for (int j = 0; j < CPT; ++j) m |= ((cb + j < lim) && srow[j] >= thr_f) ? (1u << j) : 0u;
      while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const uint64_t key = route_key(srow[j], cb + j);
        if (key > keys[KM - 1]) {
          route_sorted_insert<KM>(keys, key);
          if (keys[KM - 1] != 0ull) thr_f = key_score(keys[KM - 1]);
        }
      }
    }
    // the next iteration's __syncthreads (after staging) keeps the score
    // tile alive until every thread has read it
  }

  // merge the TPR partial lists of each row (consecutive lanes)
#pragma unroll
  for (int mask = 1; mask < TPR; mask <<= 1) route_merge_partner<KM>(keys, mask);

  if (part == 0 && qb < a.NQB) {
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
      int32_t* dst = a.idx + (static_cast<int64_t>(bh) * a.NQB + qb) * k;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j < k) dst[j] = j < n ? sel[j] : -1;
    }
    a.cnt[static_cast<int64_t>(bh) * a.NQB + qb] = n;
  }
}

}  // namespace ssa
