// K3: fused attend over the routed blocks and the local window.
//
// jonsmirl/ssa README, introduction: for each query, select a small set of
// key blocks, add a local causal window, and compute ordinary softmax
// attention over the selected keys without forming the dense n x n matrix;
// "Mathematical status": the routed set is causal once it is masked at each
// query's original position.  For query i in query block qb the key set is
// (keys of the routed blocks of qb) U {i-W < j <= i}, cut at j <= i (causal)
// or the routed blocks' keys alone (non-causal), each key counted once; the
// read is exact softmax over that set.  The append law on the same page
// (adding mass a to Z moves the read by a/(Z+a) of the displacement) is the
// online-softmax merge this kernel performs chunk by chunk.
//
// B200 design (one CTA = 128 query rows of one (b, head), i.e. 128/Bq query
// blocks; or, with GQA-shared consensus lists, 64 rows of each of two query
// heads of one KV group, which read the same key set so that every chunk
// serves all 128 rows; 192 threads):
//  * The CTA first builds the union of its query blocks' routed blocks and
//    the window's blocks in shared memory (deduplicated), each entry carrying
//    a bitmask of which query blocks routed it, with routed entries
//    interleaved across the softmax warps that need them.  The union is
//    walked in chunks of 64 keys (one or more whole blocks, or a 64-row slice
//    of a larger block), so every key block is fetched once per CTA.
//  * Warp 4 (one lane) gathers each chunk's K and V rows with tiled TMA loads
//    (one box per block, each CTA fetching its own) into a 128-byte-swizzled ring of
//    STAGES stages; Q (128 x D) is loaded once.
//  * Warp 5 (one lane) issues tcgen05.mma: S = Q K^T (M=128, N=64, fp32 in
//    TMEM, two S buffers) and O += P V (A = P read from TMEM, B = V as an
//    MN-major shared-memory operand, N = D, fp32 accumulator in TMEM).
//  * Warps 0-3 own one query row each per thread (TMEM lane = row): they
//    load S, apply the row's mask (routed bit of its query block, window,
//    causal cut), keep the running max / sum in fp32, write P as bf16 back
//    over S in TMEM, and rescale O in TMEM only when the max has grown by
//    more than 2^8 (the result is exact either way; the lazy update only
//    bounds the magnitudes).  The epilogue divides by the sum, rounds to
//    bf16 and writes O and the natural-log LSE.
//  * Every wait is bounded (mbar_wait): on a timeout the CTA raises a shared
//    abort flag, each role leaves its loop, the producer and the MMA issuer
//    wait for their copies / MMAs in flight, and TMEM is freed.
#pragma once

#include "common.cuh"

namespace ssa {

constexpr int kAtQT = 128;       // query rows per CTA (MMA M)
constexpr int kAtKT = 64;        // keys per chunk (MMA N of S)
constexpr int kAtLCap = 1024;    // window entries capacity
constexpr int kAtFarCap = 512;   // routed entries outside the window (>= 8 * 64)
constexpr int kAtThreads = 192;
constexpr uint32_t kAtTmemCols = 256;
constexpr float kAtTau = 8.0f;   // lazy-rescale threshold, log2 units

template <int D>
struct AtLayout {
  static constexpr int STAGES = (D == 64) ? 5 : 2;   // K/V ring depth
  static constexpr int NS = (D == 64) ? 3 : 2;       // S/P buffers in TMEM
  static constexpr uint32_t HALF_Q = kAtQT * 128;      // one 64-column half of Q
  static constexpr uint32_t Q_BYTES = kAtQT * D * 2;
  static constexpr uint32_t HALF_KV = kAtKT * 128;     // one 64-column half of a chunk
  static constexpr uint32_t KV_BYTES = kAtKT * D * 2;  // one K (or V) chunk
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr uint32_t OFF_WIN = OFF_V + STAGES * KV_BYTES;   // uint32 [kAtLCap]
  static constexpr uint32_t OFF_FAR = OFF_WIN + kAtLCap * 4;       // int32 [kAtFarCap]
  static constexpr uint32_t OFF_FARU = OFF_FAR + kAtFarCap * 4;    // int32 [kAtFarCap]
  static constexpr int NBAR = 1 + 2 * STAGES + 3 * NS + 1;
  static constexpr uint32_t OFF_BAR = OFF_FARU + kAtFarCap * 4;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t USED = OFF_MISC + 64;
  // request enough shared memory that at most two CTAs share an SM, so the
  // two 256-column TMEM allocations always fit in the SM's 512 columns
  static constexpr uint32_t MIN_REQ = 80 * 1024;
  static constexpr uint32_t SMEM_BYTES = (USED + 1024 > MIN_REQ) ? USED + 1024 : MIN_REQ;
  // TMEM columns: NS S buffers of 64 columns at 0, 64, ... (P overwrites the
  // first 32 columns of its S buffer as packed bf16 pairs); O after them
  static constexpr uint32_t TM_S0 = 0, TM_O = NS * 64;
  static_assert(TM_O + D <= kAtTmemCols, "TMEM budget");
};

struct AttendArgs {
  const int32_t* idx;    // [B*idx_heads, NQB, top_k]
  const int32_t* cnt;    // [B*idx_heads, NQB]
  __nv_bfloat16* o;      // [B*Hq, N, D]
  float* lse;            // [B*Hq, N] or null
  int32_t Hq, Hkv, N, NQB, NB, Bq, Bk, top_k, window, causal;
  int32_t idx_heads;     // Hq: a list per query head; Hkv: one list per KV group
  int32_t pack;          // query heads per CTA: 1, or 2 (two heads of a group
                         // sharing one list, 64 rows each)
  int32_t n_qtiles;      // ceil(N / (kAtQT / pack))
  float scale_log2;      // softmax scale * log2(e)
  uint64_t timeout_ns;
};

// union entry: (block << 8) | routed-bits (bit r: query block r of the tile
// routed this block)
__device__ __forceinline__ uint32_t at_entry(const int32_t* faru, const uint32_t* win, int nf,
                                             int wlo, int e) {
  if (e < nf) return static_cast<uint32_t>(faru[e]);
  const int w = e - nf;
  return (static_cast<uint32_t>(wlo + w) << 8) | (win[w] & 0xFFu);
}

// bits [lo, hi) of a 64-bit word
__device__ __forceinline__ uint64_t bit_range(int lo, int hi) {
  if (hi <= lo) return 0ull;
  const int n = hi - lo;
  const uint64_t m = (n >= 64) ? ~0ull : ((1ull << n) - 1ull);
  return m << lo;
}

// Union of a query tile's routed blocks and its window blocks, in shared
// memory: every key block the tile's R query blocks read, once, each routed
// entry carrying a bitmask of which query blocks routed it (bit r: query
// block qb0 + r), ordered so that chunks needed by different softmax warps
// alternate (see the comments inside).  On return (after a block-wide
// barrier) misc[2] holds the number of routed entries outside the window
// range, stored in faru[]; the window range's blocks wlo .. wlo + nwin - 1
// carry their routed bits in win[].  Called by every thread of a 192-thread
// CTA; used by the forward read and by the query-major kernel of its
// backward, so both walk exactly the same key sets.
__device__ __forceinline__ void at_build_union(const AttendArgs& a, int R, int RH, int q0, int qb0,
                                               int64_t ibh, int wlo, int nwin, int pre_n,
                                               int pre_c, uint32_t* win, int32_t* far,
                                               int32_t* faru, uint32_t* misc) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = R * a.top_k;
  const int G = (a.Bk < kAtKT) ? kAtKT / a.Bk : 1;           // blocks per chunk
  {
    for (int t = tid; t < total; t += kAtThreads) {
      const int r = t / a.top_k, e = t % a.top_k;
      const int64_t row = static_cast<int64_t>(ibh) * a.NQB + qb0 + r;
      int n = (t == tid) ? pre_n : a.cnt[row];
      if (n > a.top_k || n < 0) {
        record_error(kErrCheck, kSiteIdx);
        n = min(max(n, 0), a.top_k);
      }
      if (e >= n) continue;
      const int c = (t == tid) ? pre_c : a.idx[row * a.top_k + e];
      if (c < 0 || c >= a.NB) {
        record_error(kErrCheck, kSiteIdx);
        continue;
      }
      const uint32_t bit = 1u << r;
      if (a.causal && c >= wlo) {
        if (c - wlo < nwin) atomicOr(&win[c - wlo], bit);
        // a block entirely after the tile's last query contributes nothing
      } else {
        const int pos = static_cast<int>(atomicAdd(&misc[1], 1u));
        far[pos] = (c << 8) | static_cast<int>(bit);
      }
    }
  }
  __syncthreads();
  if (warp == 0 && static_cast<int>(misc[1]) <= 32 && G == 1) {
    // Few routed entries outside the window (the common case, e.g. 2 query
    // blocks x 16): the whole union list is built in registers, one entry
    // per lane, in the same order as the general path below.
    const int nfar = static_cast<int>(misc[1]);
    int x = lane < nfar ? far[lane] : 0x7FFFFFFF;
    // ascending bitonic sort across the lanes
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const int y = __shfl_xor_sync(0xffffffffu, x, j);
        const bool asc = (lane & k) == 0;
        const bool low = (lane & j) == 0;
        x = (low == asc) ? min(x, y) : max(x, y);
      }
    }
    // deduplicate: the first lane of each run of one block ORs the routed
    // bits of the run (at most one entry per query block of the tile: <= 8)
    const int c = x >> 8;
    const int prev = __shfl_up_sync(0xffffffffu, x, 1);
    const bool head = lane < nfar && (lane == 0 || (prev >> 8) != c);
    int bits = x & 0xFF;
#pragma unroll
    for (int d = 1; d < 8; ++d) {
      const int nb = __shfl_down_sync(0xffffffffu, x, d);
      if (lane + d < nfar && (nb >> 8) == c) bits |= nb & 0xFF;
    }
    const uint32_t hm = __ballot_sync(0xffffffffu, head);
    const int nf = __popc(hm);
    if (head) faru[__popc(hm & ((1u << lane) - 1u))] = (c << 8) | bits;
    __syncwarp();
    // interleave: class = which softmax warps need the entry; order by
    // (rank within the class, class), i.e. round-robin over the classes
    const int e = lane < nf ? faru[lane] : 0;
    int m = 32 + lane;  // distinct for the empty lanes
    if (lane < nf) {
      m = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int i_lo = q0 + (32 * w) % RH;
        const int lo = i_lo / a.Bq - qb0, hi = min(R - 1, (i_lo + 31) / a.Bq - qb0);
        const uint32_t qm = (lo < R) ? ((2u << hi) - (1u << lo)) : 0u;
        m |= ((static_cast<uint32_t>(e) & 0xFFu & qm) != 0u) << w;
      }
    }
    const uint32_t same = __match_any_sync(0xffffffffu, m);
    const int rank = __popc(same & ((1u << lane) - 1u));
    uint64_t kv = lane < nf ? ((static_cast<uint64_t>(rank * 16 + m) << 32) | static_cast<uint32_t>(e))
                            : ~0ull;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, kv, j);
        const bool asc = (lane & k) == 0;
        const bool low = (lane & j) == 0;
        kv = (low == asc) ? (kv < y ? kv : y) : (kv < y ? y : kv);
      }
    }
    if (lane < nf) faru[lane] = static_cast<int>(static_cast<uint32_t>(kv));
    if (lane == 0) misc[2] = static_cast<uint32_t>(nf);
  } else if (warp == 0) {
    const int nfar = static_cast<int>(misc[1]);
    int P = 1;
    while (P < nfar) P <<= 1;
    for (int i = nfar + lane; i < P; i += 32) far[i] = 0x7FFFFFFF;
    __syncwarp();
    for (int k = 2; k <= P; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = lane; i < P; i += 32) {
          const int l = i ^ j;
          if (l > i) {
            const int x = far[i], y = far[l];
            const bool asc = (i & k) == 0;
            if ((x > y) == asc) {
              far[i] = y;
              far[l] = x;
            }
          }
        }
        __syncwarp();
      }
    }
    int base = 0;
    for (int i0 = 0; i0 < nfar; i0 += 32) {
      const int i = i0 + lane;
      bool head = false;
      int ent = 0;
      if (i < nfar) {
        const int c = far[i] >> 8;
        head = (i == 0) || ((far[i - 1] >> 8) != c);
        if (head) {
          int bits = 0;
          for (int k = i; k < nfar && (far[k] >> 8) == c; ++k) bits |= far[k] & 0xFF;
          ent = (c << 8) | bits;
        }
      }
      const uint32_t hm = __ballot_sync(0xffffffffu, head);
      if (head) faru[base + __popc(hm & ((1u << lane) - 1u))] = ent;
      base += __popc(hm);
    }
    __syncwarp();
    // Interleave: softmax warp w serves rows 32w..32w+31, and a chunk that
    // none of its rows' query blocks routed costs it almost nothing, but the
    // warps share the S/P buffers, so they can drift only a few chunks
    // apart.  Order the routed entries round-robin over their "which warps
    // need it" classes so that chunks exclusive to different warps alternate.
    {
      const int nf = base;
      uint32_t qm[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int i_lo = q0 + (32 * w) % RH;
        const int lo = i_lo / a.Bq - qb0, hi = min(R - 1, (i_lo + 31) / a.Bq - qb0);
        qm[w] = (lo < R) ? ((2u << hi) - (1u << lo)) : 0u;
      }
      auto wmask = [&](int e) -> int {
        const uint32_t bits = static_cast<uint32_t>(faru[e]) & 0xFFu;
        int m = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) m |= ((bits & qm[w]) != 0u) << w;
        return m;
      };
      int bc[16];
#pragma unroll
      for (int bkt = 0; bkt < 16; ++bkt) bc[bkt] = 0;
      // class sizes
      for (int i0 = 0; i0 < nf; i0 += 32) {
        const int m = (i0 + lane < nf) ? wmask(i0 + lane) : -1;
#pragma unroll
        for (int bkt = 0; bkt < 16; ++bkt) bc[bkt] += __popc(__ballot_sync(0xffffffffu, m == bkt));
      }
      // Position.  With one block per chunk (Bk >= 64): round-robin over the
      // classes, so that chunks exclusive to different warps alternate.
      // With G blocks per chunk (Bk < 64): class by class, so that a chunk's
      // blocks mostly serve one warp and the other warps skip it (measured
      // on 16-key blocks: 0.360 ms against 0.395 ms for the round-robin and
      // 0.425 ms for class-pure chunks padded with masked slots).
      int seen[16];
#pragma unroll
      for (int bkt = 0; bkt < 16; ++bkt) seen[bkt] = 0;
      for (int i0 = 0; i0 < nf; i0 += 32) {
        const int e = i0 + lane;
        const int m = (e < nf) ? wmask(e) : -1;
        int rank = 0;  // index of the entry within its class, in block order
#pragma unroll
        for (int bkt = 0; bkt < 16; ++bkt) {
          const uint32_t bm = __ballot_sync(0xffffffffu, m == bkt);
          if (m == bkt) rank = seen[bkt] + __popc(bm & ((1u << lane) - 1u));
          seen[bkt] += __popc(bm);
        }
        if (e < nf) {
          int pos = 0;
          if (G == 1) {
#pragma unroll
            for (int bkt = 0; bkt < 16; ++bkt) pos += min(bc[bkt], rank) + ((bkt < m && bc[bkt] > rank) ? 1 : 0);
          } else {
#pragma unroll
            for (int bkt = 0; bkt < 16; ++bkt) pos += (bkt < m) ? bc[bkt] : 0;
            pos += rank;
          }
          far[pos] = faru[e];
        }
      }
      __syncwarp();
      for (int e = lane; e < nf; e += 32) faru[e] = far[e];
    }
    if (lane == 0) misc[2] = static_cast<uint32_t>(base);
  }
  __syncthreads();

}

template <int D>
__global__ void __launch_bounds__(kAtThreads, 2)
    attend_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const AttendArgs a) {
  using L = AtLayout<D>;
  constexpr int S = L::STAGES;
  extern __shared__ uint8_t at_smem_raw[];
  // 1024-byte aligned start, as an offset into the shared array (not through an
  // integer cast, which would drop the shared address space from every pointer
  // derived from it and turn their loads into generic ones)
  uint8_t* smem = at_smem_raw + ((1024u - (smem_u32(at_smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint32_t* win = reinterpret_cast<uint32_t*>(smem + L::OFF_WIN);
  int32_t* far = reinterpret_cast<int32_t*>(smem + L::OFF_FAR);
  int32_t* faru = reinterpret_cast<int32_t*>(smem + L::OFF_FARU);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_empty = bars + 1 + S;
  constexpr int NS = L::NS;
  uint64_t* bar_s_full = bars + 1 + 2 * S;
  uint64_t* bar_p_full = bar_s_full + NS;
  uint64_t* bar_pv_done = bar_p_full + NS;
  uint64_t* bar_drain = bar_pv_done + NS;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  // misc[0] TMEM base, misc[1] raw far count, misc[2] unique far count,
  // misc[3] abort flag
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[3]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The tile is RH consecutive query positions of `pack` query heads: rows
  // 0..RH-1 belong to head h0, rows RH..2RH-1 (pack == 2) to head h1 of the
  // same KV group, which shares h0's routed lists.  With an odd group the
  // last pair has no h1: its rows are loaded from h0 and never written.
  const int RH = kAtQT / a.pack;
  const int tile_bh = blockIdx.x / a.n_qtiles;
  const int qt = blockIdx.x % a.n_qtiles;
  const int grp = a.Hq / a.Hkv;
  int b, h0, h1;
  bool has_h1 = false;
  if (a.pack == 1) {
    b = tile_bh / a.Hq;
    h0 = tile_bh % a.Hq;
    h1 = h0;
  } else {
    const int npair = (grp + 1) / 2;
    const int bk = tile_bh / npair, pr = tile_bh % npair;
    b = bk / a.Hkv;
    h0 = (bk % a.Hkv) * grp + 2 * pr;
    has_h1 = 2 * pr + 1 < grp;
    h1 = has_h1 ? h0 + 1 : h0;
  }
  const int bh = b * a.Hq + h0;
  const int bkv = b * a.Hkv + h0 / grp;
  const int ibh = (a.idx_heads == a.Hq) ? bh : bkv;  // row block of the routed lists
  const int q0 = qt * RH;
  const int qend = min(a.N, q0 + RH);
  const int qb0 = q0 / a.Bq;
  const int R = min(max(RH / a.Bq, 1), a.NQB - qb0);
  int wlo = 0, nwin = 0;
  if (a.causal) {
    wlo = max(0, q0 - a.window + 1) / a.Bk;
    nwin = (qend - 1) / a.Bk - wlo + 1;
  }

  // this thread's first routed entry, loaded before the set-up so that the
  // load latency overlaps the barrier and TMEM set-up (reading the entry
  // past the row's count stays inside the row: rows are top_k long)
  const int total = R * a.top_k;
  int pre_n = 0, pre_c = -1;
  if (tid < total) {
    const int64_t row = static_cast<int64_t>(ibh) * a.NQB + qb0 + tid / a.top_k;
    pre_n = a.cnt[row];
    pre_c = a.idx[row * a.top_k + tid % a.top_k];
  }

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_s_full[s], 1);
      mbar_init(&bar_p_full[s], 4);  // one arrival per softmax warp
      mbar_init(&bar_pv_done[s], 1);
    }
    mbar_init(bar_drain, 1);
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&misc[0], kAtTmemCols);
    tmem_relinquish();
  }
  for (int w = tid; w < nwin; w += kAtThreads) win[w] = 0u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  // Q does not depend on the routing: start its load now
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    mbar_arrive_expect_tx(bar_q, L::Q_BYTES);
#pragma unroll
    for (int half = 0; half < D / 64; ++half) {
      // the tensor map's box is RH rows: one box per head
      tma_load_3d(smem + L::OFF_Q + half * L::HALF_Q, &tq, bar_q, half * 64, q0, bh);
      if (a.pack == 2)
        tma_load_3d(smem + L::OFF_Q + half * L::HALF_Q + 64 * 128, &tq, bar_q, half * 64, q0,
                    b * a.Hq + h1);
    }
  }

  // ------------------------------------------ union of routed and window blocks
  at_build_union(a, R, RH, q0, qb0, ibh, wlo, nwin, pre_n, pre_c, win, far, faru, misc);
  const int G = (a.Bk < kAtKT) ? kAtKT / a.Bk : 1;           // blocks per chunk
  const int nf = static_cast<int>(misc[2]);
  const int n_entries = nf + nwin;
  const int SUBS = (a.Bk > kAtKT) ? a.Bk / kAtKT : 1;        // chunks per block
  // a power of two: chunk t is sub-chunk t % SUBS of entry t / SUBS, by shifts
  // (a runtime division would cost a long dependent sequence in every chunk)
  const int subs_sh = __ffs(SUBS) - 1;
  const int T = (a.Bk >= kAtKT) ? n_entries * SUBS : (n_entries + G - 1) / G;
  int issued = 0;  // chunks the producer has put in flight

  if (warp == 4) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int t = 0; t < T; ++t) {
        const int st = t % S;
        if (t >= S && !mbar_wait(&bar_kv_empty[st], ((t / S) - 1) & 1, a.timeout_ns, abort_flag,
                                 kSiteKvEmpty))
          break;
        mbar_arrive_expect_tx(&bar_kv_full[st], 2 * L::KV_BYTES);
        uint8_t* kdst = smem + L::OFF_K + st * L::KV_BYTES;
        uint8_t* vdst = smem + L::OFF_V + st * L::KV_BYTES;
        if (a.Bk >= kAtKT) {
          const int e = t >> subs_sh, sub = t & (SUBS - 1);
          const int c = static_cast<int>(at_entry(faru, win, nf, wlo, e) >> 8);
          const int row0 = c * a.Bk + sub * kAtKT;
#pragma unroll
          for (int half = 0; half < D / 64; ++half) {
            tma_load_3d(kdst + half * L::HALF_KV, &tk, &bar_kv_full[st], half * 64, row0, bkv);
            tma_load_3d(vdst + half * L::HALF_KV, &tv, &bar_kv_full[st], half * 64, row0, bkv);
          }
        } else {
          for (int s = 0; s < G; ++s) {
            int e = t * G + s;
            if (e >= n_entries) e = t * G;  // pad a short last chunk with a real block (masked)
            const int c = static_cast<int>(at_entry(faru, win, nf, wlo, e) >> 8);
            const int row0 = c * a.Bk;
#pragma unroll
            for (int half = 0; half < D / 64; ++half) {
              tma_load_3d(kdst + half * L::HALF_KV + s * a.Bk * 128, &tk, &bar_kv_full[st],
                          half * 64, row0, bkv);
              tma_load_3d(vdst + half * L::HALF_KV + s * a.Bk * 128, &tv, &bar_kv_full[st],
                          half * 64, row0, bkv);
            }
          }
        }
        ++issued;
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------- MMA issuer
    // Event-driven: S(t) is issued as soon as chunk t has landed and its S
    // buffer is free (PV(t-NS), which read P(t-NS) from that buffer, is done),
    // up to NS chunks ahead of the PVs; PV(u) as soon as P(u) is written.
    // Probes are non-blocking; the whole loop gives up after timeout_ns
    // without progress.
    if (lane == 0 && T > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(kAtQT, kAtKT, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(kAtQT, D, false, true);
      bool ok = mbar_wait(bar_q, 0, a.timeout_ns, abort_flag, kSiteQFull);
      int ns = 0, np = 0;
      uint64_t t_last = globaltimer_ns();
      while (ok && np < T) {
        bool progress = false;
        if (ns < T && ns < np + NS) {
          bool ready = mbar_test(&bar_kv_full[ns % S], (ns / S) & 1);
          if (ready && ns >= NS) ready = mbar_test(&bar_pv_done[ns % NS], ((ns - NS) / NS) & 1);
          if (ready) {
            tc_fence_after();
            const uint32_t kbase = sbase + L::OFF_K + (ns % S) * L::KV_BYTES;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t qa = sbase + L::OFF_Q + (kk / 4) * L::HALF_Q + (kk % 4) * 32;
              const uint32_t kb = kbase + (kk / 4) * L::HALF_KV + (kk % 4) * 32;
              mma_ss(tmem + L::TM_S0 + (ns % NS) * 64, sdesc_sw128(qa, 16, 1024),
                     sdesc_sw128(kb, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar_s_full[ns % NS]);
            ++ns;
            progress = true;
          }
        }
        if (np < ns && mbar_test(&bar_p_full[np % NS], (np / NS) & 1)) {
          tc_fence_after();
          const uint32_t vbase = sbase + L::OFF_V + (np % S) * L::KV_BYTES;
          const uint32_t pcol = tmem + L::TM_S0 + (np % NS) * 64;
#pragma unroll
          for (int kk = 0; kk < kAtKT / 16; ++kk) {
            const uint64_t bdesc = sdesc_sw128(vbase + kk * 2048, L::HALF_KV, 1024);
            mma_ts(tmem + L::TM_O, pcol + kk * 8, bdesc, IDESC_O, (np > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar_pv_done[np % NS]);
          mma_commit(&bar_kv_empty[np % S]);
          ++np;
          progress = true;
        }
        if (progress) {
          t_last = globaltimer_ns();
        } else {
          if (*abort_flag) break;
          if (globaltimer_ns() - t_last > a.timeout_ns) {
            *abort_flag = 1;
            record_error(kErrTimeout, kSiteMma);
            break;
          }
        }
      }
      // every MMA issued so far must finish before TMEM is released
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0, a.timeout_ns, nullptr, kSiteDrain);
    }
  } else {
    // ------------------------------------------------------- softmax warps
    const int r = tid;  // row in the tile == TMEM lane
    const int slot = r / RH;
    const int i = q0 + r % RH;
    const bool row_ok = i < qend && (slot == 0 || has_h1);
    const int qbr = row_ok ? i / a.Bq - qb0 : 0;
    const int bh_row = b * a.Hq + (slot == 0 ? h0 : h1);
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    // running max of the raw scores (the scale is positive, so the max of the
    // scaled logits is sl2 times it) and running sum of 2^(x - max)
    float m_raw = -INFINITY, l_sum = 0.f;
    bool ok = true;

    for (int t = 0; t < T; ++t) {
      const bool got = mbar_wait(&bar_s_full[t % NS], (t / NS) & 1, a.timeout_ns, abort_flag,
                                 kSiteSFull);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t pcol = trow + L::TM_S0 + (t % NS) * 64;

      // allowed keys of this row within the chunk, as two 32-bit words
      uint32_t mlo = 0u, mhi = 0u;
      {
        uint64_t mask = 0ull;
        if (a.Bk >= kAtKT) {
          const int e = t >> subs_sh, sub = t & (SUBS - 1);
          const uint32_t ent = at_entry(faru, win, nf, wlo, e);
          const int j0 = static_cast<int>(ent >> 8) * a.Bk + sub * kAtKT;
          const bool routed = (ent >> qbr) & 1u;
          int lo = 0, hi = 0;
          if (a.causal) {
            hi = min(kAtKT, i - j0 + 1);
            lo = routed ? 0 : max(0, i - a.window + 1 - j0);
          } else {
            hi = routed ? kAtKT : 0;
          }
          mask = row_ok ? bit_range(lo, hi) : 0ull;
        } else {
          for (int s = 0; s < G; ++s) {
            const int e = t * G + s;
            if (e >= n_entries) break;
            const uint32_t ent = at_entry(faru, win, nf, wlo, e);
            if (!row_ok) continue;
            const int j0 = static_cast<int>(ent >> 8) * a.Bk;
            const bool routed = (ent >> qbr) & 1u;
            int lo = 0, hi = 0;
            if (a.causal) {
              hi = min(a.Bk, i - j0 + 1);
              lo = routed ? 0 : max(0, i - a.window + 1 - j0);
            } else {
              hi = routed ? a.Bk : 0;
            }
            mask |= bit_range(lo, hi) << (s * a.Bk);
          }
        }
        mlo = static_cast<uint32_t>(mask);
        mhi = static_cast<uint32_t>(mask >> 32);
      }

      // no row of this warp sees any key of the chunk (it was routed by the
      // tile's other query blocks only): P = 0 for these rows, nothing else
      if (__all_sync(0xffffffffu, (mlo | mhi) == 0u)) {
        uint32_t z[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) z[c] = 0u;
        tmem_st32(pcol, z);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p_full[t % NS]);
        continue;
      }

      uint32_t s0[32], s1[32];
      tmem_ld32(pcol, s0);
      tmem_ld32(pcol + 32, s1);
      tmem_ld_wait(s0);
      tmem_ld_wait(s1);
      float x[64];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[c] = __uint_as_float(s0[c]);
        x[c + 32] = __uint_as_float(s1[c]);
      }
      if (!__all_sync(0xffffffffu, (mlo & mhi) == 0xFFFFFFFFu)) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = (mlo & (1u << c)) ? x[c] : -INFINITY;
          x[c + 32] = (mhi & (1u << c)) ? x[c + 32] : -INFINITY;
        }
      }
      // row max: three-input max tree
      float mx;
      {
        float t1[22];
#pragma unroll
        for (int c = 0; c < 21; ++c) t1[c] = fmax3(x[3 * c], x[3 * c + 1], x[3 * c + 2]);
        t1[21] = x[63];
        float t2[8];
#pragma unroll
        for (int c = 0; c < 7; ++c) t2[c] = fmax3(t1[3 * c], t1[3 * c + 1], t1[3 * c + 2]);
        t2[7] = t1[21];
        mx = fmax3(fmax3(t2[0], t2[1], t2[2]), fmax3(t2[3], t2[4], t2[5]), fmaxf(t2[6], t2[7]));
      }
      const float m_new = fmaxf(m_raw, mx);
      const bool need = (m_raw != -INFINITY) && ((m_new - m_raw) * sl2 > kAtTau);
      if (__any_sync(0xffffffffu, need)) {
        // rescale the O row in TMEM; PV(t-1) must have landed first
        if (t >= 1) {
          const bool g2 = mbar_wait(&bar_pv_done[(t - 1) % NS], ((t - 1) / NS) & 1,
                                    a.timeout_ns, abort_flag, kSitePvDone);
          if (!__all_sync(0xffffffffu, g2)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const float alpha =
            (m_raw == -INFINITY || m_new == m_raw) ? 1.f : ex2_approx((m_raw - m_new) * sl2);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(trow + L::TM_O + cc * 32, ov);
          tmem_ld_wait(ov);
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          tmem_st32(trow + L::TM_O + cc * 32, ov);
        }
        tmem_st_wait();
        l_sum *= alpha;
        m_raw = m_new;
      } else if (m_raw == -INFINITY) {
        m_raw = m_new;  // first keys of this row: O and the sum are still zero
      }
      // p = 2^(x*sl2 - m*sl2): one packed FMA per pair, one ex2 per score
      const float moff = (m_raw == -INFINITY) ? 0.f : -m_raw * sl2;
      uint32_t p[32];
      float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float y0, y1, y2, y3;
        ffma2_bc(y0, y1, x[2 * c], x[2 * c + 1], sl2, moff);
        ffma2_bc(y2, y3, x[2 * c + 2], x[2 * c + 3], sl2, moff);
        const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
        const float p2 = ex2_approx(y2), p3 = ex2_approx(y3);
        fadd2(acc0, acc1, acc0, acc1, p0, p1);
        fadd2(acc2, acc3, acc2, acc3, p2, p3);
        p[c] = pack_bf16x2(p0, p1);
        p[c + 1] = pack_bf16x2(p2, p3);
      }
      l_sum += (acc0 + acc1) + (acc2 + acc3);
      tmem_st32(pcol, p);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_p_full[t % NS]);
    }

    // ------------------------------------------------------- epilogue
    if (ok && T > 0) {
      const bool got = mbar_wait(&bar_pv_done[(T - 1) % NS], ((T - 1) / NS) & 1, a.timeout_ns,
                                 abort_flag, kSitePvDone);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok && !*abort_flag) {
      tc_fence_after();
      const float inv = (l_sum > 0.f) ? 1.f / l_sum : 0.f;
      __nv_bfloat16* orow = a.o + (static_cast<int64_t>(bh_row) * a.N + i) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        if (T > 0) {
          tmem_ld32(trow + L::TM_O + cc * 32, ov);
          tmem_ld_wait(ov);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = 0u;
        }
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c] = pack_bf16x2(__uint_as_float(ov[2 * c]) * inv, __uint_as_float(ov[2 * c + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (row_ok && a.lse != nullptr) {
        const float lse2 = (l_sum > 0.f) ? m_raw * sl2 + __log2f(l_sum) : -INFINITY;
        a.lse[static_cast<int64_t>(bh_row) * a.N + i] = lse2 * 0.69314718055994530942f;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  // After an abort some copies may still be in flight: they must land before
  // the CTA exits.  On the normal path every chunk and Q were consumed, so
  // these waits return at once; Q is unconsumed when there was no chunk.
  if (warp == 4 && lane == 0) {
    if (*abort_flag) {
      for (int t = max(0, issued - S); t < issued; ++t)
        mbar_wait(&bar_kv_full[t % S], (t / S) & 1, a.timeout_ns, nullptr, kSiteDrain);
    }
    if (T == 0 || *abort_flag) mbar_wait(bar_q, 0, a.timeout_ns, nullptr, kSiteDrain);
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kAtTmemCols);
  }
}

}  // namespace ssa
