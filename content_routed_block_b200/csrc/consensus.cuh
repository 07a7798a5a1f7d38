// K2b: GQA-shared (consensus) route -- one list per (b, KV head, query block).
//
// jonsmirl/ssa README, "Complete 10M transformer result": one route is formed
// across heads by consensus and carries the blocks with the most votes;
// "Mathematical status": a highest-count reservoir keeps the items that the
// per-head selectors voted for most often.  Every query head of a KV group
// votes once for each block of its own top-k list (written by the router);
// the group keeps the first min(top_k, #voted blocks) blocks in the order
// (votes descending, block index ascending) and lists them ascending, padded
// with -1, with their count.
//
// One warp per (b, KV head, query block).  The g*top_k votes (at most
// kConsMaxVotes) are sorted in registers (bitonic: register exchanges and
// shuffles), which brings equal blocks together; each run's length is its
// vote count (read from one shared-memory copy); a second sort on the key
// (votes << 23 | (2^23 - 1 - block)) ranks the runs, and the winners are
// sorted once more by block index.
#pragma once

#include "common.cuh"

namespace ssa {

constexpr int kConsThreads = 256;
constexpr int kConsWarps = kConsThreads / 32;
constexpr int kConsMaxVotes = 512;  // g * top_k limit

struct ConsensusArgs {
  const int32_t* idx;  // [B*Hq, NQB, top_k] per-head lists
  const int32_t* cnt;  // [B*Hq, NQB]
  int32_t* idx_kv;     // [B*Hkv, NQB, top_k] consensus lists (out)
  int32_t* cnt_kv;     // [B*Hkv, NQB] (out)
  int32_t Hq, Hkv, NQB, NB, top_k;
  int64_t n_rows;      // B * Hkv * NQB
};

// bitonic sort of 32*R values held as element e = lane + 32 r in registers
// (r-th register of lane `lane`), ascending; partners at distance >= 32 sit
// in the same lane, the others are reached by shuffles
template <int R, typename T>
__device__ __forceinline__ void cons_sort_regs(T (&x)[R], int lane) {
#pragma unroll
  for (int k = 2; k <= 32 * R; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
        const int jr = j >> 5;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int pr = r ^ jr;
          if (pr > r) {
            const bool asc = ((lane + 32 * r) & k) == 0;
            const T lo = x[r] < x[pr] ? x[r] : x[pr], hi = x[r] < x[pr] ? x[pr] : x[r];
            x[r] = asc ? lo : hi;
            x[pr] = asc ? hi : lo;
          }
        }
      } else {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const T y = __shfl_xor_sync(0xffffffffu, x[r], j);
          const bool asc = ((lane + 32 * r) & k) == 0;
          const bool low = (lane & j) == 0;
          x[r] = (low == asc) ? (x[r] < y ? x[r] : y) : (x[r] < y ? y : x[r]);
        }
      }
    }
  }
}

// R = P / 32 entries per lane, P = the vote count g*top_k rounded up to a
// power of two (>= 32)
template <int R>
__global__ void __launch_bounds__(kConsThreads) consensus_kernel(const ConsensusArgs a) {
  constexpr int P = 32 * R;
  __shared__ uint32_t slab[kConsWarps][P];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kConsWarps + warp;
  if (row >= a.n_rows) return;  // warp-uniform
  const int g = a.Hq / a.Hkv;
  const int k = a.top_k;
  const int64_t bkv = row / a.NQB;
  const int qb = static_cast<int>(row % a.NQB);
  const int b = static_cast<int>(bkv / a.Hkv), kv = static_cast<int>(bkv % a.Hkv);
  const int E = g * k;
  uint32_t* x = slab[warp];
  constexpr uint32_t kEmpty = 0xFFFFFFFFu;

  // 1. the group's votes: entry e is head (e / k)'s (e % k)-th block
  uint32_t v[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = lane + 32 * r;
    uint32_t val = kEmpty;
    if (e < E) {
      const int j = e / k, t = e % k;
      const int64_t hrow = (static_cast<int64_t>(b) * a.Hq + kv * g + j) * a.NQB + qb;
      int n = a.cnt[hrow];
      if (n < 0 || n > k) {
        record_error(kErrCheck, kSiteCons);
        n = min(max(n, 0), k);
      }
      if (t < n) {
        const int c = a.idx[hrow * k + t];
        if (c >= 0 && c < a.NB)
          val = static_cast<uint32_t>(c);
        else
          record_error(kErrCheck, kSiteCons);
      }
    }
    v[r] = val;
  }
  cons_sort_regs<R>(v, lane);

  // 2. one key per distinct block (at the first entry of its run):
  //    votes << 23 | (2^23 - 1 - block); 0 elsewhere.  Blocks are < 2^23
  //    (checked by the host) and votes <= P <= 512 < 2^9.
#pragma unroll
  for (int r = 0; r < R; ++r) x[lane + 32 * r] = v[r];
  __syncwarp();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = lane + 32 * r;
    const uint32_t c = v[r];
    uint32_t key = 0u;
    if (c != kEmpty && (e == 0 || x[e - 1] != c)) {
      uint32_t votes = 1;
      while (e + static_cast<int>(votes) < P && x[e + votes] == c) ++votes;
      key = (votes << 23) | (0x7FFFFFu - c);
    }
    v[r] = ~key;  // ascending sort of ~key == descending sort of key
  }
  cons_sort_regs<R>(v, lane);

  // 3. the first min(k, #runs) keys win; list their blocks ascending.  The
  //    winners are elements 0 .. k-1 (k <= 64: registers 0 and 1).
  uint32_t w[2];
  int n_win = 0;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const uint32_t kk = (r < R) ? ~v[r] : 0u;
    const int e = lane + 32 * r;
    const bool real = e < k && kk != 0u;
    w[r] = real ? (0x7FFFFFu - (kk & 0x7FFFFFu)) : kEmpty;
    n_win += __popc(__ballot_sync(0xffffffffu, real));
  }
  if (k > 32) {
    cons_sort_regs<2>(w, lane);
  } else {
    uint32_t w1[1] = {w[0]};
    cons_sort_regs<1>(w1, lane);
    w[0] = w1[0];
  }
  int32_t* dst = a.idx_kv + (bkv * a.NQB + qb) * k;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int e = lane + 32 * r;
    if (e < k) dst[e] = e < n_win ? static_cast<int32_t>(w[r]) : -1;
  }
  if (lane == 0) a.cnt_kv[bkv * a.NQB + qb] = n_win;
}

}  // namespace ssa
