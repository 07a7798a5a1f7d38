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
// kConsMaxVotes) go to the warp's shared-memory slab, a bitonic sort brings
// equal blocks together, each run's length is its vote count, and a second
// sort on the key (votes << 23 | (2^23 - 1 - block)) ranks the runs; the
// winners are sorted once more by block index.  The work is a few hundred
// shared-memory operations per query block, negligible beside the router.
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

// bitonic sort of x[0..P) (P a power of two >= 32) by one warp, ascending or
// descending, through shared memory
__device__ __forceinline__ void cons_warp_sort(uint32_t* x, int P, bool descending, int lane) {
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < P; i += 32) {
        const int l = i ^ j;
        if (l > i) {
          const uint32_t u = x[i], w = x[l];
          const bool up = (((i & k) == 0) != descending);
          if ((u > w) == up) {
            x[i] = w;
            x[l] = u;
          }
        }
      }
      __syncwarp();
    }
  }
}

__global__ void __launch_bounds__(kConsThreads) consensus_kernel(const ConsensusArgs a) {
  __shared__ uint32_t slab[kConsWarps][kConsMaxVotes];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kConsWarps + warp;
  if (row >= a.n_rows) return;  // warp-uniform
  const int g = a.Hq / a.Hkv;
  const int k = a.top_k;
  const int64_t bkv = row / a.NQB;
  const int qb = static_cast<int>(row % a.NQB);
  const int b = static_cast<int>(bkv / a.Hkv), kv = static_cast<int>(bkv % a.Hkv);
  const int E = g * k;
  int P = 32;
  while (P < E) P <<= 1;
  uint32_t* x = slab[warp];
  constexpr uint32_t kEmpty = 0xFFFFFFFFu;

  // 1. the group's votes: entry e is head (e / k)'s (e % k)-th block
  for (int e = lane; e < P; e += 32) {
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
    x[e] = val;
  }
  __syncwarp();
  cons_warp_sort(x, P, false, lane);

  // 2. one key per distinct block (at the first entry of its run):
  //    votes << 23 | (2^23 - 1 - block); 0 elsewhere.  Blocks are < 2^23
  //    (checked by the host) and votes <= P <= 512 < 2^9.
  constexpr int kMaxPer = kConsMaxVotes / 32;
  uint32_t key[kMaxPer];
#pragma unroll
  for (int s = 0; s < kMaxPer; ++s) {
    const int e = lane + 32 * s;
    key[s] = 0u;
    if (e < P) {
      const uint32_t c = x[e];
      if (c != kEmpty && (e == 0 || x[e - 1] != c)) {
        uint32_t votes = 1;
        while (e + static_cast<int>(votes) < P && x[e + votes] == c) ++votes;
        key[s] = (votes << 23) | (0x7FFFFFu - c);
      }
    }
  }
  __syncwarp();
#pragma unroll
  for (int s = 0; s < kMaxPer; ++s) {
    const int e = lane + 32 * s;
    if (e < P) x[e] = key[s];
  }
  __syncwarp();
  cons_warp_sort(x, P, true, lane);

  // 3. the first min(k, #runs) keys win; list their blocks ascending
  int P2 = 32;
  while (P2 < k) P2 <<= 1;  // k <= 64, so P2 <= 64 <= P
  uint32_t win[2];
  int n_win = 0;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int e = lane + 32 * s;
    const uint32_t kk = (e < P2) ? x[e] : 0u;
    const bool real = e < k && kk != 0u;
    win[s] = real ? (0x7FFFFFu - (kk & 0x7FFFFFu)) : kEmpty;
    n_win += __popc(__ballot_sync(0xffffffffu, real));
  }
  __syncwarp();
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int e = lane + 32 * s;
    if (e < P2) x[e] = win[s];
  }
  __syncwarp();
  cons_warp_sort(x, P2, false, lane);
  int32_t* dst = a.idx_kv + (bkv * a.NQB + qb) * k;
  for (int e = lane; e < k; e += 32) dst[e] = e < n_win ? static_cast<int32_t>(x[e]) : -1;
  if (lane == 0) a.cnt_kv[bkv * a.NQB + qb] = n_win;
}

}  // namespace ssa
