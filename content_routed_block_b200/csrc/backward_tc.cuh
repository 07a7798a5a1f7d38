// K5 (tensor-core form): backward of the read with the selection held fixed.
//
// jonsmirl/ssa README, introduction: within a query's key set the read is
// ordinary softmax attention; the routed lists are a discrete choice and carry
// no gradient.  For query i with key set S_i, P_ij = exp(scale <q_i, k_j> -
// lse_i), upstream gradient g_i and delta_i = <g_i, o_i>:
//   dv_j += P_ij g_i,   dS_ij = P_ij (<g_i, v_j> - delta_i),
//   dq_i = scale sum_j dS_ij k_j,   dk_j += scale dS_ij q_i.
//
// The five products per (query, key) tile are dense contractions, so both
// kernels run them as tcgen05 MMAs in the forward read's two forms (the
// QK^T form, both operands K-major in shared memory; and the PV form, A from
// tensor memory, B an MN-major shared-memory tile), fp32 accumulators in TMEM:
//
//  * bwd_dq_kernel<D> (query-major): the forward's tile (128 query rows of one
//    (b, head)), the same union of key blocks (at_build_union) walked in
//    chunks of 64 keys, so it visits exactly the forward's key sets.  Per
//    chunk: S = Q K^T and dP = G V^T into TMEM; the softmax warps (thread =
//    row) form P = 2^(S scale log2e - lse log2e), masked like the forward,
//    and dS = P (dP - delta); dq += dS K (the PV form with K as the B tile).
//  * bwd_map_kernel: the transpose of the lists as a bitmap: bit qc of row
//    (b, list head, key tile kt) is set when a query block of the 64-query
//    chunk qc routes a key block of the 128-key tile kt (atomic OR, so the
//    result does not depend on the order of the updates).
//  * bwd_dkdv_kernel<D> (key-major): one CTA per (128 keys, query head).  It
//    visits the head's 64-query chunks that read the tile -- the window
//    chunks and the routed ones from the bitmap, each once, in ascending
//    order; the lists of 32 visits are read at once, one lane per visit.
//    Per visit: S^T = K Q^T and dP^T = V G^T; the softmax warps (thread =
//    key) form P^T and dS^T; dv += P^T G and dk += dS^T Q accumulate in
//    TMEM.  With one query head per KV head the result is the gradient;
//    otherwise it is the head's share, and bwd_group_sum_kernel adds the
//    group's shares in head order.  No atomics anywhere: dk and dv are
//    reproducible bit for bit.  (One CTA per (tile, KV head) would serialise
//    all of a group's visits: causal lists read the early tiles far more
//    often -- up to 1300 visits against a mean of 262 at 32K tokens.)
//
// P and dS enter the MMAs as bf16 operands.  One bf16 keeps 8 significant
// bits, so each is split into two bf16 parts, x = hi + lo + r with
// |r| <= 2^-16 |x|, and both parts are multiplied (two MMAs per product):
// the result keeps about 16 bits, below the fp32-level rounding of the sums.
// In tensor memory the hi and lo parts of 32 columns share the 32 columns
// they came from: for each 32-column half, hi of its 32 values in the first
// 16 columns and lo in the next 16, so a half can be written as soon as it
// has been read.
//
// Every wait is bounded (mbar_wait / the forward's abort protocol); after a
// timeout every role leaves its loop, copies and MMAs in flight are drained
// and TMEM is freed.
#pragma once

#include "attend.cuh"
#include "common.cuh"

namespace ssa {

struct BwdTcArgs {
  AttendArgs at;          // lists, shapes and the forward's tiling (o / lse unused)
  const float* lse;       // [B*Hq, N] the forward's natural-log LSE
  const float* delta;     // [B*Hq, N] <g_i, o_i>
  float* delta_w;         // the same, written by bwd_prep_kernel
  float* lse2;            // [B*Hq, N] lse * log2(e), written by bwd_prep_kernel
  const __nv_bfloat16* o;     // [B*Hq, N, D] the forward's output
  const __nv_bfloat16* d_o;   // [B*Hq, N, D] upstream gradient
  float* dq;              // [B*Hq, N, D] (out)
  float* dk;              // [B*Hkv, N, D] (out)
  float* dv;              // [B*Hkv, N, D] (out)
  const uint32_t* map;    // [B*list_heads, n_ktiles, map_words] list transpose
  uint32_t* map_w;        // the same, written by bwd_map_kernel
  int32_t n_ktiles;       // ceil(N / 128)
  int32_t map_words;      // ceil(ceil(N / 64) / 32)
  int32_t B;              // batch
  float* part_dk;         // [B*Hq, N, D] per-query-head dk (scaled) when Hq > Hkv
  float* part_dv;         // [B*Hq, N, D] per-query-head dv when Hq > Hkv
  float scale;            // softmax scale
};

constexpr int kBkKT = 128;   // keys per dk/dv CTA (MMA M)
constexpr int kBkQC = 64;    // queries per visit (MMA N of S^T)

// column of the hi / lo part of K16 slice kk (16 values) in a 64-column
// buffer laid out as described above
__device__ __forceinline__ uint32_t split_col(int kk, bool lo) {
  return static_cast<uint32_t>((kk >> 1) * 32 + (lo ? 16 : 0) + (kk & 1) * 8);
}

// bf16 hi / lo parts of two fp32 values, packed in pairs (the first low)
__device__ __forceinline__ void split_pack2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16x2(x0 - __bfloat162float(h.x), x1 - __bfloat162float(h.y));
}

// the same for 32 fp32 values
__device__ __forceinline__ void split_pack32(const float (&x)[32], uint32_t (&hi)[16],
                                             uint32_t (&lo)[16]) {
#pragma unroll
  for (int c = 0; c < 16; ++c) split_pack2(x[2 * c], x[2 * c + 1], hi[c], lo[c]);
}

// the same for 32 fp32 values held as bit patterns
__device__ __forceinline__ void split_pack32_bits(const uint32_t (&x)[32], uint32_t (&hi)[16],
                                                  uint32_t (&lo)[16]) {
#pragma unroll
  for (int c = 0; c < 16; ++c)
    split_pack2(__uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1]), hi[c], lo[c]);
}

// ===========================================================================
// query-major kernel: dq
// ===========================================================================
template <int D>
struct DqLayout {
  static constexpr int STAGES = (D == 64) ? 4 : 2;   // K/V ring depth
  static constexpr int NS = (D == 64) ? 2 : 1;       // S buffers in TMEM
  static constexpr uint32_t HALF_Q = kAtQT * 128;
  static constexpr uint32_t Q_BYTES = kAtQT * D * 2;
  static constexpr uint32_t HALF_KV = kAtKT * 128;
  static constexpr uint32_t KV_BYTES = kAtKT * D * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_G = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_K = OFF_G + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr uint32_t OFF_WIN = OFF_V + STAGES * KV_BYTES;
  static constexpr uint32_t OFF_FAR = OFF_WIN + kAtLCap * 4;
  static constexpr uint32_t OFF_FARU = OFF_FAR + kAtFarCap * 4;
  // q | kv_full[S] | kv_empty[S] | sd_full[NS] | ds_full[NS] | dq_done[NS] | dp_free | drain
  static constexpr int NBAR = 1 + 2 * STAGES + 3 * NS + 2;
  static constexpr uint32_t OFF_BAR = OFF_FARU + kAtFarCap * 4;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t USED = OFF_MISC + 64;
  static constexpr uint32_t MIN_REQ = 80 * 1024;   // at most two CTAs per SM (TMEM)
  static constexpr uint32_t SMEM_BYTES = (USED + 1024 > MIN_REQ) ? USED + 1024 : MIN_REQ;
  // TMEM: dq at 0, NS S buffers of 64 columns, one dP buffer of 64 columns
  static constexpr uint32_t TM_DQ = 0, TM_S0 = D, TM_DP = D + NS * 64;
  static_assert(TM_DP + 64 <= kAtTmemCols, "TMEM budget");
};

template <int D>
__global__ void __launch_bounds__(kAtThreads, D == 64 ? 2 : 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tg,
                  const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                  const BwdTcArgs ba) {
  using L = DqLayout<D>;
  constexpr int S = L::STAGES, NS = L::NS;
  const AttendArgs& a = ba.at;
  extern __shared__ uint8_t dq_smem_raw[];
  // 1024-byte aligned start, as an offset into the shared array (not through an
  // integer cast, which would drop the shared address space from every pointer
  // derived from it and turn their loads into generic ones)
  uint8_t* smem = dq_smem_raw + ((1024u - (smem_u32(dq_smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint32_t* win = reinterpret_cast<uint32_t*>(smem + L::OFF_WIN);
  int32_t* far = reinterpret_cast<int32_t*>(smem + L::OFF_FAR);
  int32_t* faru = reinterpret_cast<int32_t*>(smem + L::OFF_FARU);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_empty = bars + 1 + S;
  uint64_t* bar_sd_full = bars + 1 + 2 * S;
  uint64_t* bar_ds_full = bar_sd_full + NS;
  uint64_t* bar_dq_done = bar_ds_full + NS;
  uint64_t* bar_dp_free = bar_dq_done + NS;
  uint64_t* bar_drain = bar_dp_free + 1;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[3]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // one query head per tile (the forward's pack == 1 layout)
  const int RH = kAtQT;
  const int tile_bh = blockIdx.x / a.n_qtiles;
  const int qt = blockIdx.x % a.n_qtiles;
  const int grp = a.Hq / a.Hkv;
  const int b = tile_bh / a.Hq, h0 = tile_bh % a.Hq;
  const int bh = b * a.Hq + h0;
  const int bkv = b * a.Hkv + h0 / grp;
  const int ibh = (a.idx_heads == a.Hq) ? bh : bkv;
  const int q0 = qt * RH;
  const int qend = min(a.N, q0 + RH);
  const int qb0 = q0 / a.Bq;
  const int R = min(max(RH / a.Bq, 1), a.NQB - qb0);
  int wlo = 0, nwin = 0;
  if (a.causal) {
    wlo = max(0, q0 - a.window + 1) / a.Bk;
    nwin = (qend - 1) / a.Bk - wlo + 1;
  }
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
      mbar_init(&bar_sd_full[s], 1);
      mbar_init(&bar_ds_full[s], 4);  // one arrival per softmax warp
      mbar_init(&bar_dq_done[s], 1);
    }
    mbar_init(bar_dp_free, 4);
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

  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tg);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    mbar_arrive_expect_tx(bar_q, 2 * L::Q_BYTES);
#pragma unroll
    for (int half = 0; half < D / 64; ++half) {
      tma_load_3d(smem + L::OFF_Q + half * L::HALF_Q, &tq, bar_q, half * 64, q0, bh);
      tma_load_3d(smem + L::OFF_G + half * L::HALF_Q, &tg, bar_q, half * 64, q0, bh);
    }
  }

  at_build_union(a, R, RH, q0, qb0, ibh, wlo, nwin, pre_n, pre_c, win, far, faru, misc);
  const int G = (a.Bk < kAtKT) ? kAtKT / a.Bk : 1;
  const int nf = static_cast<int>(misc[2]);
  const int n_entries = nf + nwin;
  const int SUBS = (a.Bk > kAtKT) ? a.Bk / kAtKT : 1;
  const int subs_sh = __ffs(SUBS) - 1;   // SUBS is a power of two
  const int T = (a.Bk >= kAtKT) ? n_entries * SUBS : (n_entries + G - 1) / G;
  int issued = 0;

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
    // S(t) and dP(t) go out once chunk t has landed, its S buffer is free
    // (dq(t - NS), which read dS(t - NS) from it, is done) and the softmax has
    // read dP(t - 1); dq(t) once dS(t) is written.
    if (lane == 0 && T > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(kAtQT, kAtKT, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(kAtQT, D, false, true);
      bool ok = mbar_wait(bar_q, 0, a.timeout_ns, abort_flag, kSiteQFull);
      int ns = 0, nd = 0;
      uint64_t t_last = globaltimer_ns();
      while (ok && nd < T) {
        bool progress = false;
        if (ns < T && ns < nd + NS) {
          bool ready = mbar_test(&bar_kv_full[ns % S], (ns / S) & 1);
          if (ready && ns >= NS) ready = mbar_test(&bar_dq_done[ns % NS], ((ns - NS) / NS) & 1);
          if (ready && ns >= 1) ready = mbar_test(bar_dp_free, (ns - 1) & 1);
          if (ready) {
            tc_fence_after();
            const uint32_t kbase = sbase + L::OFF_K + (ns % S) * L::KV_BYTES;
            const uint32_t vbase = sbase + L::OFF_V + (ns % S) * L::KV_BYTES;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_q = (kk / 4) * L::HALF_Q + (kk % 4) * 32;
              const uint32_t off_k = (kk / 4) * L::HALF_KV + (kk % 4) * 32;
              mma_ss(tmem + L::TM_S0 + (ns % NS) * 64,
                     sdesc_sw128(sbase + L::OFF_Q + off_q, 16, 1024),
                     sdesc_sw128(kbase + off_k, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_q = (kk / 4) * L::HALF_Q + (kk % 4) * 32;
              const uint32_t off_k = (kk / 4) * L::HALF_KV + (kk % 4) * 32;
              mma_ss(tmem + L::TM_DP, sdesc_sw128(sbase + L::OFF_G + off_q, 16, 1024),
                     sdesc_sw128(vbase + off_k, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar_sd_full[ns % NS]);
            ++ns;
            progress = true;
          }
        }
        if (nd < ns && mbar_test(&bar_ds_full[nd % NS], (nd / NS) & 1)) {
          tc_fence_after();
          const uint32_t kbase = sbase + L::OFF_K + (nd % S) * L::KV_BYTES;
          const uint32_t scol = tmem + L::TM_S0 + (nd % NS) * 64;
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int kk = 0; kk < kAtKT / 16; ++kk) {
              const uint64_t bdesc = sdesc_sw128(kbase + kk * 2048, L::HALF_KV, 1024);
              mma_ts(tmem + L::TM_DQ, scol + split_col(kk, part == 1), bdesc, IDESC_O,
                     (nd > 0 || kk > 0 || part > 0) ? 1u : 0u);
            }
          }
          mma_commit(&bar_dq_done[nd % NS]);
          mma_commit(&bar_kv_empty[nd % S]);
          ++nd;
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
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0, a.timeout_ns, nullptr, kSiteDrain);
    }
  } else {
    // ------------------------------------------------------- softmax warps
    const int r = tid;  // row in the tile == TMEM lane
    const int i = q0 + r;
    const bool row_ok = i < qend;
    const int qbr = row_ok ? i / a.Bq - qb0 : 0;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    const float lse2 = row_ok ? ba.lse[static_cast<int64_t>(bh) * a.N + i] * 1.4426950408889634f
                              : 0.f;
    const float del = row_ok ? ba.delta[static_cast<int64_t>(bh) * a.N + i] : 0.f;
    bool ok = true;

    for (int t = 0; t < T; ++t) {
      const bool got = mbar_wait(&bar_sd_full[t % NS], (t / NS) & 1, a.timeout_ns, abort_flag,
                                 kSiteSFull);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t scol = trow + L::TM_S0 + (t % NS) * 64;

      // allowed keys of this row within the chunk (exactly the forward's mask)
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

      if (__all_sync(0xffffffffu, (mlo | mhi) == 0u)) {
        // no row of this warp sees a key of the chunk: dS = 0, dP unread
        uint32_t z[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) z[c] = 0u;
        tmem_st32(scol, z);
        tmem_st32(scol + 32, z);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar_dp_free);
          mbar_arrive(&bar_ds_full[t % NS]);
        }
        continue;
      }

      // P = 2^(S sl2 - lse2) on the row's keys (0 elsewhere) and dS = P (dP -
      // delta), half by half: the half's S and dP come in one TMEM round trip,
      // and its dS parts go over the half of S just read
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t m = half ? mhi : mlo;
        uint32_t sv[32], dv32[32];
        tmem_ld32(scol + half * 32, sv);
        tmem_ld32(trow + L::TM_DP + half * 32, dv32);
        tmem_ld_wait(sv);
        tmem_ld_wait(dv32);
        float ds[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float pc = ex2_approx(fmaf(__uint_as_float(sv[c]), sl2, -lse2));
          ds[c] = (m >> c) & 1u ? pc * (__uint_as_float(dv32[c]) - del) : 0.f;
        }
        uint32_t hi[16], lo[16];
        split_pack32(ds, hi, lo);
        tmem_st16(scol + half * 32, hi);
        tmem_st16(scol + half * 32 + 16, lo);
      }
      // dP has been read (tcgen05.ld waited): the buffer may take dP(t + 1)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dp_free);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_ds_full[t % NS]);
    }

    // ------------------------------------------------------- epilogue
    if (ok && T > 0) {
      const bool got = mbar_wait(&bar_dq_done[(T - 1) % NS], ((T - 1) / NS) & 1, a.timeout_ns,
                                 abort_flag, kSitePvDone);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok && !*abort_flag) {
      tc_fence_after();
      float* drow = ba.dq + (static_cast<int64_t>(bh) * a.N + i) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        if (T > 0) {
          tmem_ld32(trow + L::TM_DQ + cc * 32, v);
          tmem_ld_wait(v);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = 0u;
        }
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(drow + cc * 32);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_float4(__uint_as_float(v[4 * c]) * ba.scale,
                                 __uint_as_float(v[4 * c + 1]) * ba.scale,
                                 __uint_as_float(v[4 * c + 2]) * ba.scale,
                                 __uint_as_float(v[4 * c + 3]) * ba.scale);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
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

// ===========================================================================
// transpose of the lists: bitmap of (key tile, query chunk) pairs
// ===========================================================================
// One thread per list slot.  Entries are checked like the CUDA-core
// backward checked them (count, range, ascending order, causal
// admissibility); a bad entry is reported through the error word and left
// out of the map.
__global__ void __launch_bounds__(256) bwd_map_kernel(const BwdTcArgs ba, int64_t n_slots) {
  const AttendArgs& a = ba.at;
  const int64_t s = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (s >= n_slots) return;
  const int64_t row = s / a.top_k;            // (b * list heads + lh) * NQB + qb
  const int e = static_cast<int>(s % a.top_k);
  const int qb = static_cast<int>(row % a.NQB);
  int n = a.cnt[row];
  if (n < 0 || n > a.top_k) {
    if (e == 0) record_error(kErrCheck, kSiteBwd);
    n = min(max(n, 0), a.top_k);
  }
  if (e >= n) return;
  const int c = a.idx[row * a.top_k + e];
  const int prev = e > 0 ? a.idx[row * a.top_k + e - 1] : -1;
  if (c < 0 || c >= a.NB || c <= prev ||
      (a.causal && static_cast<int64_t>(c + 1) * a.Bk > static_cast<int64_t>(qb) * a.Bq)) {
    record_error(kErrCheck, kSiteBwd);
    return;
  }
  const int kt = static_cast<int>(static_cast<int64_t>(c) * a.Bk / kBkKT);
  const int qc0 = static_cast<int>(static_cast<int64_t>(qb) * a.Bq / kBkQC);
  const int nqc = a.Bq > kBkQC ? a.Bq / kBkQC : 1;
  uint32_t* m = ba.map_w + ((row / a.NQB) * ba.n_ktiles + kt) * ba.map_words;
  for (int q = qc0; q < qc0 + nqc; ++q) atomicOr(&m[q >> 5], 1u << (q & 31));
}

// ===========================================================================
// key-major kernel: dk, dv
// ===========================================================================
template <int D>
struct DkvLayout {
  static constexpr int STG = 4;                       // visit stages
  static constexpr int NSW = 8;                       // softmax warps (2 per TMEM lane quarter)
  static constexpr int THREADS = (NSW + 2) * 32;      // + producer warp + MMA warp
  static constexpr uint32_t HALF_K = kBkKT * 128;     // one 64-column half of the K tile
  static constexpr uint32_t K_BYTES = kBkKT * D * 2;
  static constexpr uint32_t HALF_Q = kBkQC * 128;     // one 64-column half of a Q chunk
  static constexpr uint32_t Q_BYTES = kBkQC * D * 2;
  // a stage: Q chunk | G chunk | lse * log2(e) (64 f32) | delta (64 f32) | descriptor
  static constexpr uint32_t ST_Q = 0, ST_G = Q_BYTES, ST_LSE = 2 * Q_BYTES;
  static constexpr uint32_t ST_DEL = ST_LSE + kBkQC * 4, ST_DESC = ST_DEL + kBkQC * 4;
  static constexpr uint32_t STAGE_BYTES = (ST_DESC + 16 + 1023) / 1024 * 1024;
  static constexpr uint32_t OFF_K = 0, OFF_V = K_BYTES, OFF_ST = 2 * K_BYTES;
  // kv | full[STG] | empty[STG] | sd_full[2] | p_full[2] | pd_done[2] | drain
  static constexpr int NBAR = 1 + 2 * STG + 6 + 1;
  static constexpr uint32_t OFF_BAR = OFF_ST + STG * STAGE_BYTES;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t USED = OFF_MISC + 64;
  // one CTA per SM: it holds all 512 TMEM columns
  static constexpr uint32_t MIN_REQ = 120 * 1024;
  static constexpr uint32_t SMEM_BYTES = (USED + 1024 > MIN_REQ) ? USED + 1024 : MIN_REQ;
  // TMEM: two S^T buffers (P^T over them), two dP^T buffers (dS^T over them), dk, dv
  static constexpr uint32_t TM_S0 = 0, TM_DP0 = 128, TM_DK = 256, TM_DV = 256 + D;
  static constexpr uint32_t COLS = 512;
  static_assert(TM_DV + D <= COLS, "TMEM budget");
};

struct DkvDesc {
  int32_t h;        // query head
  int32_t qc;       // query chunk (queries qc*64 .. qc*64 + 63)
  uint32_t routed;  // bit lq*8 + cl: query block lq of the chunk routes key block cl of the tile
  int32_t end;      // 1: no more visits
};

// 4 consecutive floats of shared memory
__device__ __forceinline__ float4 lds_f4(uint32_t saddr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(saddr));
  return v;
}

template <int D>
__global__ void __launch_bounds__(DkvLayout<D>::THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tg,
                    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const BwdTcArgs ba) {
  using L = DkvLayout<D>;
  constexpr int STG = L::STG, NSW = L::NSW;
  const AttendArgs& a = ba.at;
  extern __shared__ uint8_t kv_smem_raw[];
  // 1024-byte aligned start, as an offset into the shared array (not through an
  // integer cast, which would drop the shared address space from every pointer
  // derived from it and turn their loads into generic ones)
  uint8_t* smem = kv_smem_raw + ((1024u - (smem_u32(kv_smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_full = bars + 1;
  uint64_t* bar_empty = bars + 1 + STG;
  uint64_t* bar_sd_full = bars + 1 + 2 * STG;   // [2]
  uint64_t* bar_p_full = bar_sd_full + 2;        // [2]
  uint64_t* bar_pd_done = bar_p_full + 2;        // [2]
  uint64_t* bar_drain = bar_pd_done + 2;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[3]);
  auto stage = [&](int st) { return smem + L::OFF_ST + st * L::STAGE_BYTES; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // one CTA per (128-key tile, query head); all heads of tile 0 first (the
  // early tiles are read by the most query blocks)
  const int n_bh = a.Hq * ba.B;
  const int kt = blockIdx.x / n_bh;
  const int bh = blockIdx.x % n_bh;              // b * Hq + query head
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int grp = a.Hq / a.Hkv;
  const int kvh = h / grp;
  const int bk = b * a.Hkv + kvh;                // b * Hkv + KV head
  const int j0 = kt * kBkKT;
  const int nqc = (a.N + kBkQC - 1) / kBkQC;

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < STG; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_sd_full[s], 1);
      mbar_init(&bar_p_full[s], NSW);   // one arrival per softmax warp
      mbar_init(&bar_pd_done[s], 1);
    }
    mbar_init(bar_drain, 1);
    misc[3] = 0;
    fence_barrier_init();
  }
  if (warp == NSW + 1) {
    tmem_alloc(&misc[0], L::COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  int produced = 0;   // visits put in flight (producer lane 0)

  if (warp == NSW) {
    // ------------------------------------------------------- visit producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tg);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      mbar_arrive_expect_tx(bar_kv, 2 * L::K_BYTES);
#pragma unroll
      for (int half = 0; half < D / 64; ++half) {
        tma_load_3d(smem + L::OFF_K + half * L::HALF_K, &tk, bar_kv, half * 64, j0, bk);
        tma_load_3d(smem + L::OFF_V + half * L::HALF_K, &tv, bar_kv, half * 64, j0, bk);
      }
    }
    // window chunks: queries i with i - W < j <= i for a key j of the tile
    int wq0 = 1, wq1 = 0;
    if (a.causal) {
      wq0 = j0 / kBkQC;
      wq1 = min(nqc - 1, (j0 + kBkKT - 2 + a.window) / kBkQC);
    }
    const int c_first = j0 / a.Bk;
    const int nkb = a.Bk < kBkKT ? kBkKT / a.Bk : 1;        // key blocks in the tile
    const int qpc = a.Bq < kBkQC ? kBkQC / a.Bq : 1;         // query blocks in a chunk
    const int lh = a.idx_heads == a.Hq ? h : kvh;
    const int64_t lrow0 = static_cast<int64_t>(b) * a.idx_heads + lh;   // list row block
    const uint32_t* mrow = ba.map + (lrow0 * ba.n_ktiles + kt) * ba.map_words;
    bool live = true;
    int v = 0;        // visits issued so far (uniform across the warp)
    int nb = 0;       // visits collected in the current batch
    int my_qc = 0;    // lane l holds the batch's l-th visit
    // Issue the collected batch: every lane first reads the lists of its own
    // visit (which query block of the chunk routes which key block of the
    // tile), so a batch costs one round of list loads; then lane 0 puts the
    // visits in flight in order.
    auto flush = [&]() {
      uint32_t routed = 0u;
      if (lane < nb && a.top_k > 0) {
        const int qbf = static_cast<int>(static_cast<int64_t>(my_qc) * kBkQC / a.Bq);
        for (int lq = 0; lq < qpc; ++lq) {
          const int qb = qbf + lq;
          if (qb >= a.NQB) break;
          const int64_t row = lrow0 * a.NQB + qb;
          const int n = min(max(a.cnt[row], 0), a.top_k);
          const int32_t* lst = a.idx + row * a.top_k;
#pragma unroll 4
          for (int e = 0; e < n; ++e) {
            const int c = lst[e] - c_first;
            if (c >= 0 && c < nkb) routed |= 1u << (lq * 8 + c);
          }
        }
      }
      for (int u = 0; u < nb && live; ++u) {
        const int qc = __shfl_sync(0xffffffffu, my_qc, u);
        const uint32_t rb = __shfl_sync(0xffffffffu, routed, u);
        if (lane == 0) {
          const int st = v % STG;
          if (v >= STG && !mbar_wait(&bar_empty[st], ((v / STG) - 1) & 1, a.timeout_ns,
                                     abort_flag, kSiteKvEmpty)) {
            live = false;
          } else {
            uint8_t* sp = stage(st);
            DkvDesc* dsc = reinterpret_cast<DkvDesc*>(sp + L::ST_DESC);
            dsc->h = h;
            dsc->qc = qc;
            dsc->routed = rb;
            dsc->end = 0;
            const int i0 = qc * kBkQC;
            const uint32_t vb = static_cast<uint32_t>(min(kBkQC, a.N - i0)) * 4u;
            mbar_arrive_expect_tx(&bar_full[st], 2 * L::Q_BYTES + 2 * vb);
#pragma unroll
            for (int half = 0; half < D / 64; ++half) {
              tma_load_3d(sp + L::ST_Q + half * L::HALF_Q, &tq, &bar_full[st], half * 64, i0, bh);
              tma_load_3d(sp + L::ST_G + half * L::HALF_Q, &tg, &bar_full[st], half * 64, i0, bh);
            }
            bulk_load(sp + L::ST_LSE, ba.lse2 + static_cast<int64_t>(bh) * a.N + i0, vb,
                      &bar_full[st]);
            bulk_load(sp + L::ST_DEL, ba.delta + static_cast<int64_t>(bh) * a.N + i0, vb,
                      &bar_full[st]);
            ++produced;
          }
        }
        live = __shfl_sync(0xffffffffu, live, 0);
        ++v;
      }
      nb = 0;
    };
    for (int w0 = 0; w0 < ba.map_words && live; w0 += 32) {
      const int w = w0 + lane;
      uint32_t word = 0u;
      if (w < ba.map_words) {
        word = a.top_k > 0 ? mrow[w] : 0u;
        const int lo = max(wq0, 32 * w), hi = min(wq1, 32 * w + 31);
        if (lo <= hi) word |= static_cast<uint32_t>(bit_range(lo - 32 * w, hi - 32 * w + 1));
      }
      uint32_t nz = __ballot_sync(0xffffffffu, word != 0u);
      while (nz != 0u && live) {
        const int src = __ffs(nz) - 1;
        nz &= nz - 1u;
        uint32_t bits = __shfl_sync(0xffffffffu, word, src);
        while (bits != 0u && live) {
          // lanes nb .. nb + take - 1 take the word's lowest `take` chunks
          const int take = min(__popc(bits), 32 - nb);
          if (lane >= nb && lane < nb + take)
            my_qc = (w0 + src) * 32 + static_cast<int>(__fns(bits, 0, lane - nb + 1));
          const int last = static_cast<int>(__fns(bits, 0, take));
          bits = (last >= 31) ? 0u : (bits & ~((2u << last) - 1u));
          nb += take;
          if (nb == 32) flush();
        }
      }
    }
    if (live && nb > 0) flush();
    // end marker
    if (lane == 0 && live) {
      const int st = v % STG;
      if (v < STG || mbar_wait(&bar_empty[st], ((v / STG) - 1) & 1, a.timeout_ns, abort_flag,
                               kSiteKvEmpty)) {
        reinterpret_cast<DkvDesc*>(stage(st) + L::ST_DESC)->end = 1;
        mbar_arrive(&bar_full[st]);
      }
    }
  } else if (warp == NSW + 1) {
    // ------------------------------------------------------- MMA issuer
    // Event-driven, two visits in flight: the products of visit v (S^T, dP^T
    // into buffer v % 2) go out once its chunk has landed and visit v - 2's
    // dv / dk products (which read that buffer) are done; visit u's dv / dk
    // products go out once its P^T / dS^T are written.  The loop gives up
    // after timeout_ns without progress.
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(kBkKT, kBkQC, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(kBkKT, D, false, true);
      bool ok = mbar_wait(bar_kv, 0, a.timeout_ns, abort_flag, kSiteQFull);
      int n1 = 0, n2 = 0;      // visits whose first / second products are issued
      bool ended = false;
      uint64_t t_last = globaltimer_ns();
      while (ok && (!ended || n2 < n1)) {
        bool progress = false;
        if (!ended && n1 < n2 + 2) {
          const int st = n1 % STG;
          bool ready = mbar_test(&bar_full[st], (n1 / STG) & 1);
          if (ready && reinterpret_cast<const DkvDesc*>(stage(st) + L::ST_DESC)->end) {
            ended = true;
            ready = false;
            progress = true;
          }
          if (ready && n1 >= 2) ready = mbar_test(&bar_pd_done[n1 & 1], ((n1 - 2) >> 1) & 1);
          if (ready) {
            tc_fence_after();
            const uint32_t qs = smem_u32(stage(st) + L::ST_Q), gs = smem_u32(stage(st) + L::ST_G);
            const uint32_t buf = static_cast<uint32_t>(n1 & 1) * 64;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_k = (kk / 4) * L::HALF_K + (kk % 4) * 32;
              const uint32_t off_q = (kk / 4) * L::HALF_Q + (kk % 4) * 32;
              mma_ss(tmem + L::TM_S0 + buf, sdesc_sw128(sbase + L::OFF_K + off_k, 16, 1024),
                     sdesc_sw128(qs + off_q, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_k = (kk / 4) * L::HALF_K + (kk % 4) * 32;
              const uint32_t off_q = (kk / 4) * L::HALF_Q + (kk % 4) * 32;
              mma_ss(tmem + L::TM_DP0 + buf, sdesc_sw128(sbase + L::OFF_V + off_k, 16, 1024),
                     sdesc_sw128(gs + off_q, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar_sd_full[n1 & 1]);
            ++n1;
            progress = true;
          }
        }
        if (n2 < n1 && mbar_test(&bar_p_full[n2 & 1], (n2 >> 1) & 1)) {
          tc_fence_after();
          const int st = n2 % STG;
          const uint32_t qs = smem_u32(stage(st) + L::ST_Q), gs = smem_u32(stage(st) + L::ST_G);
          const uint32_t buf = static_cast<uint32_t>(n2 & 1) * 64;
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int kk = 0; kk < kBkQC / 16; ++kk) {
              const uint32_t acc = (n2 > 0 || kk > 0 || part > 0) ? 1u : 0u;
              mma_ts(tmem + L::TM_DV, tmem + L::TM_S0 + buf + split_col(kk, part == 1),
                     sdesc_sw128(gs + kk * 2048, L::HALF_Q, 1024), IDESC_O, acc);
              mma_ts(tmem + L::TM_DK, tmem + L::TM_DP0 + buf + split_col(kk, part == 1),
                     sdesc_sw128(qs + kk * 2048, L::HALF_Q, 1024), IDESC_O, acc);
            }
          }
          mma_commit(&bar_pd_done[n2 & 1]);
          mma_commit(&bar_empty[st]);
          ++n2;
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
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0, a.timeout_ns, nullptr, kSiteDrain);
    }
  } else {
    // ------------------------------------------------------- softmax warps
    // warp w: keys of TMEM lane quarter w % 4, query columns of half w / 4
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;   // key row in the tile == TMEM lane
    const int j = j0 + r;
    const bool row_ok = j < a.N;
    const int cl = (a.Bk < kBkKT) ? r / a.Bk : 0;           // key block within the tile
    const int bq_c = a.Bq < kBkQC ? a.Bq : kBkQC;           // columns of one query block
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sl2 = a.scale_log2;
    bool ok = true;
    int v = 0;
    for (;; ++v) {
      const int st = v % STG;
      const bool got = mbar_wait(&bar_full[st], (v / STG) & 1, a.timeout_ns, abort_flag,
                                 kSiteKvFull);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      const uint8_t* sp = stage(st);
      const DkvDesc dsc = *reinterpret_cast<const DkvDesc*>(sp + L::ST_DESC);
      if (dsc.end) break;
      const bool got2 = mbar_wait(&bar_sd_full[v & 1], (v >> 1) & 1, a.timeout_ns, abort_flag,
                                  kSiteSFull);
      if (!__all_sync(0xffffffffu, got2)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int i0 = dsc.qc * kBkQC;
      // queries of this warp's half that read this key
      uint32_t m = 0u;
      if (row_ok) {
        uint64_t mm = 0ull;
        const int nq = min(kBkQC, a.N - i0);
#pragma unroll 1
        for (int lq = 0; lq * bq_c < kBkQC; ++lq)
          if ((dsc.routed >> (lq * 8 + cl)) & 1u) mm |= bit_range(lq * bq_c, (lq + 1) * bq_c);
        if (a.causal) mm |= bit_range(max(0, j - i0), min(kBkQC, j + a.window - i0));
        mm &= bit_range(0, nq);
        m = static_cast<uint32_t>(mm >> (32 * half));
      }
      const uint32_t scol = trow + L::TM_S0 + (v & 1) * 64 + half * 32;
      const uint32_t dcol = trow + L::TM_DP0 + (v & 1) * 64 + half * 32;
      if (__all_sync(0xffffffffu, m == 0u)) {
        uint32_t z[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) z[c] = 0u;
        tmem_st16(scol, z);
        tmem_st16(scol + 16, z);
        tmem_st16(dcol, z);
        tmem_st16(dcol + 16, z);
      } else {
        uint32_t sv[32], dv32[32];
        tmem_ld32(scol, sv);
        tmem_ld32(dcol, dv32);
        // the half's lse * log2(e) and delta, 4 at a time
        const uint32_t lsa = smem_u32(sp + L::ST_LSE) + half * 128;
        const uint32_t dla = smem_u32(sp + L::ST_DEL) + half * 128;
        float ls[32], dl[32];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 x = lds_f4(lsa + c4 * 16), y = lds_f4(dla + c4 * 16);
          ls[4 * c4] = x.x; ls[4 * c4 + 1] = x.y; ls[4 * c4 + 2] = x.z; ls[4 * c4 + 3] = x.w;
          dl[4 * c4] = y.x; dl[4 * c4 + 1] = y.y; dl[4 * c4 + 2] = y.z; dl[4 * c4 + 3] = y.w;
        }
        tmem_ld_wait(sv);
        tmem_ld_wait(dv32);
        // P^T and dS^T in place of S^T and dP^T (float bits)
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const bool on = (m >> c) & 1u;
          const float pc = ex2_approx(fmaf(__uint_as_float(sv[c]), sl2, -ls[c]));
          dv32[c] = __float_as_uint(on ? pc * (__uint_as_float(dv32[c]) - dl[c]) : 0.f);
          sv[c] = __float_as_uint(on ? pc : 0.f);
        }
        uint32_t hi[16], lo[16];
        split_pack32_bits(dv32, hi, lo);
        tmem_st16(dcol, hi);
        tmem_st16(dcol + 16, lo);
        split_pack32_bits(sv, hi, lo);
        tmem_st16(scol, hi);
        tmem_st16(scol + 16, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_p_full[v & 1]);
    }

    // ------------------------------------------------------- epilogue
    if (ok && v > 0) {
      const bool got = mbar_wait(&bar_pd_done[(v - 1) & 1], ((v - 1) >> 1) & 1, a.timeout_ns,
                                 abort_flag, kSitePvDone);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok && !*abort_flag) {
      tc_fence_after();
      // one query head per KV head: the gradients themselves; otherwise this
      // head's share, summed over the group by bwd_group_sum_kernel
      const bool direct = grp == 1;
      const int64_t off = (static_cast<int64_t>(direct ? bk : bh) * a.N + j) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        float* dst_row = (which == 0 ? (direct ? ba.dk : ba.part_dk)
                                     : (direct ? ba.dv : ba.part_dv)) + off;
        const float f = which == 0 ? ba.scale : 1.f;
        const uint32_t col = (which == 0 ? L::TM_DK : L::TM_DV) + half * (D / 2);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          uint32_t x[32];
          if (v > 0) {
            tmem_ld32(trow + col + cc * 32, x);
            tmem_ld_wait(x);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] = 0u;
          }
          if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(dst_row + half * (D / 2) + cc * 32);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_float4(__uint_as_float(x[4 * c]) * f, __uint_as_float(x[4 * c + 1]) * f,
                                   __uint_as_float(x[4 * c + 2]) * f,
                                   __uint_as_float(x[4 * c + 3]) * f);
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == NSW && lane == 0) {
    // after an abort, copies in flight must land before the CTA exits; on the
    // normal path every stage and the K/V tile were consumed
    if (*abort_flag) {
      for (int t = max(0, produced - STG); t < produced; ++t)
        mbar_wait(&bar_full[t % STG], (t / STG) & 1, a.timeout_ns, nullptr, kSiteDrain);
      mbar_wait(bar_kv, 0, a.timeout_ns, nullptr, kSiteDrain);
    }
  }
  __syncthreads();
  if (warp == NSW + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::COLS);
  }
}

// delta_i = <g_i, o_i> (fp32, from the bf16 output and gradient) and
// lse_i * log2(e), the exponent offset the key-major kernel reads; one warp
// per row
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdTcArgs ba, int64_t n_rows) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(ba.o + row * D);
  const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(ba.d_o + row * D);
  float s = 0.f;
#pragma unroll
  for (int c = lane; c < D / 2; c += 32) {
    const float2 x = __bfloat1622float2(o2[c]), y = __bfloat1622float2(g2[c]);
    s = fmaf(x.x, y.x, s);
    s = fmaf(x.y, y.y, s);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  if (lane == 0) {
    ba.delta_w[row] = s;
    ba.lse2[row] = ba.lse[row] * 1.4426950408889634f;
  }
}

// dk, dv of a KV head = the sum of its query heads' shares, in ascending
// head order (a fixed order: the result is reproducible bit for bit).  One
// thread per 4 consecutive entries of [B * Hkv, N, D].
template <int D>
__global__ void __launch_bounds__(256) bwd_group_sum_kernel(const BwdTcArgs ba, int64_t n4) {
  const AttendArgs& a = ba.at;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n4) return;
  const int grp = a.Hq / a.Hkv;
  const int64_t per_bk = static_cast<int64_t>(a.N) * (D / 4);   // float4s per (b, KV head)
  const int64_t bk = t / per_bk, rem = t % per_bk;
  const int64_t b = bk / a.Hkv, kvh = bk % a.Hkv;
  const int64_t bh0 = b * a.Hq + kvh * grp;
  const float4* pk = reinterpret_cast<const float4*>(ba.part_dk);
  const float4* pv = reinterpret_cast<const float4*>(ba.part_dv);
  float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
  for (int hh = 0; hh < grp; ++hh) {
    const int64_t src = (bh0 + hh) * per_bk + rem;
    const float4 x = pk[src], y = pv[src];
    sk.x += x.x; sk.y += x.y; sk.z += x.z; sk.w += x.w;
    sv.x += y.x; sv.y += y.y; sv.z += y.z; sv.w += y.w;
  }
  reinterpret_cast<float4*>(ba.dk)[t] = sk;
  reinterpret_cast<float4*>(ba.dv)[t] = sv;
}

}  // namespace ssa
