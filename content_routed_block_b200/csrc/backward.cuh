// K5: backward of the read with the selection held fixed.
//
// jonsmirl/ssa README, introduction: within a query's key set the read is
// ordinary softmax attention; the routed lists are a discrete choice and carry
// no gradient.  For query i with key set S_i, P_ij = exp(scale <q_i, k_j> -
// lse_i), upstream gradient g_i:
//   dv_j += P_ij g_i,  dP_ij = <g_i, v_j>,  dS_ij = P_ij (dP_ij - delta_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j += scale dS_ij q_i,
// with delta_i = <g_i, o_i> = sum_j P_ij dP_ij (the forward's output and
// log-sum-exp are reused, so no second pass over the keys is needed).
//
// On the CUDA cores:
//  * bwd_delta_kernel: delta_i = <g_i, o_i> in fp32, one warp per row.
//  * bwd_kernel<D>: one CTA per (b, query head, tile of RT query rows: up to
//    64 for D = 64, 32 for D = 128).  The tile walks the same key set as the
//    forward: the key blocks of its window range (mask j <= i and
//    (j > i - W or the block is routed)), then the routed blocks before that
//    range (every key visible).  Per chunk of CK keys (up to 32 for D = 64,
//    64 for D = 128), K and V are staged in shared memory as fp32, and the
//    five products run as register outer products fed by vector
//    shared-memory loads, each operand kept in the layout its product reads
//    (Q, g and K also transposed):
//      S, dP  (2 rows x 4 keys over D)     -> P and dS in shared memory
//      dq    += dS K  (4 rows x 4 columns, 4 keys per step, registers)
//      dk, dv  = scale dS^T Q, P^T g  (4 keys x TC columns over the rows),
//    and dk, dv go to global fp32 with vector atomic reductions: many query
//    tiles of a KV group read the same key.  For D = 64 the shared memory
//    (113 KB) and registers allow two CTAs per SM.
#pragma once

#include "common.cuh"

namespace ssa {

constexpr int kBwdThreads = 256;

struct BwdArgs {
  const __nv_bfloat16* q;    // [B*Hq, N, D]
  const __nv_bfloat16* k;    // [B*Hkv, N, D]
  const __nv_bfloat16* v;    // [B*Hkv, N, D]
  const __nv_bfloat16* o;    // [B*Hq, N, D] the forward's output
  const __nv_bfloat16* d_o;  // [B*Hq, N, D] upstream gradient
  const float* lse;          // [B*Hq, N] the forward's natural-log LSE
  const int32_t* idx;        // [B*LH, NQB, top_k] the lists the forward read
  const int32_t* cnt;        // [B*LH, NQB]
  float* delta;              // [B*Hq, N] scratch
  float* dq;                 // [B*Hq, N, D] (out)
  float* dk;                 // [B*Hkv, N, D] (out, accumulated: zeroed first)
  float* dv;                 // [B*Hkv, N, D] (out, accumulated: zeroed first)
  int32_t Hq, Hkv, N, Bq, Bk, top_k, window, causal, list_heads, NQB, NB;
  int32_t RT, CK;            // rows per CTA, keys per chunk
  float scale;               // softmax scale
};

template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const BwdArgs a, int64_t n_rows) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(a.o + row * D);
  const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(a.d_o + row * D);
  float s = 0.f;
#pragma unroll
  for (int c = lane; c < D / 2; c += 32) {
    const float2 x = __bfloat1622float2(o2[c]), y = __bfloat1622float2(g2[c]);
    s = fmaf(x.x, y.x, s);
    s = fmaf(x.y, y.y, s);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  if (lane == 0) a.delta[row] = s;
}

// Tile shape per head dimension: rows per CTA, keys per chunk, and the
// column width of the dk/dv micro-tiles, chosen so that every phase has 256
// micro-tiles and (for D = 64) two CTAs fit on an SM.
template <int D>
__host__ __device__ constexpr int bwd_rows() { return D == 64 ? 64 : 32; }
template <int D>
__host__ __device__ constexpr int bwd_keys() { return D == 64 ? 32 : 64; }
template <int D>
__host__ __device__ constexpr int bwd_kcols() { return D == 64 ? 2 : 4; }

// Shared-memory layout (fp32; transposed arrays padded by 4 words per row,
// which keeps float4 alignment):
//   QT, GT [D][RTM+4]   queries / upstream gradients, transposed
//   QR, GR [RTM][D]     the same, row-major
//   KT, VT [D][CKM+4]   the chunk's keys / values, transposed
//   KR     [CKM][D]     the chunk's keys, row-major
//   PM, SM [RTM][CKM+4] P and dS
//   lse, delta [RTM]; the list [64]
template <int D>
struct BwdLayout {
  static constexpr int RTM = bwd_rows<D>();
  static constexpr int CKM = bwd_keys<D>();
  static constexpr int LQ = RTM + 4, LK = CKM + 4;
  static constexpr int QT = 0, GT = QT + D * LQ, QR = GT + D * LQ, GR = QR + RTM * D;
  static constexpr int KT = GR + RTM * D, VT = KT + D * LK, KR = VT + D * LK;
  static constexpr int PM = KR + CKM * D, SM = PM + RTM * LK;
  static constexpr int LSE = SM + RTM * LK, DEL = LSE + RTM, LIST = DEL + RTM;
  static constexpr int TOTAL = LIST + 64;
};

template <int D>
__host__ __device__ constexpr size_t bwd_smem_bytes() {
  return static_cast<size_t>(BwdLayout<D>::TOTAL) * 4;
}

template <int N>
struct BwdVec;
template <>
struct BwdVec<2> {
  using T = float2;
  __device__ static void to(const T& v, float (&a)[2]) { a[0] = v.x; a[1] = v.y; }
  __device__ static T make(const float (&a)[2]) { return make_float2(a[0], a[1]); }
};
template <>
struct BwdVec<4> {
  using T = float4;
  __device__ static void to(const T& v, float (&a)[4]) {
    a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
  }
  __device__ static T make(const float (&a)[4]) { return make_float4(a[0], a[1], a[2], a[3]); }
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, D == 64 ? 2 : 1) bwd_kernel(const BwdArgs a) {
  using L = BwdLayout<D>;
  constexpr int TC = bwd_kcols<D>();   // dk/dv micro-tile columns
  using VC = BwdVec<TC>;
  extern __shared__ __align__(16) float bsm[];
  const int RT = a.RT, CK = a.CK;
  float* QT = bsm + L::QT;
  float* GT = bsm + L::GT;
  float* QR = bsm + L::QR;
  float* GR = bsm + L::GR;
  float* KT = bsm + L::KT;
  float* VT = bsm + L::VT;
  float* KR = bsm + L::KR;
  float* PM = bsm + L::PM;
  float* SM = bsm + L::SM;
  float* lse_s = bsm + L::LSE;
  float* del_s = bsm + L::DEL;
  int* list_s = reinterpret_cast<int*>(bsm + L::LIST);
  constexpr int LQ = L::LQ, LK = L::LK;
  const int tid = threadIdx.x;

  const int64_t bh = blockIdx.y;                    // b * Hq + h
  const int b = static_cast<int>(bh / a.Hq), h = static_cast<int>(bh % a.Hq);
  const int grp = a.Hq / a.Hkv;
  const int64_t bkv = static_cast<int64_t>(b) * a.Hkv + h / grp;
  const int i0 = blockIdx.x * RT;                   // first query row of the tile
  const int qb = i0 / a.Bq;
  const int lh = a.list_heads == a.Hq ? h : h / grp;
  const int64_t lrow = (static_cast<int64_t>(b) * a.list_heads + lh) * a.NQB + qb;
  const float l2e = 1.4426950408889634f;
  const float sl2 = a.scale * l2e;

  // the tile's query rows and upstream gradients (fp32, both layouts)
  const int64_t qoff = (bh * a.N + i0) * D;
  for (int t = tid; t < RT * D / 2; t += kBwdThreads) {
    const float2 x = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.q + qoff)[t]);
    const float2 y = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.d_o + qoff)[t]);
    const int i = (2 * t) / D, d = (2 * t) % D;
    reinterpret_cast<float2*>(QR + i * D + d)[0] = x;
    reinterpret_cast<float2*>(GR + i * D + d)[0] = y;
    QT[d * LQ + i] = x.x;
    QT[(d + 1) * LQ + i] = x.y;
    GT[d * LQ + i] = y.x;
    GT[(d + 1) * LQ + i] = y.y;
  }
  for (int t = tid; t < RT; t += kBwdThreads) {
    lse_s[t] = a.lse[bh * a.N + i0 + t] * l2e;
    del_s[t] = a.delta[bh * a.N + i0 + t];
  }
  // the routed list: count within 0..top_k, blocks admissible and ascending
  int n = a.top_k > 0 ? a.cnt[lrow] : 0;
  if (n < 0 || n > a.top_k) {
    if (tid == 0) record_error(kErrCheck, kSiteBwd);
    n = min(max(n, 0), a.top_k);
  }
  for (int t = tid; t < n; t += kBwdThreads) {
    int c = a.idx[lrow * a.top_k + t];
    const int prev = t > 0 ? a.idx[lrow * a.top_k + t - 1] : -1;
    const bool bad = c < 0 || c >= a.NB || c <= prev ||
                     (a.causal && static_cast<int64_t>(c + 1) * a.Bk > static_cast<int64_t>(qb) * a.Bq);
    if (bad) {
      record_error(kErrCheck, kSiteBwd);
      c = -1;
    }
    list_s[t] = c;
  }
  __syncthreads();

  // dq tile of this thread: rows 4 rq .. +3, columns 4 cq .. +3
  const int n_qtiles = (RT / 4) * (D / 4);
  const bool has_q = tid < n_qtiles;
  const int cq = tid % (D / 4), rq = tid / (D / 4);
  float dq[4][4];
#pragma unroll
  for (int e = 0; e < 4; ++e)
#pragma unroll
    for (int f = 0; f < 4; ++f) dq[e][f] = 0.f;

  // blocks to visit: causal -- the window range [wlo, whi], then routed
  // blocks below wlo; non-causal -- the routed blocks
  const int wlo = a.causal ? max(0, i0 - a.window + 1) / a.Bk : 0;
  const int whi = a.causal ? (i0 + RT - 1) / a.Bk : -1;
  const int n_win = a.causal ? whi - wlo + 1 : 0;
  const int chunks_per_block = a.Bk / CK;
  int below = 0;  // routed blocks below the window range (ascending: a prefix)
  if (a.causal)
    while (below < n && list_s[below] >= 0 && list_s[below] < wlo) ++below;  // uniform
  const int n_visit = a.causal ? n_win + below : n;
  const int n_stiles = (RT / 2) * (CK / 4);       // phase 1: 2 rows x 4 keys
  const int n_ktiles = (CK / 4) * (D / TC);       // phase 2b: 4 keys x TC columns

  for (int vi = 0; vi < n_visit; ++vi) {
    int c;
    bool full;      // every key of the block is in every row's set
    bool routed_c;  // for window-range blocks: is the block routed too
    if (!a.causal) {
      c = list_s[vi];
      full = true;
      routed_c = true;
    } else if (vi < n_win) {
      c = wlo + vi;
      full = false;
      routed_c = false;
      for (int t = below; t < n; ++t) routed_c |= (list_s[t] == c);
    } else {
      c = list_s[vi - n_win];
      full = true;
      routed_c = true;
    }
    if (c < 0) continue;  // a rejected list entry (uniform)
    for (int ch = 0; ch < chunks_per_block; ++ch) {
      const int j0 = c * a.Bk + ch * CK;
      __syncthreads();  // the previous chunk's arrays are no longer read
      const int64_t koff = (bkv * a.N + j0) * D;
      for (int t = tid; t < CK * D / 2; t += kBwdThreads) {
        const float2 x = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.k + koff)[t]);
        const float2 y = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.v + koff)[t]);
        const int jj = (2 * t) / D, d = (2 * t) % D;
        reinterpret_cast<float2*>(KR + jj * D + d)[0] = x;
        KT[d * LK + jj] = x.x;
        KT[(d + 1) * LK + jj] = x.y;
        VT[d * LK + jj] = y.x;
        VT[(d + 1) * LK + jj] = y.y;
      }
      __syncthreads();
      // phase 1: S and dP for rows 2 rs, 2 rs + 1 x keys 4 ks .. +3, then P, dS
      for (int u = tid; u < n_stiles; u += kBwdThreads) {
        const int ks = u % (CK / 4), rs = u / (CK / 4);
        float sv[2][4], dp[2][4];
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int f = 0; f < 4; ++f) sv[e][f] = dp[e][f] = 0.f;
#pragma unroll 4
        for (int d = 0; d < D; ++d) {
          const float2 qx = *reinterpret_cast<const float2*>(QT + d * LQ + 2 * rs);
          const float2 gx = *reinterpret_cast<const float2*>(GT + d * LQ + 2 * rs);
          const float4 kx = *reinterpret_cast<const float4*>(KT + d * LK + 4 * ks);
          const float4 vx = *reinterpret_cast<const float4*>(VT + d * LK + 4 * ks);
          const float qa[2] = {qx.x, qx.y}, ga[2] = {gx.x, gx.y};
          const float ka[4] = {kx.x, kx.y, kx.z, kx.w}, va[4] = {vx.x, vx.y, vx.z, vx.w};
#pragma unroll
          for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              sv[e][f] = fmaf(qa[e], ka[f], sv[e][f]);
              dp[e][f] = fmaf(ga[e], va[f], dp[e][f]);
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 2 * rs + e;
          const int pos = i0 + i;
          float pt[4], st[4];
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            const int j = j0 + 4 * ks + f;
            const bool ok = full || (j <= pos && (j > pos - a.window || routed_c));
            const float p = ok ? exp2f(fmaf(sv[e][f], sl2, -lse_s[i])) : 0.f;
            pt[f] = p;
            st[f] = p * (dp[e][f] - del_s[i]);
          }
          *reinterpret_cast<float4*>(PM + i * LK + 4 * ks) = make_float4(pt[0], pt[1], pt[2], pt[3]);
          *reinterpret_cast<float4*>(SM + i * LK + 4 * ks) = make_float4(st[0], st[1], st[2], st[3]);
        }
      }
      __syncthreads();
      // phase 2a: dq += dS K over the chunk's keys, 4 keys at a time (rows
      // 4 rq.., columns 4 cq..)
      if (has_q) {
#pragma unroll 2
        for (int jj = 0; jj < CK; jj += 4) {
          float sa[4][4], ka[4][4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            BwdVec<4>::to(*reinterpret_cast<const float4*>(SM + (4 * rq + e) * LK + jj), sa[e]);
#pragma unroll
          for (int g = 0; g < 4; ++g)
            BwdVec<4>::to(*reinterpret_cast<const float4*>(KR + (jj + g) * D + 4 * cq), ka[g]);
#pragma unroll
          for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
              for (int f = 0; f < 4; ++f) dq[e][f] = fmaf(sa[e][g], ka[g][f], dq[e][f]);
        }
      }
      // phase 2b: the chunk's dk = scale dS^T Q and dv = P^T g (keys 4 kk..,
      // columns TC ck..), added to global memory with vector atomics
      for (int u = tid; u < n_ktiles; u += kBwdThreads) {
        const int ck = u % (D / TC), kk = u / (D / TC);
        float gk[4][TC], gv[4][TC];
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int f = 0; f < TC; ++f) gk[e][f] = gv[e][f] = 0.f;
#pragma unroll 2
        for (int i = 0; i < RT; ++i) {
          float sa[4], pa[4], qa[TC], ga[TC];
          BwdVec<4>::to(*reinterpret_cast<const float4*>(SM + i * LK + 4 * kk), sa);
          BwdVec<4>::to(*reinterpret_cast<const float4*>(PM + i * LK + 4 * kk), pa);
          VC::to(*reinterpret_cast<const typename VC::T*>(QR + i * D + TC * ck), qa);
          VC::to(*reinterpret_cast<const typename VC::T*>(GR + i * D + TC * ck), ga);
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int f = 0; f < TC; ++f) {
              gk[e][f] = fmaf(sa[e], qa[f], gk[e][f]);
              gv[e][f] = fmaf(pa[e], ga[f], gv[e][f]);
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t off = (bkv * a.N + j0 + 4 * kk + e) * D + TC * ck;
#pragma unroll
          for (int f = 0; f < TC; ++f) gk[e][f] *= a.scale;
          atomicAdd(reinterpret_cast<typename VC::T*>(a.dk + off), VC::make(gk[e]));
          atomicAdd(reinterpret_cast<typename VC::T*>(a.dv + off), VC::make(gv[e]));
        }
      }
    }
  }
  // dq of the tile's rows
  if (has_q) {
#pragma unroll
    for (int e = 0; e < 4; ++e)
      *reinterpret_cast<float4*>(a.dq + (bh * a.N + i0 + 4 * rq + e) * D + 4 * cq) =
          make_float4(dq[e][0] * a.scale, dq[e][1] * a.scale, dq[e][2] * a.scale,
                      dq[e][3] * a.scale);
  }
}

}  // namespace ssa
