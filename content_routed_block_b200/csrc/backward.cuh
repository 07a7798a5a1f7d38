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
// First form, on the CUDA cores:
//  * bwd_delta_kernel: delta_i = <g_i, o_i> in fp32, one warp per row.
//  * bwd_kernel<D>: one CTA per (b, query head, tile of RT = min(Bq, 64)
//    query rows).  The tile walks the same key set as the forward: the key
//    blocks of its window range (mask j <= i and (j > i - W or the block is
//    routed)), then the routed blocks before that range (every key visible).
//    Per chunk of CK = min(Bk, 64) keys, K and V are staged in shared memory
//    (fp32, rows padded by one word), each thread scores 4 rows x 1 key
//    (S and dP over D), writes P and dS to shared memory, then accumulates
//    dq in registers (4 rows x 1 column per task) and the chunk's dk and dv
//    (1 key x 4 columns per task) which it adds to global fp32 with
//    vector (float4) atomic reductions: many query tiles of a KV group read
//    the same key.
#pragma once

#include "common.cuh"

namespace ssa {

constexpr int kBwdThreads = 256;
constexpr int kBwdRows = 64;   // query rows per CTA (at most)
constexpr int kBwdKeys = 64;   // keys per chunk (at most)

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

template <int D>
__host__ __device__ constexpr size_t bwd_smem_bytes() {
  // Q, dO [RT][D]; K, V [CK][D+1]; P, dS [RT][CK+1]; lse, delta [RT]; list
  return static_cast<size_t>(2 * kBwdRows * D + 2 * kBwdKeys * (D + 1) +
                             2 * kBwdRows * (kBwdKeys + 1) + 2 * kBwdRows) * 4 + 64 * 4;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads) bwd_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) float bsm[];
  const int RT = a.RT, CK = a.CK;
  float* Qs = bsm;                          // [RT][D]
  float* Gs = Qs + kBwdRows * D;            // [RT][D]   upstream gradient
  float* Ks = Gs + kBwdRows * D;            // [CK][D+1]
  float* Vs = Ks + kBwdKeys * (D + 1);      // [CK][D+1]
  float* Ps = Vs + kBwdKeys * (D + 1);      // [RT][CK+1]
  float* Ss = Ps + kBwdRows * (kBwdKeys + 1);  // [RT][CK+1] dS
  float* lse_s = Ss + kBwdRows * (kBwdKeys + 1);
  float* del_s = lse_s + kBwdRows;
  int* list_s = reinterpret_cast<int*>(del_s + kBwdRows);  // [top_k <= 64]
  const int tid = threadIdx.x;
  const int PD = D + 1, PK = CK + 1;

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

  // the tile's query rows and upstream gradients (fp32), LSE and delta
  const int64_t qoff = (bh * a.N + i0) * D;
  for (int t = tid; t < RT * D / 2; t += kBwdThreads) {
    const float2 x = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.q + qoff)[t]);
    const float2 y = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.d_o + qoff)[t]);
    Qs[2 * t] = x.x;
    Qs[2 * t + 1] = x.y;
    Gs[2 * t] = y.x;
    Gs[2 * t + 1] = y.y;
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

  // dq accumulators: task u = tid + 256 r covers rows 4 (u / D) .. +3, column u % D
  constexpr int QT = (kBwdRows / 4) * D / kBwdThreads;  // tasks per thread at RT = 64
  float acc[QT][4];
#pragma unroll
  for (int r = 0; r < QT; ++r)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[r][e] = 0.f;

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
      __syncthreads();  // the previous chunk's K, V, P, dS are no longer read
      const int64_t koff = (bkv * a.N + j0) * D;
      for (int t = tid; t < CK * D / 2; t += kBwdThreads) {
        const float2 x = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.k + koff)[t]);
        const float2 y = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.v + koff)[t]);
        const int jj = (2 * t) / D, d = (2 * t) % D;
        Ks[jj * PD + d] = x.x;
        Ks[jj * PD + d + 1] = x.y;
        Vs[jj * PD + d] = y.x;
        Vs[jj * PD + d + 1] = y.y;
      }
      __syncthreads();
      // phase 1: P and dS, 4 rows x 1 key per task
      for (int u = tid; u < (RT / 4) * CK; u += kBwdThreads) {
        const int ig = u / CK, jj = u % CK;
        const int j = j0 + jj;
        float s[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
          const float kx = Ks[jj * PD + d], vx = Vs[jj * PD + d];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            s[e] = fmaf(Qs[(4 * ig + e) * D + d], kx, s[e]);
            dp[e] = fmaf(Gs[(4 * ig + e) * D + d], vx, dp[e]);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * ig + e;
          const int pos = i0 + i;
          const bool ok = full || (j <= pos && (j > pos - a.window || routed_c));
          const float p = ok ? exp2f(fmaf(s[e], sl2, -lse_s[i])) : 0.f;
          Ps[i * PK + jj] = p;
          Ss[i * PK + jj] = p * (dp[e] - del_s[i]);
        }
      }
      __syncthreads();
      // phase 2a: dq += dS K (4 rows x 1 column per task)
#pragma unroll
      for (int r = 0; r < QT; ++r) {
        const int u = tid + kBwdThreads * r;
        if (u < (RT / 4) * D) {
          const int ig = u / D, d = u % D;
          for (int jj = 0; jj < CK; ++jj) {
            const float kx = Ks[jj * PD + d];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[r][e] = fmaf(Ss[(4 * ig + e) * PK + jj], kx, acc[r][e]);
          }
        }
      }
      // phase 2b: the chunk's dk (dS^T Q) and dv (P^T dO), 1 key x 4 columns
      for (int u = tid; u < CK * (D / 4); u += kBwdThreads) {
        const int jj = u / (D / 4), d4 = u % (D / 4);
        float4 gk = make_float4(0.f, 0.f, 0.f, 0.f), gv = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < RT; ++i) {
          const float ds = Ss[i * PK + jj], p = Ps[i * PK + jj];
          const float4 qx = reinterpret_cast<const float4*>(Qs + i * D)[d4];
          const float4 gx = reinterpret_cast<const float4*>(Gs + i * D)[d4];
          gk.x = fmaf(ds, qx.x, gk.x);
          gk.y = fmaf(ds, qx.y, gk.y);
          gk.z = fmaf(ds, qx.z, gk.z);
          gk.w = fmaf(ds, qx.w, gk.w);
          gv.x = fmaf(p, gx.x, gv.x);
          gv.y = fmaf(p, gx.y, gv.y);
          gv.z = fmaf(p, gx.z, gv.z);
          gv.w = fmaf(p, gx.w, gv.w);
        }
        gk.x *= a.scale;
        gk.y *= a.scale;
        gk.z *= a.scale;
        gk.w *= a.scale;
        const int64_t off = (bkv * a.N + j0 + jj) * D + 4 * d4;
        atomicAdd(reinterpret_cast<float4*>(a.dk + off), gk);
        atomicAdd(reinterpret_cast<float4*>(a.dv + off), gv);
      }
    }
  }
  // dq of the tile's rows
#pragma unroll
  for (int r = 0; r < QT; ++r) {
    const int u = tid + kBwdThreads * r;
    if (u < (RT / 4) * D) {
      const int ig = u / D, d = u % D;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        a.dq[(bh * a.N + i0 + 4 * ig + e) * D + d] = acc[r][e] * a.scale;
    }
  }
}

}  // namespace ssa
