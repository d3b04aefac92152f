// decode_front.cuh -- router, dispatch and row gather of a small batch (T <= 8 tokens) in one
// launch: one cluster of 8 CTAs.
//
//   1. CTA r computes fp64 partial logits of all 8 tokens x E experts over the h-slice
//      [r*H/8, (r+1)*H/8) (8 warps, each an FMA chain in ascending h over an eighth of the
//      slice, added in warp order), plus partial squared norms, and writes them into CTA 0's
//      shared memory through distributed shared memory (st.shared::cluster);
//   2. cluster barrier; CTA 0 adds the 8 partials in rank order and finishes every token
//      exactly as router_select_kernel does (rank, verify against the rounding bound,
//      sequential exact recomputation when too close, renormalised weights), then runs the
//      single-CTA dispatch (counts, offsets, stable permutation, tile list);
//   3. (only when an Xp buffer is given) cluster barrier; all warps of the cluster copy the
//      x rows into Xp.  By default GEMM-1 gathers the rows itself and this step is skipped.
// The summation depth per logit is H/64 + 7 + 7 + 1 (<= H + 8), inside the bound the
// verification uses.
#pragma once
#include "ptx.cuh"
#include "router.cuh"
#include "dispatch.cuh"

namespace moe {

constexpr int kFrontRanks = 8;
constexpr int kFrontMaxTokens = 8;
constexpr int kFrontWarps = 8;      // one token per warp in the finishing CTA

// Dynamic shared memory (doubles): part [8][8][E] | pxn [8][8] | pwn [8][E] | work region
// max(hs*8, warps*8*E) (x stage, then the cross-warp reduction).
__host__ __device__ inline size_t decode_front_smem_bytes(int H, int E) {
  const size_t hs = (size_t)H / kFrontRanks;
  const size_t red = (size_t)kFrontWarps * 8 * E;
  const size_t work = hs * 8 > red ? hs * 8 : red;
  return sizeof(double) * ((size_t)kFrontRanks * 8 * E + kFrontRanks * 8 + (size_t)kFrontRanks * E + work);
}

template <int EPL>
__global__ void __cluster_dims__(kFrontRanks, 1, 1) __launch_bounds__(32 * kFrontWarps, 1)
    decode_front_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr,
                        const float* __restrict__ bias, int T, int H, int E, int k, int renorm,
                        double beta_scale, int32_t* __restrict__ ids, float* __restrict__ wts,
                        unsigned* __restrict__ stats, int32_t* __restrict__ counts,
                        int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                        int32_t* __restrict__ inv, int32_t* __restrict__ tile_num,
                        int32_t* __restrict__ tile_expert, int32_t* __restrict__ tile_row0,
                        int32_t* __restrict__ tile_rows, int32_t* __restrict__ gemm_counters,
                        int n_counters, int BM, uint4* __restrict__ xp, int nvec) {
  pdl_trigger();
  pdl_wait();
  constexpr int TT = kFrontMaxTokens, NW = kFrontWarps;
  extern __shared__ double fsm[];
  __shared__ int s_cnt[256], s_off[256], s_base[256], s_tstart[256];
  double* part = fsm;                                   // [8][TT][E]   (filled in CTA 0)
  double* pxn = part + kFrontRanks * TT * E;            // [8][TT]
  double* pwn = pxn + kFrontRanks * TT;                 // [8][E]
  double* work = pwn + kFrontRanks * E;                 // x stage / cross-warp reduction
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int hs = H / kFrontRanks, h0 = rank * hs;
  const int nt = T;

  // ---- 1. partial logits over this CTA's h-slice
  // x slice as 16-byte vectors, 4 per thread in flight before any is used.
  {
    const int nv = hs / 8, total = TT * nv;
    for (int b0 = tid; b0 < total; b0 += 4 * blockDim.x) {
      uint4 r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = b0 + u * blockDim.x;
        const int tt = idx / nv, v = idx - tt * nv;
        r[u] = make_uint4(0, 0, 0, 0);
        if (idx < total && tt < nt)
          r[u] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)tt * H + h0) + v);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = b0 + u * blockDim.x;
        if (idx < total) {
          const int tt = idx / nv, v = idx - tt * nv;
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&r[u]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p2[i]);
            work[(8 * v + 2 * i) * TT + tt] = (double)f.x;
            work[(8 * v + 2 * i + 1) * TT + tt] = (double)f.y;
          }
        }
      }
    }
  }
  __syncthreads();
  for (int tt = warp; tt < TT; tt += NW) {
    double s = 0.0;
    for (int hh = lane; hh < hs; hh += 32) {
      const double v = work[hh * TT + tt];
      s = fma(v, v, s);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) st_cluster_f64(mapa_shared(smem_u32(pxn + rank * TT + tt), 0), s);
  }
  const int sub = hs / NW, hb = warp * sub, e0 = lane * EPL;
  const bool active = e0 < E;
  double acc[TT][EPL], wn[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    wn[i] = 0.0;
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t][i] = 0.0;
  }
  if (active) {
    using Vec = typename std::conditional<EPL == 4, uint2, uint4>::type;
    const __nv_bfloat16* wp = wr + (size_t)(h0 + hb) * E + e0;
    for (int hb0 = 0; hb0 < sub; hb0 += 16) {
      Vec raw[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (hb0 + u < sub) raw[u] = *reinterpret_cast<const Vec*>(wp + (size_t)(hb0 + u) * E);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (hb0 + u < sub) {
          double wv[EPL];
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
          for (int i = 0; i < EPL / 2; ++i) {
            wv[2 * i] = (double)__low2float(p[i]);
            wv[2 * i + 1] = (double)__high2float(p[i]);
          }
          const double* xr = work + (hb + hb0 + u) * TT;
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            const double xv = xr[t];
#pragma unroll
            for (int i = 0; i < EPL; ++i) acc[t][i] = fma(xv, wv[i], acc[t][i]);
          }
#pragma unroll
          for (int i = 0; i < EPL; ++i) wn[i] = fma(wv[i], wv[i], wn[i]);
        }
      }
    }
  }
  __syncthreads();                      // x stage dead: reuse it for the warp reduction
  double* red = work;                   // [NW][TT][E]
  if (active) {
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
      for (int i = 0; i < EPL; ++i) red[((size_t)warp * TT + t) * E + e0 + i] = acc[t][i];
  }
  __syncthreads();
  for (int idx = tid; idx < TT * E; idx += blockDim.x) {
    const int t = idx / E, e = idx - t * E;
    double v = red[t * E + e];
#pragma unroll
    for (int w = 1; w < NW; ++w) v += red[((size_t)w * TT + t) * E + e];
    st_cluster_f64(mapa_shared(smem_u32(part + ((size_t)rank * TT + t) * E + e), 0), v);
  }
  __syncthreads();
  if (active) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) red[(size_t)warp * E + e0 + i] = wn[i];
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    double v = red[e];
#pragma unroll
    for (int w = 1; w < NW; ++w) v += red[(size_t)w * E + e];
    st_cluster_f64(mapa_shared(smem_u32(pwn + (size_t)rank * E + e), 0), v);
  }
  cluster_sync();

  // ---- 2. CTA 0: finish every token, then dispatch
  if (rank == 0) {
    if (tid == 0) stats[3] = 0;   // path: fp64 logits
    for (int t = warp; t < nt; t += NW) {
      double xn2 = 0.0;
      for (int r = 0; r < kFrontRanks; ++r) xn2 += pxn[r * TT + t];
      double L[EPL], beta[EPL];
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        L[i] = -DBL_MAX;
        beta[i] = 0.0;
        if (e < E) {
          double v = part[(size_t)t * E + e], wn2 = pwn[e];
          for (int r = 1; r < kFrontRanks; ++r) {
            v += part[((size_t)r * TT + t) * E + e];
            wn2 += pwn[(size_t)r * E + e];
          }
          const double b = bias ? (double)bias[e] : 0.0;
          if (bias) v += b;
          L[i] = v;
          beta[i] = beta_scale * (sqrt(xn2 * wn2) * (1.0 + 1e-6) + fabs(b));
        }
      }
      router_finish_token<EPL>(L, beta, t, x, wr, bias, H, E, k, renorm, ids, wts, stats);
    }
    __threadfence();
    __syncthreads();
    dispatch_small_block(ids, nt * k, E, BM, counts, offsets, perm, inv, tile_num, tile_expert,
                         tile_row0, tile_rows, gemm_counters, n_counters, s_cnt, s_off, s_base,
                         s_tstart);
    __threadfence();
  }
  if (xp == nullptr) return;   // the grouped GEMM gathers the rows itself
  cluster_sync();

  // ---- 3. gather the x rows of the sorted pairs (16-byte vectors, 8 per thread in flight)
  const int P = nt * k;
  const long long total = (long long)P * nvec;
  const int nthr = kFrontRanks * blockDim.x;
  for (long long b0 = rank * blockDim.x + tid; b0 < total; b0 += 8LL * nthr) {
    uint4 r[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const long long idx = b0 + (long long)u * nthr;
      if (idx < total) {
        const int pos = (int)(idx / nvec), v = (int)(idx - (long long)pos * nvec);
        const int t = __ldcg(perm + pos) / k;
        r[u] = __ldg(reinterpret_cast<const uint4*>(x) + (size_t)t * nvec + v);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const long long idx = b0 + (long long)u * nthr;
      if (idx < total) xp[idx] = r[u];
    }
  }
}

}  // namespace moe
