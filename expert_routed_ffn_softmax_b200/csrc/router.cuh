// router.cuh -- the MoE router: logits x.W_router, softmax, top-k with ties to the lower
// expert id, renormalised weights (the fused "gating top-k softmax" router op of the
// cann-recipes-infer Gemma-4-26B-A4B optimisation report, §5 阶段3 融合算子; 128 experts,
// top-8 on a 2816 hidden, §1 模型概况).
//
// Exactness.  The ranking must agree bit for bit with a double-precision sum of the exact
// bf16 products taken in ascending h.  Two kernels do it:
//   1. router_partial_kernel: every (token, expert) logit in fp64, the H axis split over
//      `ks` CTAs and 4 warps (each bf16 x bf16 product is exact in fp64; each thread sums
//      its slice in ascending h with FMA), plus squared norms of x rows and W columns;
//   2. router_select_kernel: one warp per token adds the ks partials in a fixed order,
//      takes the top-k by (value desc, id asc), and checks that every decision it made is
//      separated by more than the rounding error either summation order can have
//      (beta_e = 2*gamma_{H+8} * (|x_t|_2 |w_e|_2 + |b_e|), gamma_n = n u / (1 - n u)).
//      When a decision is closer than that (a near-tie or an exact tie), the warp
//      recomputes every logit of that token sequentially in ascending h -- the same
//      sequence of roundings as the ascending-order definition -- and ranks those.
#pragma once
#include <cfloat>
#include <climits>
#include "ptx.cuh"

namespace moe {

constexpr int kRouterTokens = 8;    // tokens per CTA in router_partial_kernel
constexpr int kRouterWarps = 4;

// Partial logits over the h-slice [ks*hs, (ks+1)*hs) for tokens [tg*8, tg*8+8).
// part_logit [ks][T][E] fp64, part_xn2 [ks][T] fp64, part_wn2 [ks][E] fp64 (only the
// CTAs of token group 0 write part_wn2).  Dynamic smem: max(hs*8, 4*8*E) doubles.
template <int EPL>
__global__ void __launch_bounds__(128) router_partial_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr, int T, int H,
    int E, int hs, double* __restrict__ part_logit, double* __restrict__ part_xn2,
    double* __restrict__ part_wn2) {
  constexpr int TT = kRouterTokens;
  extern __shared__ double rsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * TT, ks = blockIdx.y, h0 = ks * hs;
  const int nt = min(TT, T - t0);

  // Stage x[t0:t0+TT, h0:h0+hs] as double, layout [h][t]; missing tokens are zero.
  for (int i = tid; i < hs * TT; i += blockDim.x) {
    const int tt = i / hs, hh = i - tt * hs;
    double v = 0.0;
    if (tt < nt) v = (double)__bfloat162float(x[(size_t)(t0 + tt) * H + h0 + hh]);
    rsm[hh * TT + tt] = v;
  }
  __syncthreads();

  // Squared norm of each token's slice (exact squares; fp64 sums).
  if (warp < nt) {
    double s = 0.0;
    for (int hh = lane; hh < hs; hh += 32) {
      const double v = rsm[hh * TT + warp];
      s = fma(v, v, s);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) part_xn2[(size_t)ks * T + t0 + warp] = s;
  }
  for (int tt = kRouterWarps + warp; tt < nt; tt += kRouterWarps) {
    double s = 0.0;
    for (int hh = lane; hh < hs; hh += 32) {
      const double v = rsm[hh * TT + tt];
      s = fma(v, v, s);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) part_xn2[(size_t)ks * T + t0 + tt] = s;
  }

  // Main loop: lane owns experts [lane*EPL, lane*EPL+EPL); warp owns h-sub-slice.
  const int sub = hs / kRouterWarps;
  const int hb = warp * sub;
  const int e0 = lane * EPL;
  const bool active = e0 < E;
  double acc[TT][EPL];
  double wn[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    wn[i] = 0.0;
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t][i] = 0.0;
  }
  if (active) {
    const __nv_bfloat16* wp = wr + (size_t)(h0 + hb) * E + e0;
#pragma unroll 2
    for (int h = 0; h < sub; ++h, wp += E) {
      double wv[EPL];
      if constexpr (EPL == 4) {
        const uint2 raw = *reinterpret_cast<const uint2*>(wp);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        wv[0] = (double)__low2float(a);
        wv[1] = (double)__high2float(a);
        wv[2] = (double)__low2float(b);
        wv[3] = (double)__high2float(b);
      } else {
        const uint4 raw = *reinterpret_cast<const uint4*>(wp);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < EPL / 2; ++i) {
          wv[2 * i] = (double)__low2float(p[i]);
          wv[2 * i + 1] = (double)__high2float(p[i]);
        }
      }
      const double* xr = rsm + (hb + h) * TT;
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
  __syncthreads();  // x stage no longer needed: reuse smem for the cross-warp reduction

  // red[warp][t][e]
  double* red = rsm;
  if (active) {
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
      for (int i = 0; i < EPL; ++i) red[((size_t)warp * TT + t) * E + e0 + i] = acc[t][i];
  }
  __syncthreads();
  for (int idx = tid; idx < TT * E; idx += blockDim.x) {
    const int t = idx / E, e = idx - t * E;
    if (t < nt) {
      double v = red[(0 * TT + t) * E + e];
#pragma unroll
      for (int w = 1; w < kRouterWarps; ++w) v += red[((size_t)w * TT + t) * E + e];
      part_logit[((size_t)ks * T + t0 + t) * E + e] = v;
    }
  }
  if (blockIdx.x == 0) {
    __syncthreads();
    if (active) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) red[(size_t)warp * E + e0 + i] = wn[i];
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
      double v = red[e];
#pragma unroll
      for (int w = 1; w < kRouterWarps; ++w) v += red[(size_t)w * E + e];
      part_wn2[(size_t)ks * E + e] = v;
    }
  }
}

// (value desc, id asc) order: does (va, ea) come before (vb, eb)?
__device__ __forceinline__ bool rank_before(double va, int ea, double vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

// k rounds of a warp-wide argmax.  Lane owns experts lane + 32*i.  On return every lane
// holds the selected ids/values in slot order; `taken` marks the lane's own selections.
template <int EPL>
__device__ __forceinline__ void warp_topk(const double (&L)[EPL], int E, int k, bool (&taken)[EPL],
                                          int (&sel_e)[8], double (&sel_v)[8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < EPL; ++i) taken[i] = false;
  for (int r = 0; r < k; ++r) {
    double bv = -DBL_MAX;
    int be = INT_MAX;
    bool have = false;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !taken[i] && (!have || rank_before(L[i], e, bv, be))) {
        bv = L[i];
        be = e;
        have = true;
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (rank_before(ov, oe, bv, be)) {
        bv = ov;
        be = oe;
      }
    }
    sel_e[r] = be;
    sel_v[r] = bv;
    if ((be & 31) == lane) {
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (i == (be >> 5)) taken[i] = true;
    }
  }
}

// One warp per token.  Finishes the logits, selects, verifies, computes the weights.
template <int EPL>
__global__ void __launch_bounds__(256) router_select_kernel(
    const double* __restrict__ part_logit, const double* __restrict__ part_xn2,
    const double* __restrict__ part_wn2, int ks, const float* __restrict__ bias,
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr, int T, int H,
    int E, int k, int renorm, double beta_scale, int32_t* __restrict__ ids,
    float* __restrict__ wts, unsigned* __restrict__ n_exact) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T;
       t += gridDim.x * warps_per_block) {
    // Partials are added in ascending split order.  The loads of 8 splits are issued
    // before their adds so that the latency of a long split list is paid once per 8.
    double L[EPL], beta[EPL];
    double xn2 = 0.0;
    for (int s0 = 0; s0 < ks; s0 += 8) {
      double p[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) p[u] = (s0 + u < ks) ? part_xn2[(size_t)(s0 + u) * T + t] : 0.0;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (s0 + u < ks) xn2 += p[u];
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      L[i] = -DBL_MAX;
      beta[i] = 0.0;
      if (e < E) {
        double v = 0.0, wn2 = 0.0;
        for (int s0 = 0; s0 < ks; s0 += 8) {
          double p[8], q[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const bool in = s0 + u < ks;
            p[u] = in ? part_logit[((size_t)(s0 + u) * T + t) * E + e] : 0.0;
            q[u] = in ? part_wn2[(size_t)(s0 + u) * E + e] : 0.0;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (s0 + u < ks) {
              v = (s0 + u == 0) ? p[u] : v + p[u];
              wn2 += q[u];
            }
        }
        const double b = bias ? (double)bias[e] : 0.0;
        if (bias) v += b;
        L[i] = v;
        beta[i] = beta_scale * (sqrt(xn2 * wn2) * (1.0 + 1e-6) + fabs(b));
      }
    }
    bool taken[EPL];
    int sel_e[8];
    double sel_v[8];
    warp_topk<EPL>(L, E, k, taken, sel_e, sel_v);

    // Verify every decision against the rounding bound.
    double sel_b[8];
    for (int r = 0; r < k; ++r) {
      const int owner = sel_e[r] & 31, slot = sel_e[r] >> 5;
      double mine = 0.0;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (i == slot) mine = beta[i];
      sel_b[r] = __shfl_sync(0xffffffffu, mine, owner);
    }
    bool ok = true;
    for (int r = 0; r + 1 < k; ++r) ok = ok && (sel_v[r] - sel_v[r + 1] > sel_b[r] + sel_b[r + 1]);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !taken[i]) ok = ok && (sel_v[k - 1] - L[i] > sel_b[k - 1] + beta[i]);
    }
    ok = __all_sync(0xffffffffu, ok);

    if (!ok) {
      // Too close to call: redo every logit of this token in ascending h (one FMA chain
      // per expert, the product being exact), then rank those values.
      if (lane == 0) atomicAdd(n_exact, 1u);
      double acc[EPL];
#pragma unroll
      for (int i = 0; i < EPL; ++i) acc[i] = 0.0;
      const __nv_bfloat16* xr = x + (size_t)t * H;
      for (int h = 0; h < H; ++h) {
        const double xv = (double)__bfloat162float(xr[h]);
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          if (e < E) acc[i] = fma(xv, (double)__bfloat162float(wr[(size_t)h * E + e]), acc[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) L[i] = bias ? acc[i] + (double)bias[e] : acc[i];
      }
      warp_topk<EPL>(L, E, k, taken, sel_e, sel_v);
    }

    // Weights: softmax over all E, renormalised over the k selected (or not).
    const double m = sel_v[0];
    double denom = 0.0;
    if (renorm) {
      for (int r = 0; r < k; ++r) denom += exp(sel_v[r] - m);
    } else {
      double s = 0.0;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i < E) s += exp(L[i] - m);
#pragma unroll
      for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      denom = s;
    }
    for (int r = 0; r < k; ++r) {
      if (lane == r) {
        ids[(size_t)t * k + r] = sel_e[r];
        wts[(size_t)t * k + r] = (float)(exp(sel_v[r] - m) / denom);
      }
    }
  }
}

}  // namespace moe
