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
// Large batches take the screen path at the end of this file instead: a tensor-core screen
// picks each token's candidates, whose logits are recomputed first as fp32 pair sums of
// the exact products (bounded error, one fp32 -> fp64 conversion per pair), then -- only
// for the candidates of decisions those cannot settle -- in fp64, then, if still too close,
// by the same sequential ascending-h chains.
#pragma once
#include <cfloat>
#include <climits>
#include <type_traits>
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
  pdl_trigger();
  pdl_wait();
  constexpr int TT = kRouterTokens;
  extern __shared__ double rsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * TT, ks = blockIdx.y, h0 = ks * hs;
  const int nt = min(TT, T - t0);

  // Stage x[t0:t0+TT, h0:h0+hs] as double, layout [h][t]; missing tokens are zero.
  // 16-byte vectors, 4 per thread in flight before any is used (hs % 8 == 0).
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
          r[u] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt) * H + h0) + v);
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
            rsm[(8 * v + 2 * i) * TT + tt] = (double)f.x;
            rsm[(8 * v + 2 * i + 1) * TT + tt] = (double)f.y;
          }
        }
      }
    }
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
    // 16 rows of W are loaded before any of them is used, so one memory latency covers 16
    // h-steps; the FMAs still run in ascending h for every accumulator.
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
          const double* xr = rsm + (hb + hb0 + u) * TT;
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

// k rounds of a warp-wide argmax over values V with unique ids (INT_MAX = empty slot).
// On return every lane holds the selected ids/values in slot order; `taken` marks the
// lane's own selected slots.
template <int EPL>
__device__ __forceinline__ void warp_topk_ids(const double (&V)[EPL], const int (&id)[EPL], int k,
                                              bool (&taken)[EPL], int (&sel_e)[8],
                                              double (&sel_v)[8]) {
#pragma unroll
  for (int i = 0; i < EPL; ++i) taken[i] = false;
  for (int r = 0; r < k; ++r) {
    double bv = -DBL_MAX;
    int be = INT_MAX;
    bool have = false;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      if (id[i] != INT_MAX && !taken[i] && (!have || rank_before(V[i], id[i], bv, be))) {
        bv = V[i];
        be = id[i];
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
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (id[i] == be) taken[i] = true;
  }
}

// Experts lane + 32*i (ids >= E are empty).
template <int EPL>
__device__ __forceinline__ void warp_topk(const double (&L)[EPL], int E, int k, bool (&taken)[EPL],
                                          int (&sel_e)[8], double (&sel_v)[8]) {
  const int lane = threadIdx.x & 31;
  int id[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) id[i] = (lane + 32 * i < E) ? lane + 32 * i : INT_MAX;
  warp_topk_ids<EPL>(L, id, k, taken, sel_e, sel_v);
}

// The same selection by rank counting through shared memory: every lane ranks its own
// experts against all E values (broadcast reads of `scratch`), and the expert of rank r < k
// takes slot r.  Ranks are unique because ties go to the lower id.  NaN logits rank below
// every number.  One pass of E comparisons instead of k dependent shuffle reductions.
// scratch: this warp's E + 16 doubles.
template <int EPL>
__device__ __forceinline__ void warp_topk_ranked(const double (&L)[EPL], int E, int k,
                                                 double* scratch, bool (&taken)[EPL],
                                                 int (&sel_e)[8], double (&sel_v)[8]) {
  const int lane = threadIdx.x & 31;
  double* s_sv = scratch + E;
  int* s_se = reinterpret_cast<int*>(s_sv + 8);
  double v[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    v[i] = isnan(L[i]) ? -INFINITY : L[i];
    if (lane + 32 * i < E) scratch[lane + 32 * i] = v[i];
  }
  __syncwarp();
  int rank[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) rank[i] = 0;
  for (int e2 = 0; e2 < E; ++e2) {
    const double v2 = scratch[e2];
#pragma unroll
    for (int i = 0; i < EPL; ++i) rank[i] += rank_before(v2, e2, v[i], lane + 32 * i) ? 1 : 0;
  }
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    taken[i] = lane + 32 * i < E && rank[i] < k;
    if (taken[i]) {
      s_sv[rank[i]] = L[i];
      s_se[rank[i]] = lane + 32 * i;
    }
  }
  __syncwarp();
  for (int r = 0; r < k; ++r) {
    sel_v[r] = s_sv[r];
    sel_e[r] = s_se[r];
  }
  __syncwarp();   // scratch free again
}

// Value held by the lane/slot whose id is `e` (every lane gets it).
template <int EPL>
__device__ __forceinline__ double warp_value_of(const double (&V)[EPL], const int (&id)[EPL], int e) {
  double mine = 0.0;
  bool have = false;
#pragma unroll
  for (int i = 0; i < EPL; ++i)
    if (id[i] == e) {
      mine = V[i];
      have = true;
    }
  const unsigned m = __ballot_sync(0xffffffffu, have);
  return __shfl_sync(0xffffffffu, mine, __ffs(m) - 1);
}

// Given a token's logits L (expert lane + 32 i) and their rounding bounds beta: select the
// top-k by (value desc, id asc), verify every decision against the bounds, recompute the
// token exactly when one is too close to call, then write ids and (renormalised) weights.
// scratch: this warp's E + 16 doubles of shared memory.
template <int EPL>
__device__ __forceinline__ void router_finish_token(
    double (&L)[EPL], const double (&beta)[EPL], int t, const __nv_bfloat16* __restrict__ x,
    const __nv_bfloat16* __restrict__ wr, const float* __restrict__ bias, int H, int E, int k,
    int renorm, int32_t* __restrict__ ids, float* __restrict__ wts,
    unsigned* __restrict__ stats, double* scratch) {
  const int lane = threadIdx.x & 31;
  bool taken[EPL];
  int sel_e[8];
  double sel_v[8];
  warp_topk_ranked<EPL>(L, E, k, scratch, taken, sel_e, sel_v);

  // Verify every decision against the rounding bound.
  int eid[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) eid[i] = (lane + 32 * i < E) ? lane + 32 * i : INT_MAX;
  double sel_b[8];
  for (int r = 0; r < k; ++r) sel_b[r] = warp_value_of<EPL>(beta, eid, sel_e[r]);
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
    if (lane == 0) atomicAdd(&stats[1], 1u);
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
    warp_topk_ranked<EPL>(L, E, k, scratch, taken, sel_e, sel_v);
  }

  // Weights: softmax over all E, renormalised over the k selected (or not).  Lane r < k
  // evaluates slot r's exponential; the denominator is summed in slot (or expert) order.
  const double m = sel_v[0];
  double mine = 0.0;
  for (int r = 0; r < k; ++r)
    if (lane == r) mine = sel_v[r];
  const double ex = lane < k ? exp(mine - m) : 0.0;
  double denom = 0.0;
  if (renorm) {
    for (int r = 0; r < k; ++r) denom += __shfl_sync(0xffffffffu, ex, r);
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
      wts[(size_t)t * k + r] = (float)(ex / denom);
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
    float* __restrict__ wts, unsigned* __restrict__ stats) {
  pdl_trigger();
  pdl_wait();
  if (blockIdx.x == 0 && threadIdx.x == 0) stats[3] = 0;   // path: fp64 logits
  __shared__ double s_topk[8][256 + 16];   // per-warp top-k scratch (blocks of 8 warps)
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T;
       t += gridDim.x * warps_per_block) {
    // Partials are added in ascending split order.  The loads of 4 splits (for every
    // expert of the lane and the norms) are issued before their adds, so a long split list
    // costs one memory latency per 4 splits.
    double L[EPL], beta[EPL], wn2[EPL];
    double xn2 = 0.0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      L[i] = 0.0;
      wn2[i] = 0.0;
    }
    for (int s0 = 0; s0 < ks; s0 += 4) {
      double p[4][EPL], q[4][EPL], xq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = s0 + u < ks;
        xq[u] = in ? part_xn2[(size_t)(s0 + u) * T + t] : 0.0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          const bool ok = in && e < E;
          p[u][i] = ok ? part_logit[((size_t)(s0 + u) * T + t) * E + e] : 0.0;
          q[u][i] = ok ? part_wn2[(size_t)(s0 + u) * E + e] : 0.0;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (s0 + u < ks) {
          xn2 += xq[u];
#pragma unroll
          for (int i = 0; i < EPL; ++i) {
            L[i] = (s0 + u == 0) ? p[u][i] : L[i] + p[u][i];
            wn2[i] += q[u][i];
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      beta[i] = 0.0;
      if (e < E) {
        const double b = bias ? (double)bias[e] : 0.0;
        if (bias) L[i] += b;
        beta[i] = beta_scale * (sqrt(xn2 * wn2[i]) * (1.0 + 1e-6) + fabs(b));
      } else {
        L[i] = -DBL_MAX;
      }
    }
    router_finish_token<EPL>(L, beta, t, x, wr, bias, H, E, k, renorm, ids, wts, stats,
                             s_topk[threadIdx.x >> 5]);
  }
}

// ----------------------------------------------------------------------------- screen
// Large batches: the logits are first screened on the tensor cores (x . Wr in bf16 with
// fp32 accumulation, the grouped GEMM in EPI_F32 mode), then only the experts that can
// still reach the top-k are recomputed in fp64.
//
// Screen error bound.  The tensor cores multiply bf16 pairs exactly and add them into an
// fp32 accumulator, one K = 16 block per instruction; with truncation in the block sum and
// in the accumulation each instruction adds at most ~2^-22 (|acc| + sum|a b|) of error, so
// |screen - L| <= (H/16) * 2^-21 * sum_h |x_h w_h| ~ 2^-15.5 |x| |w| at H = 2816.  The
// kernel uses delta_e = screen_c * |x_t| |w_e| with screen_c = 2^-10 (a 20x margin over that
// model), plus 4 beta_e, and records the largest |screen - L| / (|x| |w|) it sees so the
// tests can check the model with its margin.
//
// Candidates.  tau = min over the screened top-k of (s_e - delta_e): at least k experts have
// L >= tau + 4 beta, so an expert with s_e + delta_e < tau cannot reach the top-k, in exact
// arithmetic or in either fp64 summation order.  The rest are recomputed in fp64 and
// ranked and checked exactly as in router_select_kernel.

// WrT[e][h] = Wr[h][e] (32x32 tiles through shared memory).
__global__ void __launch_bounds__(256) router_transpose_kernel(const __nv_bfloat16* __restrict__ wr,
                                                               int H, int E,
                                                               __nv_bfloat16* __restrict__ wrT) {
  pdl_trigger();
  pdl_wait();
  __shared__ __nv_bfloat16 tile[32][33];
  const int h0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int h = h0 + i, e = e0 + threadIdx.x;
    if (h < H && e < E) tile[i][threadIdx.x] = wr[(size_t)h * E + e];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int e = e0 + i, h = h0 + threadIdx.x;
    if (h < H && e < E) wrT[(size_t)e * H + h] = tile[threadIdx.x][i];
  }
}

// wn[e] >= |W[:, e]|_2: sum_h Wr[h][e]^2 in fp64 (every square exact), one 256-thread block
// per expert over its transposed row, lanes then warps added in a fixed order; then the
// square root, raised by 1e-6 relative to cover its rounding and the sum's.
__global__ void __launch_bounds__(256) router_wnorm_kernel(const __nv_bfloat16* __restrict__ wrT,
                                                           int H, int E, double* __restrict__ wn) {
  pdl_trigger();
  pdl_wait();
  __shared__ double s_part[8];
  const int e = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(wrT + (size_t)e * H);
  double s = 0.0;
  for (int p = threadIdx.x; 2 * p < H; p += 256) {
    const uint32_t w2 = __ldg(row + p);
    const double a = (double)__uint_as_float(w2 << 16), b = (double)__uint_as_float(w2 & 0xffff0000u);
    s = fma(b, b, fma(a, a, s));
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) s_part[warp] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += s_part[w];
    wn[e] = sqrt(t) * (1.0 + 1e-6);
  }
}

constexpr int kScreenWarps = 8;

// Weight accuracy of the pair-sum recheck: its values are kept only when the renormalised
// weights they give are provably within this of the weights of the fp64 logits.  With every
// logit off by at most b, each weight w_r moves by at most w_r (e^{2b} - 1), so
// 2 b max_r w_r bounds the difference to first order (b <= 1e-4 here, the second order is
// below 1e-4 of it); the fp32 store adds at most 2^-24 w_r.
constexpr double kPairWeightErr = 8e-6;

// Order-preserving maps onto unsigned integers (a larger value gets a larger key).
__device__ __forceinline__ uint32_t ord_f32(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float unord_f32(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
// Doubles: -0 is taken as +0 and NaN maps to 1, below every number (0 marks an empty slot).
__device__ __forceinline__ uint64_t ord_f64(double d) {
  if (isnan(d)) return 1ull;
  const uint64_t b = (uint64_t)__double_as_longlong(d == 0.0 ? 0.0 : d);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
__device__ __forceinline__ double unord_f64(uint64_t k) {
  return __longlong_as_double((long long)((k >> 63) ? (k & 0x7fffffffffffffffull) : ~k));
}

// x_lo w_lo + x_hi w_hi for two packed bf16 pairs with ONE fp32 rounding: bf16 x bf16 is
// exact in fp32 (8-bit significands), so the first fused multiply-add (onto +0) is exact
// and the second rounds once.  Error <= 2^-24 |sum| (or <= 2^-150 in the subnormal range).
__device__ __forceinline__ float bf16_pair_dot(uint32_t xw, uint32_t ww) {
  float d;
  asm("{.reg .b16 xl, xh, wl, wh;\n\t.reg .f32 p;\n\t"
      "mov.b32 {xl, xh}, %1;\n\tmov.b32 {wl, wh}, %2;\n\t"
      "fma.rn.f32.bf16 p, xl, wl, 0f00000000;\n\t"
      "fma.rn.f32.bf16 %0, xh, wh, p;\n\t}"
      : "=f"(d)
      : "r"(xw), "r"(ww));
  return d;
}

// Dot products of one token row x with G candidate rows of W^T (wrow[u]), split over the
// warp: lane l owns h = 256 j + 8 l + i (i < 8), read as 16-byte vectors; a fixed xor tree
// adds the lanes in fp64.  Two precisions:
//   PAIRS: each pair (h, h+1) summed with one fp32 rounding (bf16_pair_dot), the pair sums
//     accumulated in fp64.  |result - sum_h x_h w_h| <= 2^-24 sum_h |x_h w_h| + H 2^-150
//     + the fp64 accumulation's error (well inside the fp64 bound beta).
//   !PAIRS: every value converted to fp64, fp64 fused multiply-adds (error inside beta).
// UNR: unroll of the vector loop (a shorter body issues from the instruction cache better
// when many warps share an SM).
template <bool PAIRS, int G, int UNR>
__device__ __forceinline__ void screen_dot(const __nv_bfloat16* __restrict__ xr,
                                           const uint4* (&wrow)[G], int H, double (&acc)[G]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int u = 0; u < G; ++u) acc[u] = 0.0;
  const uint4* xv4 = reinterpret_cast<const uint4*>(xr);
#pragma unroll UNR
  for (int v = lane; 8 * v < H; v += 32) {   // 16-byte vector index within the row
    const uint4 xq = __ldg(xv4 + v);
    uint4 wq[G];
#pragma unroll
    for (int u = 0; u < G; ++u) wq[u] = __ldg(wrow[u] + v);
    const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xq);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const uint32_t ww = reinterpret_cast<const uint32_t*>(&wq[u])[i];
        if constexpr (PAIRS) {
          acc[u] += (double)bf16_pair_dot(xw[i], ww);
        } else {
          acc[u] = fma((double)__uint_as_float(xw[i] << 16), (double)__uint_as_float(ww << 16),
                       acc[u]);
          acc[u] = fma((double)__uint_as_float(xw[i] & 0xffff0000u),
                       (double)__uint_as_float(ww & 0xffff0000u), acc[u]);
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < G; ++u) {
#pragma unroll
    for (int off = 16; off; off >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
  }
}

// Recompute n candidates of this warp's token into val[] (+ bias): slot j is
// sub ? sub[j] : j, its expert cand[slot].  Four rows at a time, two for a tail of <= 2.
template <bool PAIRS, int UNR>
__device__ __forceinline__ void screen_recheck(const __nv_bfloat16* __restrict__ xr,
                                               const __nv_bfloat16* __restrict__ wrT,
                                               const float* __restrict__ bias, int H,
                                               const int* cand, const int* sub, int n,
                                               double* val) {
  const int lane = threadIdx.x & 31;
  __syncwarp();   // every lane is done reading val
  auto slot = [&](int j) { return sub ? sub[j] : j; };
  for (int c0 = 0; c0 < n;) {
    if (n - c0 > 2) {
      const uint4* wrow[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        wrow[u] = reinterpret_cast<const uint4*>(wrT + (size_t)cand[slot(min(c0 + u, n - 1))] * H);
      double acc[4];
      screen_dot<PAIRS, 4, UNR>(xr, wrow, H, acc);
      double v = acc[0];
#pragma unroll
      for (int u = 1; u < 4; ++u)
        if (lane == u) v = acc[u];
      if (lane < 4 && c0 + lane < n) {
        const int c = slot(c0 + lane), e = cand[c];
        val[c] = bias ? v + (double)bias[e] : v;
      }
      c0 += 4;
    } else {
      const uint4* wrow[2];
#pragma unroll
      for (int u = 0; u < 2; ++u)
        wrow[u] = reinterpret_cast<const uint4*>(wrT + (size_t)cand[slot(min(c0 + u, n - 1))] * H);
      double acc[2];
      screen_dot<PAIRS, 2, UNR>(xr, wrow, H, acc);
      const double v = lane == 1 ? acc[1] : acc[0];
      if (lane < 2 && c0 + lane < n) {
        const int c = slot(c0 + lane), e = cand[c];
        val[c] = bias ? v + (double)bias[e] : v;
      }
      c0 += 2;
    }
  }
  __syncwarp();
}

// k rounds of a warp-wide argmax by (value desc, id asc) over the slots (id INT_MAX = empty;
// at least k slots are filled).  Each round takes every lane's best free slot and reduces
// the 64-bit value keys and then the ids with redux.sync.  On return every lane holds the
// selected ids, values and bounds in rank order; `taken` marks the lane's selected slots.
template <int EPL>
__device__ __forceinline__ void warp_rank_select(const double (&V)[EPL], const double (&B)[EPL],
                                                 const int (&id)[EPL], int k,
                                                 bool (&taken)[EPL], int (&sel_e)[8],
                                                 double (&sel_v)[8], double (&sel_b)[8]) {
  uint64_t key[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    taken[i] = false;
    key[i] = id[i] != INT_MAX ? ord_f64(V[i]) : 0ull;
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    sel_e[r] = INT_MAX;
    sel_v[r] = 0.0;
    sel_b[r] = 0.0;
    if (r < k) {
      uint64_t bk = 0;
      int bid = INT_MAX;
      double bb = 0.0;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (!taken[i] && key[i] != 0 && (key[i] > bk || (key[i] == bk && id[i] < bid))) {
          bk = key[i];
          bid = id[i];
          bb = B[i];
        }
      const uint32_t hi = (uint32_t)(bk >> 32), lo = (uint32_t)bk;
      const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
      const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
      const bool top = bk != 0 && hi == mhi && lo == mlo;
      const int wid = __reduce_min_sync(0xffffffffu, top ? bid : INT_MAX);
      const unsigned wl = __ballot_sync(0xffffffffu, top && bid == wid);
      sel_e[r] = wid;
      sel_v[r] = unord_f64(((uint64_t)mhi << 32) | mlo);
      sel_b[r] = __shfl_sync(0xffffffffu, bb, __ffs(wl) - 1);
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (id[i] == wid) taken[i] = true;
    }
  }
}

// Rank the candidates (slot c = lane + 32 i) by their recomputed values and check every
// decision against B_e = beta_e, plus c_extra |x| |w_e| + abs_extra for a slot whose value
// is a pair sum (prec[c] == 0 or prec == nullptr).  Returns true when all of them hold;
// V, cid, taken, sel_* describe the ranking either way, b_max = max selected B, and need[i]
// marks the slots of the decisions that failed (and of non-finite values).
template <int EPL>
__device__ __forceinline__ bool screen_rank_verify(const int* cand, const double* val,
                                                   const uint8_t* prec, int nc,
                                                   const double* __restrict__ wn,
                                                   const float* __restrict__ bias, double xn,
                                                   double beta_scale, double c_extra,
                                                   double abs_extra, int k, double (&V)[EPL],
                                                   int (&cid)[EPL], bool (&taken)[EPL],
                                                   bool (&need)[EPL], int (&sel_e)[8],
                                                   double (&sel_v)[8], double& b_max) {
  const int lane = threadIdx.x & 31;
  double B[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int c = lane + 32 * i;
    cid[i] = INT_MAX;
    V[i] = -DBL_MAX;
    B[i] = 0.0;
    need[i] = false;
    if (c < nc) {
      const int e = cand[c];
      cid[i] = e;
      V[i] = val[c];
      need[i] = !isfinite(V[i]);
      const double xw = xn * wn[e];
      B[i] = beta_scale * (xw + (bias ? fabs((double)bias[e]) : 0.0));
      if (!(prec && prec[c])) B[i] += c_extra * xw + abs_extra;
    }
  }
  double sel_b[8];
  warp_rank_select<EPL>(V, B, cid, k, taken, sel_e, sel_v, sel_b);
  b_max = 0.0;
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (r < k) b_max = fmax(b_max, sel_b[r]);
  // adjacent selected pairs that are not separated (bit r: ranks r and r + 1)
  unsigned bad = 0u;
#pragma unroll
  for (int r = 0; r + 1 < 8; ++r)
    if (r + 1 < k && !(sel_v[r] - sel_v[r + 1] > sel_b[r] + sel_b[r + 1])) bad |= 1u << r;
  double v_last = sel_v[0], b_last = sel_b[0];
  int e_last = sel_e[0];
#pragma unroll
  for (int r = 1; r < 8; ++r)
    if (r == k - 1) {
      v_last = sel_v[r];
      b_last = sel_b[r];
      e_last = sel_e[r];
    }
  // unselected candidates not separated from the k-th
  bool bnd = false;
#pragma unroll
  for (int i = 0; i < EPL; ++i)
    if (cid[i] != INT_MAX && !taken[i] && !(v_last - V[i] > b_last + B[i])) {
      need[i] = true;
      bnd = true;
    }
  bnd = __any_sync(0xffffffffu, bnd);
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    if (cid[i] == INT_MAX) continue;
    if (bnd && cid[i] == e_last) need[i] = true;
#pragma unroll
    for (int r = 0; r + 1 < 8; ++r)
      if (((bad >> r) & 1u) && (cid[i] == sel_e[r] || cid[i] == sel_e[r + 1])) need[i] = true;
  }
  bool any = false;
#pragma unroll
  for (int i = 0; i < EPL; ++i) any = any || need[i];
  return !__any_sync(0xffffffffu, any) && isfinite(b_max);
}

// Screen path, one warp per token.  screen: ks <= kMaxScreenSplit fp32 partial-sum slices
// of kstride floats each ([T][E] per slice, added here in fp64 in slice order).
// stats[0] += candidates, stats[1] += exact recomputations,
// stats[2] = max over candidates of |screen - L| / (|x| |w|) (float bits, atomicMax),
// stats[3] = 1 (the screen path), stats[4] += tokens with a candidate recomputed in fp64.
// MINB CTAs per SM: 2 (128 registers) keeps each token's chain of L2 round trips short; 4
// (64 registers, some spills) hides more of them when the batch is many waves deep.  The
// recheck loop is unrolled twice in the first form and not at all in the second (measured
// fastest for each; the arithmetic and its order do not depend on it).
constexpr int kMaxScreenSplit = 8;
template <int EPL, int MINB = 2>
__global__ void __launch_bounds__(256, MINB) router_screen_select_kernel(
    const float* __restrict__ screen, int ks, long long kstride,
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wrT,
    const double* __restrict__ wn, const float* __restrict__ bias, int T, int H, int E, int k,
    double screen_c, double beta_scale, int32_t* __restrict__ ids, float* __restrict__ wts,
    unsigned* __restrict__ stats) {
  constexpr int kUnr = MINB >= 4 ? 1 : 2;
  pdl_trigger();
  pdl_wait();
  if (blockIdx.x == 0 && threadIdx.x == 0) stats[3] = 1;   // path: screen + recheck
  __shared__ int s_cand[kScreenWarps][32 * EPL];
  __shared__ int s_sub[kScreenWarps][32 * EPL];
  __shared__ double s_val[kScreenWarps][32 * EPL];
  __shared__ float s_scr[kScreenWarps][32 * EPL];   // screen sums by expert (statistic)
  __shared__ uint8_t s_prec[kScreenWarps][32 * EPL];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  // bound of the pair sums: 2^-24 sum |x_h w_h| <= 2^-24 |x| |w| (+ 1%), underflow H 2^-150
  const double pair_c = 1.01 * 0x1p-24, pair_abs = (double)H * 0x1p-149;
  int* cand = s_cand[warp];
  int* sub = s_sub[warp];
  double* val = s_val[warp];
  uint8_t* prec = s_prec[warp];
  // statistics are gathered per warp and published once, not per token
  unsigned st_cand = 0, st_exact = 0, st_fp64 = 0;
  float st_err = 0.f;
  for (int t = blockIdx.x * kScreenWarps + warp; t < T; t += gridDim.x * kScreenWarps) {
    const __nv_bfloat16* xr = x + (size_t)t * H;
    // Screen sums first: every partial of every slot in flight at once.
    double sv[EPL];
    {
      float part[kMaxScreenSplit][EPL];
#pragma unroll
      for (int z = 0; z < kMaxScreenSplit; ++z)
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          part[z][i] = (z < ks && lane + 32 * i < E)
                           ? __ldg(screen + z * kstride + (size_t)t * E + lane + 32 * i)
                           : 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        sv[i] = 0.0;
#pragma unroll
        for (int z = 0; z < kMaxScreenSplit; ++z) sv[i] += (double)part[z][i];
      }
    }
    // |x_t| bound: squares of bf16 values are exact in fp32; each lane sums its H/32 of them
    // in fp32 (relative error < (H/32) 2^-24, + H/32 2^-150 for underflow), 16-byte loads
    float q = 0.f;
    {
      const uint4* xv4 = reinterpret_cast<const uint4*>(xr);
#pragma unroll 4
      for (int v = lane; 8 * v < H; v += 32) {
        const uint4 xq = __ldg(xv4 + v);
        q += bf16_pair_dot(xq.x, xq.x) + bf16_pair_dot(xq.y, xq.y) +
             bf16_pair_dot(xq.z, xq.z) + bf16_pair_dot(xq.w, xq.w);
      }
    }
    double xn2 = (double)q;
#pragma unroll
    for (int off = 16; off; off >>= 1) xn2 += __shfl_xor_sync(0xffffffffu, xn2, off);
    xn2 = xn2 * (1.0 + (double)(H / 32 + 2) * 0x1p-23) + (double)H * 0x1p-149;
    if (!isfinite(xn2)) {   // fp32 overflow: the norm again in fp64
      xn2 = 0.0;
      for (int h = lane; h < H; h += 32) {
        const double v = (double)__bfloat162float(xr[h]);
        xn2 = fma(v, v, xn2);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) xn2 += __shfl_xor_sync(0xffffffffu, xn2, off);
    }
    const double xn = sqrt(xn2) * (1.0 + 1e-6);

    // Screened logits S, their bounds D, and a threshold tau below the k-th largest lower
    // bound S - D: tau = min of S - D over k experts of the largest S (any k experts give a
    // valid tau; the largest S make it tight).  An expert with S + D < tau cannot reach the
    // top-k, in exact arithmetic or in either fp64 summation order.
    double S[EPL], D[EPL];
    uint32_t skey[EPL];
    bool finite = true;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      S[i] = -DBL_MAX;
      D[i] = 0.0;
      skey[i] = 0u;
      if (e < E) {
        s_scr[warp][e] = (float)sv[i];
        const double xw = xn * wn[e];
        const double beta = beta_scale * (xw + (bias ? fabs((double)bias[e]) : 0.0));
        if (isfinite(sv[i])) {
          S[i] = bias ? sv[i] + (double)bias[e] : sv[i];
          D[i] = screen_c * xw + 4.0 * beta;
          // 24 high bits of the value, then 255 - e: unique keys, larger S first
          skey[i] = (ord_f32((float)S[i]) & 0xffffff00u) | (uint32_t)(255 - e);
        } else {
          finite = false;
        }
      }
    }
    finite = __all_sync(0xffffffffu, finite);
    double tau = -DBL_MAX;
    if (finite) {
      float lo_min = FLT_MAX;
      bool chosen[EPL];
#pragma unroll
      for (int i = 0; i < EPL; ++i) chosen[i] = false;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r < k) {
          uint32_t m = 0u;
#pragma unroll
          for (int i = 0; i < EPL; ++i)
            if (!chosen[i]) m = max(m, skey[i]);
          const uint32_t w = __reduce_max_sync(0xffffffffu, m);
#pragma unroll
          for (int i = 0; i < EPL; ++i)
            if (w != 0u && skey[i] == w) chosen[i] = true;
        }
      }
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (chosen[i]) lo_min = fminf(lo_min, __double2float_rd(S[i] - D[i]));
      tau = (double)unord_f32(__reduce_min_sync(0xffffffffu, ord_f32(lo_min)));
    }
    // Compact the candidates in ascending expert id.
    int nc = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      const bool c = e < E && (!finite || S[i] + D[i] >= tau);
      const unsigned m = __ballot_sync(0xffffffffu, c);
      if (c) {
        cand[nc + __popc(m & lt)] = e;
        prec[nc + __popc(m & lt)] = 0;
      }
      nc += __popc(m);
    }
    __syncwarp();

    // First recheck: fp32 pair sums.  Kept when every ranking decision clears the pair-sum
    // bound and the weights they give are within kPairWeightErr of the fp64 ones.
    screen_recheck<true, kUnr>(xr, wrT, bias, H, cand, nullptr, nc, val);
    double V[EPL];
    int cid[EPL];
    bool taken[EPL], need[EPL];
    int sel_e[8];
    double sel_v[8];
    double b_max;
    bool ok = screen_rank_verify<EPL>(cand, val, prec, nc, wn, bias, xn, beta_scale, pair_c,
                                      pair_abs, k, V, cid, taken, need, sel_e, sel_v, b_max);
    // this lane's share of the renormalised weights: lane r < k holds exp(L_r - L_0)
    auto lane_weight = [&](double& ev, double& denom, int& my_e) {
      double my_v = sel_v[0];
      my_e = sel_e[0];
#pragma unroll
      for (int r = 1; r < 8; ++r)
        if (lane == r) {
          my_v = sel_v[r];
          my_e = sel_e[r];
        }
      ev = lane < k ? exp(my_v - sel_v[0]) : 0.0;
      denom = ev;
#pragma unroll
      for (int off = 16; off; off >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, off);
    };
    double ev, denom;
    int my_e;
    lane_weight(ev, denom, my_e);
    const bool weights_ok = 2.0 * b_max / denom <= kPairWeightErr;   // 1 / denom: max weight
    if (!ok || !weights_ok) {
      ++st_fp64;
      // Second recheck in fp64: only the slots of the failed decisions when the weights were
      // fine, every candidate otherwise; each recomputed slot then carries the fp64 bound.
      int ns = 0;
      if (weights_ok) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const unsigned m = __ballot_sync(0xffffffffu, need[i]);
          if (need[i]) sub[ns + __popc(m & lt)] = lane + 32 * i;
          ns += __popc(m);
        }
        __syncwarp();
      }
      if (ns > 0 && ns < nc) {
        screen_recheck<false, kUnr>(xr, wrT, bias, H, cand, sub, ns, val);
        for (int j = lane; j < ns; j += 32) prec[sub[j]] = 1;
        __syncwarp();
        ok = screen_rank_verify<EPL>(cand, val, prec, nc, wn, bias, xn, beta_scale, pair_c,
                                     pair_abs, k, V, cid, taken, need, sel_e, sel_v, b_max);
        lane_weight(ev, denom, my_e);
        ok = ok && 2.0 * b_max / denom <= kPairWeightErr;
      } else {
        ok = false;
      }
      if (!ok) {
        screen_recheck<false, kUnr>(xr, wrT, bias, H, cand, nullptr, nc, val);
        ok = screen_rank_verify<EPL>(cand, val, nullptr, nc, wn, bias, xn, beta_scale, 0.0, 0.0,
                                     k, V, cid, taken, need, sel_e, sel_v, b_max);
      }
      if (!ok) {
        // Too close to call: each lane recomputes its candidates as one FMA chain in
        // ascending h (the definition's sequence of roundings), then the warp ranks again.
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          if (cid[i] != INT_MAX) {
            const __nv_bfloat16* wrow = wrT + (size_t)cid[i] * H;
            double a = 0.0;
            for (int h = 0; h < H; ++h)
              a = fma((double)__bfloat162float(xr[h]), (double)__bfloat162float(wrow[h]), a);
            V[i] = bias ? a + (double)bias[cid[i]] : a;
          }
        }
        double Bz[EPL], sel_bz[8];
#pragma unroll
        for (int i = 0; i < EPL; ++i) Bz[i] = 0.0;
        warp_rank_select<EPL>(V, Bz, cid, k, taken, sel_e, sel_v, sel_bz);
        ++st_exact;
      }
      lane_weight(ev, denom, my_e);
    }
    // largest |screen - L| / (|x| |w|) over the candidates, L from the last recheck
    float err = 0.f;
    if (finite) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        if (cid[i] != INT_MAX) {
          const int e = cid[i];
          const double L0 = bias ? V[i] - (double)bias[e] : V[i];
          err = fmaxf(err, (float)(fabs((double)s_scr[warp][e] - L0) / (xn * wn[e])));
        }
      }
    }
    st_cand += (unsigned)nc;
    st_err = fmaxf(st_err, err);   // lanes differ; the warp-wide max is taken below

    // Renormalised weights: softmax over the k selected logits, lane r writes slot r.
    if (lane < k) {
      ids[(size_t)t * k + lane] = my_e;
      wts[(size_t)t * k + lane] = (float)(ev / denom);
    }
    __syncwarp();
  }
  st_err = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(st_err)));
  if (lane == 0 && st_cand) {
    atomicAdd(&stats[0], st_cand);
    if (st_exact) atomicAdd(&stats[1], st_exact);
    if (st_fp64) atomicAdd(&stats[4], st_fp64);
    atomicMax(&stats[2], __float_as_uint(st_err));
  }
}

}  // namespace moe
