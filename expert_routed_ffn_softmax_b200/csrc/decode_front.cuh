// decode_front.cuh -- router and dispatch of a small batch (T <= 8 tokens) in one launch:
// one cluster of 8 CTAs (the role of the fused gating top-k softmax op in the
// cann-recipes-infer "Gemma-4-26B-A4B 模型优化报告", §5 阶段3, plus the per-expert split
// sizes of §6.1, for a decode batch).
//
//   1. CTA r copies its h-slice [r*H/8, (r+1)*H/8) of W_router into shared memory with
//      four bulk copies (one per pair of warps, so a warp starts as soon as its rows land)
//      and stages the x slice as doubles; its 8 warps compute fp64 partial logits of all
//      tokens x E experts (each an FMA chain in ascending h over an eighth of the slice,
//      added in warp order) and partial squared norms; token t's partial row, the norm
//      partials and the token's |x|^2 partial go to CTA t through distributed shared memory;
//   2. cluster barrier; CTA t (t < T) adds the 8 partials in rank order and finishes token t
//      with all its threads (thread e ranks expert e against the others, every decision is
//      verified against the rounding bound; a token too close to call goes to the warp path
//      of router_select_kernel, which recomputes it exactly); its ids also go to CTA 0;
//   3. cluster barrier; CTA 0 runs the dispatch of the T*k <= 64 pairs from shared memory
//      (counts, offsets, stable permutation, tile list); the GEMM counters were zeroed by
//      all CTAs in step 1;
//   4. (only when an Xp buffer is given, for decode tiles) cluster barrier; all warps of
//      the cluster copy the x rows into Xp.  By default GEMM-1 gathers the rows itself.
// The summation depth per logit is H/64 + 7 + 7 + 1 (<= H + 8), inside the bound the
// verification uses.  Every wait is bounded.
#pragma once
#include "ptx.cuh"
#include "router.cuh"
#include "dispatch.cuh"

namespace moe {

constexpr int kFrontRanks = 8;
constexpr int kFrontMaxTokens = 8;
constexpr int kFrontWarps = 8;
constexpr int kFrontChunks = 4;     // bulk copies of the W_router slice (2 warps each)

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Dynamic shared memory layout (bytes from a 16-byte aligned base):
//   W   max(hs*E*2, NW*TT*E*8)   W_router slice (bf16), later the cross-warp reduction
//   XS  hs*TT*8                  x slice as doubles [h][t]
//   PART kFrontRanks*E*8         this CTA's token: partial logits per source rank
//   PWN  kFrontRanks*E*8         |W[:,e]|^2 partials per source rank
//   PXN  kFrontRanks*8           |x_t|^2 partials per source rank
//   TOPK (3E+64)*8               logits, bounds, selection; then the warp path's scratch
//   IDS  64*4                    (CTA 0) ids of every pair
//   OFF  128*4                   (CTA 0) offsets of the experts
//   CNT  128*4                   (CTA 0) pairs per expert
//   BEF  64*4                    (CTA 0) rank of each pair among its expert's pairs
//   BARS kFrontChunks*8
struct FrontSmem {
  size_t w, xs, part, pwn, pxn, topk, ids, off, cnt, bef, bars, total;
};
__host__ __device__ inline FrontSmem decode_front_layout(int H, int E) {
  const size_t hs = (size_t)H / kFrontRanks;
  FrontSmem L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 15) & ~size_t(15);
    return o;
  };
  const size_t wbytes = hs * E * 2, red = (size_t)kFrontWarps * kFrontMaxTokens * E * 8;
  L.w = take(wbytes > red ? wbytes : red);
  L.xs = take(hs * kFrontMaxTokens * 8);
  L.part = take((size_t)kFrontRanks * E * 8);
  L.pwn = take((size_t)kFrontRanks * E * 8);
  L.pxn = take((size_t)kFrontRanks * 8);
  L.topk = take((size_t)(3 * E + 64) * 8);
  L.ids = take(64 * 4);
  L.off = take(128 * 4);
  L.cnt = take(128 * 4);
  L.bef = take(64 * 4);
  L.bars = take(kFrontChunks * 8);
  L.total = off + 16;   // base alignment slack
  return L;
}
__host__ __device__ inline size_t decode_front_smem_bytes(int H, int E) {
  return decode_front_layout(H, E).total;
}

// EPL = 4: experts 4*lane .. 4*lane+3 in the partial-logit loop (E <= 128).
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
  static_assert(EPL == 4, "the partial-logit loop reads 4 experts per lane");
  pdl_trigger();
  constexpr int TT = kFrontMaxTokens, NW = kFrontWarps;
  extern __shared__ uint8_t fsm_raw[];
  uint8_t* fsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fsm_raw) + 15) & ~uintptr_t(15));
  const FrontSmem SL = decode_front_layout(H, E);
  __nv_bfloat16* wsl = reinterpret_cast<__nv_bfloat16*>(fsm + SL.w);
  double* red = reinterpret_cast<double*>(fsm + SL.w);   // after the slice is consumed
  double* xs = reinterpret_cast<double*>(fsm + SL.xs);
  double* part = reinterpret_cast<double*>(fsm + SL.part);
  double* pwn = reinterpret_cast<double*>(fsm + SL.pwn);
  double* pxn = reinterpret_cast<double*>(fsm + SL.pxn);
  double* topk = reinterpret_cast<double*>(fsm + SL.topk);
  int* s_ids = reinterpret_cast<int*>(fsm + SL.ids);
  int* s_off = reinterpret_cast<int*>(fsm + SL.off);
  int* s_cnt = reinterpret_cast<int*>(fsm + SL.cnt);
  int* s_bef = reinterpret_cast<int*>(fsm + SL.bef);
  const uint32_t bars = smem_u32(fsm + SL.bars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int hs = H / kFrontRanks, h0 = rank * hs, nt = T;
  const int crow = hs / kFrontChunks;   // rows per bulk copy

  // ---- 1. W_router slice -> shared memory.  This kernel is launched in plain stream order
  // (not as a dependent launch), so every earlier write to W_router and x is visible.
  if (tid == 0) {
    for (int c = 0; c < kFrontChunks; ++c) mbar_init(bars + 8 * c, 1);
    fence_barrier_init();
    for (int c = 0; c < kFrontChunks; ++c) {
      const uint32_t bytes = (uint32_t)crow * E * 2;
      mbar_arrive_expect_tx(bars + 8 * c, bytes);
      bulk_load(smem_u32(wsl) + c * bytes, wr + (size_t)(h0 + c * crow) * E, bytes, bars + 8 * c);
    }
  }
  pdl_wait();   // (a no-op in plain stream order; kept for a dependent launch)
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
            xs[(8 * v + 2 * i) * TT + tt] = (double)f.x;
            xs[(8 * v + 2 * i + 1) * TT + tt] = (double)f.y;
          }
        }
      }
    }
  }
  // The GEMM counters are zeroed by all CTAs while the W_router copies are in flight (this
  // launch runs in plain stream order: no earlier GEMM is still using them).
  for (int i = rank * blockDim.x + tid; i < n_counters; i += kFrontRanks * blockDim.x)
    gemm_counters[i] = 0;
  __syncthreads();   // also publishes the barrier initialisation
  // |x_t|^2 over the slice -> CTA t
  for (int tt = warp; tt < nt; tt += NW) {
    double s = 0.0;
    for (int hh = lane; hh < hs; hh += 32) {
      const double v = xs[hh * TT + tt];
      s = fma(v, v, s);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) st_cluster_f64(mapa_shared(smem_u32(pxn + rank), tt), s);
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
  // This warp's rows lie in one bulk copy (sub = crow / 2).  If it does not land in time
  // (the error word then says so), the warp skips its rows; every CTA still takes every
  // cluster barrier below, so the cluster ends together.
  const bool landed = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (hb / crow), 0));
  if (active && landed) {
#pragma unroll 4
    for (int r = 0; r < sub; ++r) {
      const uint2 raw = *reinterpret_cast<const uint2*>(wsl + (size_t)(hb + r) * E + e0);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
      double wv[EPL];
#pragma unroll
      for (int i = 0; i < EPL / 2; ++i) {
        wv[2 * i] = (double)__low2float(p[i]);
        wv[2 * i + 1] = (double)__high2float(p[i]);
      }
      const double* xr = xs + (hb + r) * TT;
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
  __syncthreads();   // the slice is consumed: its space becomes the reduction buffer
  if (active) {
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
      for (int i = 0; i < EPL; ++i) red[((size_t)warp * TT + t) * E + e0 + i] = acc[t][i];
  }
  __syncthreads();
  // token t's partial row -> CTA t (warp order), and the |W[:,e]|^2 partials -> every CTA
  for (int idx = tid; idx < nt * E; idx += blockDim.x) {
    const int t = idx / E, e = idx - t * E;
    double v = red[t * E + e];
#pragma unroll
    for (int w = 1; w < NW; ++w) v += red[((size_t)w * TT + t) * E + e];
    st_cluster_f64(mapa_shared(smem_u32(part + (size_t)rank * E + e), t), v);
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
    const uint32_t a = smem_u32(pwn + (size_t)rank * E + e);
    for (int t = 0; t < nt; ++t) st_cluster_f64(mapa_shared(a, t), v);
  }
  cluster_sync();

  // ---- 2. CTA t finishes token t with all its threads: thread e < E owns expert e
  const int t = (int)rank;
  double* sL = topk;                 // [E] logits
  double* sB = topk + E;             // [E] rounding bounds
  double* sSelV = topk + 2 * E;      // [8] selected logits, slot order
  double* sSelB = sSelV + 8;         // [8] their bounds
  int* sSelE = reinterpret_cast<int*>(sSelB + 8);   // [8] selected experts
  if (t < nt) {
    if (t == 0 && tid == 0) stats[3] = 0;   // path: fp64 logits
    if (tid < E) {
      double xn2 = 0.0;
      for (int r = 0; r < kFrontRanks; ++r) xn2 += pxn[r];
      const int e = tid;
      double v = part[e], wn2 = pwn[e];
      for (int r = 1; r < kFrontRanks; ++r) {
        v += part[(size_t)r * E + e];
        wn2 += pwn[(size_t)r * E + e];
      }
      const double b = bias ? (double)bias[e] : 0.0;
      if (bias) v += b;
      sL[e] = v;
      sB[e] = beta_scale * (sqrt(xn2 * wn2) * (1.0 + 1e-6) + fabs(b));
    }
    __syncthreads();
    // rank of expert e by (logit desc, id asc); NaN ranks below every number
    int my_rank = E;
    if (tid < E) {
      const double ve = isnan(sL[tid]) ? -INFINITY : sL[tid];
      int r = 0;
#pragma unroll 8
      for (int e2 = 0; e2 < E; ++e2) {
        const double v2 = sL[e2];
        r += rank_before(isnan(v2) ? -INFINITY : v2, e2, ve, tid) ? 1 : 0;
      }
      my_rank = r;
      if (r < k) {
        sSelE[r] = tid;
        sSelV[r] = sL[tid];
        sSelB[r] = sB[tid];
      }
    }
    __syncthreads();
    // every decision must hold under the rounding bounds (as in router_finish_token)
    bool ok = true;
    if (tid < E && my_rank >= k) ok = sSelV[k - 1] - sL[tid] > sSelB[k - 1] + sB[tid];
    if (tid + 1 < k) ok = ok && (sSelV[tid] - sSelV[tid + 1] > sSelB[tid] + sSelB[tid + 1]);
    ok = __syncthreads_and(ok);
    if (warp == 0) {
      if (!ok) {
        // too close to call: the warp path recomputes the token exactly and writes it
        double L4[4], B4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = lane + 32 * i;
          L4[i] = e < E ? sL[e] : -DBL_MAX;
          B4[i] = e < E ? sB[e] : 0.0;
        }
        router_finish_token<4>(L4, B4, t, x, wr, bias, H, E, k, renorm, ids, wts, stats,
                               topk + 2 * E + 32);
        __syncwarp();
        if (lane < k)
          st_cluster_u32(mapa_shared(smem_u32(s_ids + t * k + lane), 0),
                         (uint32_t)ids[(size_t)t * k + lane]);
      } else {
        // weights exactly as router_finish_token forms them (slot-order denominator)
        const double m = sSelV[0];
        const double ex = lane < k ? exp(sSelV[lane] - m) : 0.0;
        double denom = 0.0;
        if (renorm) {
          for (int r = 0; r < k; ++r) denom += __shfl_sync(0xffffffffu, ex, r);
        } else {
          double sum = 0.0;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (lane + 32 * i < E) sum += exp(sL[lane + 32 * i] - m);
#pragma unroll
          for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
          denom = sum;
        }
        if (lane < k) {
          ids[(size_t)t * k + lane] = sSelE[lane];
          wts[(size_t)t * k + lane] = (float)(ex / denom);
          st_cluster_u32(mapa_shared(smem_u32(s_ids + t * k + lane), 0), (uint32_t)sSelE[lane]);
        }
      }
    }
  }
  cluster_sync();

  // ---- 3. CTA 0: dispatch of the P = T*k <= 64 pairs from shared memory, all threads
  if (rank == 0) {
    const int P = nt * k;
    if (tid < E) {   // pairs of expert tid
      int c = 0;
#pragma unroll 8
      for (int q = 0; q < P; ++q) c += (s_ids[q] == tid);
      s_cnt[tid] = c;
    } else if (tid >= 128 && tid - 128 < P) {   // pair q's rank among its expert's pairs
      const int q = tid - 128, e = s_ids[q];
      int before = 0;
#pragma unroll 8
      for (int q2 = 0; q2 < q; ++q2) before += (s_ids[q2] == e);
      s_bef[q] = before;
      if ((unsigned)e >= (unsigned)E) raise_error(MOE_DEVERR_BAD_INDEX);
    }
    __syncthreads();
    if (warp == 0) {
      // exclusive scans of counts and of tiles; lane owns experts 4*lane .. 4*lane+3
      int c[4], nt4[4], cs = 0, ts = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 4 * lane + i;
        c[i] = e < E ? s_cnt[e] : 0;
        nt4[i] = (c[i] + BM - 1) / BM;
        cs += c[i];
        ts += nt4[i];
      }
      int ci = cs, ti = ts;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, ci, off);
        const int b = __shfl_up_sync(0xffffffffu, ti, off);
        if (lane >= off) {
          ci += a;
          ti += b;
        }
      }
      int o = ci - cs, tt = ti - ts;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 4 * lane + i;
        if (e < E) {
          s_off[e] = o;
          counts[e] = c[i];
          offsets[e] = o;
          for (int m = 0; m < nt4[i]; ++m) {
            tile_expert[tt + m] = e;
            tile_row0[tt + m] = o + m * BM;
            tile_rows[tt + m] = min(BM, c[i] - m * BM);
          }
        }
        o += c[i];
        tt += nt4[i];
      }
      if (lane == 31) {
        offsets[E] = o;
        *tile_num = tt;
      }
    }
    __syncthreads();
    if (tid < P) {
      const int e = s_ids[tid];
      if ((unsigned)e < (unsigned)E) {
        const int pos = s_off[e] + s_bef[tid];
        perm[pos] = tid;
        inv[tid] = pos;
      }
    }
  }
  if (!landed) {
    // drain the late bulk copies of this CTA before it ends
    for (int c = 0; c < kFrontChunks; ++c) mbar_wait_ns(bars + 8 * c, 0, kDrainLimitNs);
  }
  if (xp == nullptr) return;   // the grouped GEMM gathers the rows itself
  cluster_sync();

  // ---- 4. gather the x rows of the sorted pairs (16-byte vectors, 8 per thread in flight)
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
        const int tok = __ldcg(perm + pos) / k;
        r[u] = __ldg(reinterpret_cast<const uint4*>(x) + (size_t)tok * nvec + v);
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
