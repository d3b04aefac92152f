// decode_front.cuh -- router and dispatch of a small batch (T <= 8 tokens) in one launch:
// one cluster of 8 CTAs per token (the role of the fused gating top-k softmax op in the
// cann-recipes-infer "Gemma-4-26B-A4B 模型优化报告", §5 阶段3, plus the per-expert split
// sizes of §6.1, for a decode batch).
//
//   1. CTA r of token t's cluster copies the h-slice [r*H/8, (r+1)*H/8) of W_router into
//      shared memory with four bulk copies (one per pair of warps, so a warp starts as soon
//      as its rows land), stages the token's x slice as doubles, and its 8 warps compute
//      fp64 partial logits over the slice (each an FMA chain in ascending h over an eighth
//      of it, added in warp order) and partial squared norms; these go to the cluster's
//      CTA 0 through distributed shared memory.  All CTAs zero the GEMM counters while
//      their copies are in flight;
//   2. cluster barrier; CTA 0 adds the 8 partials in rank order and finishes token t with
//      all its threads (thread e ranks expert e against the others, every decision is
//      verified against the rounding bound; a token too close to call goes to the warp path
//      of router_select_kernel, which recomputes it exactly);
//   3. the token's CTA 0 that finishes last (a counter in global memory) runs the dispatch
//      of the T*k <= 64 pairs (counts, offsets, stable permutation, tile list).
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

// Dynamic shared memory layout (bytes from a 16-byte aligned base):
//   W   max(hs*E*2, 2*NW*E*8)    W_router slice (bf16), later the cross-warp reduction
//   XS  hs*8                     the token's x slice as doubles
//   PART kFrontRanks*E*8         (CTA 0) partial logits per source rank
//   PWN  kFrontRanks*E*8         |W[:,e]|^2 partials per source rank
//   PXN  kFrontRanks*8           (CTA 0) |x_t|^2 partials per source rank
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
  const size_t wbytes = hs * E * 2, red = (size_t)2 * kFrontWarps * E * 8;
  L.w = take(wbytes > red ? wbytes : red);
  L.xs = take(hs * 8);
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
// Grid: T clusters of kFrontRanks CTAs (cluster c = token c).  done: a counter in global
// memory that is zero at launch (the finisher of the dispatch leaves it zero).
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
                        int n_counters, int BM, unsigned* __restrict__ done) {
  static_assert(EPL == 4, "the partial-logit loop reads 4 experts per lane");
  pdl_trigger();
  constexpr int NW = kFrontWarps;
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
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int t = (int)(blockIdx.x / kFrontRanks);   // this cluster's token
  const int hs = H / kFrontRanks, h0 = rank * hs;
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
  // the token's x slice as doubles
  for (int v = tid; v < hs / 8; v += blockDim.x) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + h0) + v);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p2[i]);
      xs[8 * v + 2 * i] = (double)f.x;
      xs[8 * v + 2 * i + 1] = (double)f.y;
    }
  }
  // The GEMM counters are zeroed by all CTAs while the W_router copies are in flight (this
  // launch runs in plain stream order: no earlier GEMM is still using them).
  for (int i = blockIdx.x * blockDim.x + tid; i < n_counters; i += gridDim.x * blockDim.x)
    gemm_counters[i] = 0;
  __syncthreads();   // also publishes the barrier initialisation
  // |x_t|^2 over the slice -> CTA 0
  if (warp == 0) {
    double sq = 0.0;
    for (int hh = lane; hh < hs; hh += 32) sq = fma(xs[hh], xs[hh], sq);
#pragma unroll
    for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (lane == 0) st_cluster_f64(mapa_shared(smem_u32(pxn + rank), 0), sq);
  }
  const int sub = hs / NW, hb = warp * sub, e0 = lane * EPL;
  const bool active = e0 < E;
  double acc[EPL], wn[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) acc[i] = wn[i] = 0.0;
  // This warp's rows lie in one bulk copy (sub = crow / 2).  If it does not land in time
  // (the error word then says so), the warp skips its rows; every CTA still takes every
  // cluster barrier below, so the cluster ends together.
  const bool landed = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (hb / crow), 0));
  if (active && landed) {
#pragma unroll 4
    for (int r = 0; r < sub; ++r) {
      const uint2 raw = *reinterpret_cast<const uint2*>(wsl + (size_t)(hb + r) * E + e0);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
      const double xv = xs[hb + r];
#pragma unroll
      for (int i = 0; i < EPL / 2; ++i) {
        const double w0 = (double)__low2float(p[i]), w1 = (double)__high2float(p[i]);
        acc[2 * i] = fma(xv, w0, acc[2 * i]);
        acc[2 * i + 1] = fma(xv, w1, acc[2 * i + 1]);
        wn[2 * i] = fma(w0, w0, wn[2 * i]);
        wn[2 * i + 1] = fma(w1, w1, wn[2 * i + 1]);
      }
    }
  }
  __syncthreads();   // the slice is consumed: its space becomes the reduction buffer
  if (active) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      red[(size_t)warp * E + e0 + i] = acc[i];
      red[(size_t)(NW + warp) * E + e0 + i] = wn[i];
    }
  }
  __syncthreads();
  // partial logits and |W[:,e]|^2 partials (warp order) -> CTA 0
  for (int e = tid; e < E; e += blockDim.x) {
    double v = red[e], w2 = red[(size_t)NW * E + e];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      v += red[(size_t)w * E + e];
      w2 += red[(size_t)(NW + w) * E + e];
    }
    st_cluster_f64(mapa_shared(smem_u32(part + (size_t)rank * E + e), 0), v);
    st_cluster_f64(mapa_shared(smem_u32(pwn + (size_t)rank * E + e), 0), w2);
  }
  cluster_sync();

  // ---- 2. CTA 0 finishes token t with all its threads: thread e < E owns expert e
  double* sL = topk;                 // [E] logits
  double* sB = topk + E;             // [E] rounding bounds
  double* sSelV = topk + 2 * E;      // [8] selected logits, slot order
  double* sSelB = sSelV + 8;         // [8] their bounds
  int* sSelE = reinterpret_cast<int*>(sSelB + 8);   // [8] selected experts
  if (rank == 0) {
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
        }
      }
      // ---- 3. the last token to finish runs the dispatch
      __threadfence();
      __syncwarp();
      if (lane == 0) {
        const unsigned prev = atomicAdd(done, 1u);
        s_last = prev == (unsigned)T - 1;
        if (s_last) *done = 0;   // ready for the next launch
      }
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      const int P = T * k;
      if (tid < P) s_ids[tid] = __ldcg(ids + tid);
      __syncthreads();
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
  }
  if (!landed) {
    // drain the late bulk copies of this CTA before it ends
    for (int c = 0; c < kFrontChunks; ++c) mbar_wait_ns(bars + 8 * c, 0, kDrainLimitNs);
  }
}

}  // namespace moe
