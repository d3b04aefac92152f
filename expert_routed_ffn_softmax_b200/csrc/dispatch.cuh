// dispatch.cuh -- per-expert histogram, exclusive scan, stable permutation and the row
// gather that makes each expert's tokens contiguous (the per-expert "split sizes" of the
// double_routing dispatch, cann-recipes-infer Gemma-4-26B-A4B optimisation report §6.1
// 方案), plus the unpermute-combine y[t] = sum_j w[t,j] * O[inv[t,j]].
//
// The permutation lists, expert by expert, the pairs q = t*k + j in ascending q, so it is
// unique and identical to the definition: pairs are cut into fixed chunks, each chunk
// counts its experts, a scan turns the counts into per-(chunk, expert) bases, and one
// warp per chunk ranks its pairs in order with __match_any_sync.
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kDispatchChunk = 2048;   // pairs per chunk

// chunk_counts[c][e] = #pairs with id e in chunk c.
__global__ void __launch_bounds__(256) dispatch_count_kernel(const int32_t* __restrict__ ids,
                                                              int P, int E,
                                                              int32_t* __restrict__ chunk_counts) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int q0 = blockIdx.x * kDispatchChunk, q1 = min(P, q0 + kDispatchChunk);
  for (int q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
    const int e = ids[q];
    if ((unsigned)e < (unsigned)E)
      atomicAdd(&hist[e], 1);
    else
      raise_error(MOE_DEVERR_BAD_INDEX);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[(size_t)blockIdx.x * E + e] = hist[e];
}

// One CTA (blockDim >= E).  counts, offsets, chunk_base[c][e] = offsets[e] + pairs of e in
// chunks before c, and the GEMM tile list: for every expert with n_e > 0, tiles of BM rows
// (expert, first sorted row, rows in tile), in expert order.  Also zeroes the split-unit
// counters the grouped GEMMs use.  Thread e walks its column of chunk counts with 8 loads
// in flight; warp 0 scans the experts (8 per lane) with shuffles.
__device__ __forceinline__ void dispatch_scan_block(
    const int32_t* __restrict__ chunk_counts, int nchunks, int E, int P, int BM,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ chunk_base,
    int32_t* __restrict__ tile_num, int32_t* __restrict__ tile_expert,
    int32_t* __restrict__ tile_row0, int32_t* __restrict__ tile_rows,
    int32_t* __restrict__ gemm_counters, int n_counters, int* s_cnt, int* s_off, int* s_tstart) {
  for (int i = threadIdx.x; i < n_counters; i += blockDim.x) gemm_counters[i] = 0;
  const int e = threadIdx.x, lane = threadIdx.x & 31;
  int run = 0;
  if (e < E) {
    for (int c0 = 0; c0 < nchunks; c0 += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = c0 + u < nchunks ? __ldcg(chunk_counts + (size_t)(c0 + u) * E + e) : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (c0 + u < nchunks) chunk_base[(size_t)(c0 + u) * E + e] = run;
        run += v[u];
      }
    }
    s_cnt[e] = run;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // exclusive scans of counts and tiles over the experts; lane owns 8*lane .. 8*lane+7
    int c[8], nt[8], cs = 0, ts = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = 8 * lane + i;
      c[i] = ee < E ? s_cnt[ee] : 0;
      nt[i] = (c[i] + BM - 1) / BM;
      cs += c[i];
      ts += nt[i];
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
    for (int i = 0; i < 8; ++i) {
      const int ee = 8 * lane + i;
      if (ee < E) {
        s_off[ee] = o;
        s_tstart[ee] = tt;
      }
      o += c[i];
      tt += nt[i];
    }
    if (lane == 31) {
      offsets[E] = o;
      *tile_num = tt;
    }
  }
  __syncthreads();
  if (e < E) {
    const int off = s_off[e];
    counts[e] = run;
    offsets[e] = off;
    for (int c = 0; c < nchunks; ++c) chunk_base[(size_t)c * E + e] += off;
    const int nt = (run + BM - 1) / BM;
    for (int m = 0; m < nt; ++m) {
      const int i = s_tstart[e] + m;
      tile_expert[i] = e;
      tile_row0[i] = off + m * BM;
      tile_rows[i] = min(BM, run - m * BM);
    }
  }
}

__global__ void __launch_bounds__(256) dispatch_scan_kernel(
    const int32_t* __restrict__ chunk_counts, int nchunks, int E, int P, int BM,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ chunk_base,
    int32_t* __restrict__ tile_num, int32_t* __restrict__ tile_expert,
    int32_t* __restrict__ tile_row0, int32_t* __restrict__ tile_rows,
    int32_t* __restrict__ gemm_counters, int n_counters) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_cnt[256], s_off[256], s_tstart[256];
  dispatch_scan_block(chunk_counts, nchunks, E, P, BM, counts, offsets, chunk_base, tile_num,
                      tile_expert, tile_row0, tile_rows, gemm_counters, n_counters, s_cnt, s_off,
                      s_tstart);
}

// One CTA of 8 warps per chunk: warp w takes pairs [256 w, 256 w + 256) of the chunk
// (8 per lane, loaded up front), counts them per expert, the warps' counts are scanned in
// warp order per expert, and each warp ranks its pairs in order with __match_any_sync:
// pos = chunk_base[c][e] + pairs of e in earlier warps + rank within the warp's earlier
// pairs.  perm[pos] = q, inv[q] = pos.  Dynamic shared memory: 9 * E ints.
constexpr int kRankWarps = 8;
constexpr int kRankSub = kDispatchChunk / kRankWarps;   // 256 pairs per warp

// This warp's pairs of chunk c (expert ids; -1 past P, -2 for an id out of range) and its
// per-expert counts in wcnt[warp][e] (zeroed by the caller).
__device__ __forceinline__ void rank_load_count(const int32_t* __restrict__ ids, int P, int E,
                                                int c, int* wcnt, int (&ev)[kRankSub / 32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q0 = c * kDispatchChunk + warp * kRankSub;
#pragma unroll
  for (int it = 0; it < kRankSub / 32; ++it) {
    const int q = q0 + 32 * it + lane;
    int e = q < P ? __ldcg(ids + q) : -1;
    if (q < P && (unsigned)e >= (unsigned)E) e = -2;   // counted as an error already
    ev[it] = e;
  }
#pragma unroll
  for (int it = 0; it < kRankSub / 32; ++it) {
    const int e = ev[it];
    const unsigned grp = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == 31 - __clz(grp)) wcnt[warp * E + e] += __popc(grp);
    __syncwarp();
  }
}

// After the warps' counts and base[e] = chunk_base[c][e] are in shared memory (and a block
// barrier): scan the counts over the warps, then place every pair.
__device__ __forceinline__ void rank_place(int E, int c, int* wcnt, const int* base,
                                           const int (&ev)[kRankSub / 32],
                                           int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // exclusive scan over the warps, per expert (in place): wcnt[w][e] = pairs of e in warps < w
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = base[e];
#pragma unroll
    for (int w = 0; w < kRankWarps; ++w) {
      const int v = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  int* wb = wcnt + warp * E;   // this warp's running base per expert
  const unsigned lt = (1u << lane) - 1u;
  const int q0 = c * kDispatchChunk + warp * kRankSub;
#pragma unroll
  for (int it = 0; it < kRankSub / 32; ++it) {
    const int q = q0 + 32 * it + lane;
    const int e = ev[it];
    const unsigned grp = __match_any_sync(0xffffffffu, e);
    int pos = 0;
    if (e >= 0) pos = wb[e] + __popc(grp & lt);
    __syncwarp();
    if (e >= 0 && lane == 31 - __clz(grp)) wb[e] += __popc(grp);
    __syncwarp();
    if (e >= 0) {
      perm[pos] = q;
      inv[q] = pos;
    }
  }
}

__global__ void __launch_bounds__(32 * kRankWarps) dispatch_rank_kernel(
    const int32_t* __restrict__ ids, int P, int E, const int32_t* __restrict__ chunk_base,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int rank_sm[];
  int* wcnt = rank_sm;                   // [kRankWarps][E] pairs of e in warp w
  int* base = rank_sm + kRankWarps * E;  // [E] chunk base
  const int c = blockIdx.x;
  for (int i = threadIdx.x; i < kRankWarps * E; i += blockDim.x) wcnt[i] = 0;
  for (int i = threadIdx.x; i < E; i += blockDim.x) base[i] = chunk_base[(size_t)c * E + i];
  __syncthreads();
  int ev[kRankSub / 32];
  rank_load_count(ids, P, E, c, wcnt, ev);
  __syncthreads();
  rank_place(E, c, wcnt, base, ev, perm, inv);
}

// The three kernels above in one launch, for few chunks (every CTA must be resident at
// once, so at most the SM count): CTA c counts chunk c and publishes its counts; the CTA that arrives last (a counter)
// runs the scan and raises a flag; every CTA waits (bounded) for the flag, reads its chunk's
// bases and ranks its pairs.  sync[0] (arrivals) and sync[1] (flag) are zero at launch.
// Dynamic shared memory: (kRankWarps + 1) * E ints.
__global__ void __launch_bounds__(32 * kRankWarps) dispatch_fused_kernel(
    const int32_t* __restrict__ ids, int P, int E, int BM, int nchunks,
    int32_t* __restrict__ chunk_counts, int32_t* __restrict__ chunk_base,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv, int32_t* __restrict__ tile_num, int32_t* __restrict__ tile_expert,
    int32_t* __restrict__ tile_row0, int32_t* __restrict__ tile_rows,
    int32_t* __restrict__ gemm_counters, int n_counters, int* __restrict__ sync) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int rank_sm[];
  int* wcnt = rank_sm;
  int* base = rank_sm + kRankWarps * E;
  __shared__ int s_cnt[256], s_off[256], s_tstart[256];
  __shared__ int s_last, s_ok;
  const int c = blockIdx.x;
  for (int i = threadIdx.x; i < kRankWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  int ev[kRankSub / 32];
  rank_load_count(ids, P, E, c, wcnt, ev);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int n = 0;
#pragma unroll
    for (int w = 0; w < kRankWarps; ++w) n += wcnt[w * E + e];
    chunk_counts[(size_t)c * E + e] = n;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&sync[0], 1) == nchunks - 1;
  __syncthreads();
  if (s_last) {
    __threadfence();   // every chunk's counts before reading them
    dispatch_scan_block(chunk_counts, nchunks, E, P, BM, counts, offsets, chunk_base, tile_num,
                        tile_expert, tile_row0, tile_rows, gemm_counters, n_counters, s_cnt,
                        s_off, s_tstart);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) red_release_add_gpu(&sync[1], 1);
  }
  if (threadIdx.x == 0) s_ok = wait_counter_geq(&sync[1], 1);
  __syncthreads();
  if (!s_ok) return;   // timed out: the error word is set
  for (int i = threadIdx.x; i < E; i += blockDim.x) base[i] = __ldcg(chunk_base + (size_t)c * E + i);
  __syncthreads();
  rank_place(E, c, wcnt, base, ev, perm, inv);
}

// Whole dispatch for a batch of at most one chunk (P <= kDispatchChunk) by one CTA (any
// size >= 32 threads; warp 0 scans and ranks): histogram, scan, tile list and the stable
// ranks, as the kernels above compute them for many chunks; also zeroes the split-unit
// counters of the grouped GEMMs.  s_*: four shared arrays of 256 ints.
__device__ __forceinline__ void dispatch_small_block(
    const int32_t* __restrict__ ids, int P, int E, int BM, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    int32_t* __restrict__ tile_num, int32_t* __restrict__ tile_expert,
    int32_t* __restrict__ tile_row0, int32_t* __restrict__ tile_rows,
    int32_t* __restrict__ gemm_counters, int n_counters, int* s_cnt, int* s_off, int* s_base,
    int* s_tstart) {
  // s_base: running rank base per expert (advanced by the ranking warp); s_off stays the
  // expert's first row for the tile list, which other threads build at the same time.
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < n_counters; i += blockDim.x) gemm_counters[i] = 0;
  for (int i = tid; i < 256; i += blockDim.x) s_cnt[i] = 0;
  __syncthreads();
  for (int q = tid; q < P; q += blockDim.x) {
    const int e = __ldcg(ids + q);
    if ((unsigned)e < (unsigned)E)
      atomicAdd(&s_cnt[e], 1);
    else
      raise_error(MOE_DEVERR_BAD_INDEX);
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scans of counts and of tiles per expert; lane owns experts 8*lane..8*lane+7
    int c[8], nt[8], cs = 0, ts = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      c[i] = e < E ? s_cnt[e] : 0;
      nt[i] = (c[i] + BM - 1) / BM;
      cs += c[i];
      ts += nt[i];
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
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < E) {
        s_off[e] = o;
        s_base[e] = o;
        s_tstart[e] = tt;
        counts[e] = c[i];
        offsets[e] = o;
      }
      o += c[i];
      tt += nt[i];
    }
    if (lane == 31) {
      offsets[E] = o;
      *tile_num = tt;
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int n = s_cnt[e], off = s_off[e], nt = (n + BM - 1) / BM;
    for (int m = 0; m < nt; ++m) {
      const int i = s_tstart[e] + m;
      tile_expert[i] = e;
      tile_row0[i] = off + m * BM;
      tile_rows[i] = min(BM, n - m * BM);
    }
  }
  if (warp == 0) {
    const unsigned lt = (1u << lane) - 1u;
    for (int qb = 0; qb < P; qb += 32) {
      const int q = qb + lane;
      int e = q < P ? __ldcg(ids + q) : -1;
      if (q < P && (unsigned)e >= (unsigned)E) e = -2;
      const unsigned grp = __match_any_sync(0xffffffffu, e);
      int pos = 0;
      if (e >= 0) pos = s_base[e] + __popc(grp & lt);
      __syncwarp();
      if (e >= 0 && lane == 31 - __clz(grp)) s_base[e] += __popc(grp);
      __syncwarp();
      if (e >= 0) {
        perm[pos] = q;
        inv[q] = pos;
      }
    }
  }
}

__global__ void __launch_bounds__(256) dispatch_small_kernel(
    const int32_t* __restrict__ ids, int P, int E, int BM, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    int32_t* __restrict__ tile_num, int32_t* __restrict__ tile_expert,
    int32_t* __restrict__ tile_row0, int32_t* __restrict__ tile_rows,
    int32_t* __restrict__ gemm_counters, int n_counters) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_cnt[256], s_off[256], s_base[256], s_tstart[256];
  dispatch_small_block(ids, P, E, BM, counts, offsets, perm, inv, tile_num, tile_expert,
                       tile_row0, tile_rows, gemm_counters, n_counters, s_cnt, s_off, s_base,
                       s_tstart);
}

// Xp[pos, :] = x[perm[pos] / k, :] for pos < P   (16-byte vectors over all (row, vector)
// pairs, 8 loads per thread issued before the stores).  perm holds pair indices t*k + j below
// n_pairs (it may be a slice of a longer permutation).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ perm, int P,
                                                          int k, int n_pairs, int nvec,
                                                          uint4* __restrict__ xp) {
  pdl_trigger();
  pdl_wait();
  // After a timeout upstream perm may be stale: skip the work (the error word says why).
  if (*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT) return;
  const long long total = (long long)P * nvec;
  const long long nthr = (long long)gridDim.x * blockDim.x;
  for (long long b0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; b0 < total;
       b0 += 8 * nthr) {
    uint4 r[8];
    bool ok[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const long long idx = b0 + u * nthr;
      ok[u] = false;
      if (idx < total) {
        const int pos = (int)(idx / nvec), v = (int)(idx - (long long)pos * nvec);
        const int q = perm[pos];
        if ((unsigned)q < (unsigned)n_pairs) {   // the source row t = q / k is then < T
          r[u] = x[(size_t)(q / k) * nvec + v];
          ok[u] = true;
        } else {
          raise_error(MOE_DEVERR_BAD_INDEX);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const long long idx = b0 + u * nthr;
      if (ok[u]) xp[idx] = r[u];
    }
  }
}

// y[t, :] = sum_{j ascending} w[t,j] * O[inv[t,j], :]   (fp32, one rounding to the output)
// One warp per item (token t, chunk c of 64 16-byte vectors of the row): lanes j < k fetch
// slot j's row and weight, which the warp shares by shuffles; then each lane loads its two
// vectors of all k rows (16 loads in flight) and sums them in slot order.  Only sorted rows
// in [row_lo, row_hi) contribute (the rest count as zero): the whole layer passes [0, T*k);
// an expert-parallel rank passes the rows of its own experts and writes an fp32 partial sum
// (F32OUT) for the cross-rank reduction.  y holds 8 values per 16-byte vector of O.
constexpr int kCombineChunkVec = 64;
template <bool F32OUT>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ O,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ w, int T, int k,
                                                      int nvec, int row_lo, int row_hi,
                                                      void* __restrict__ y_out) {
  pdl_trigger();
  pdl_wait();
  // After a timeout upstream inv may be stale: skip the work (the error word says why).
  if (*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT) return;
  const int lane = threadIdx.x & 31;
  const int P = T * k;
  const int nch = (nvec + kCombineChunkVec - 1) / kCombineChunkVec;
  const long long items = (long long)T * nch;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long it = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items;
       it += nwarps) {
    const int t = (int)(it / nch), c = (int)(it - (long long)t * nch);
    int myp = 0;
    float myw = 0.f;
    bool myon = false;
    if (lane < k) {
      myp = __ldg(inv + (size_t)t * k + lane);
      myw = __ldg(w + (size_t)t * k + lane);
      if ((unsigned)myp >= (unsigned)P) {   // never written so: read nothing for this slot
        raise_error(MOE_DEVERR_BAD_INDEX);
      } else {
        myon = myp >= row_lo && myp < row_hi;
      }
      if (!myon) {
        myp = 0;
        myw = 0.f;
      }
    }
    const unsigned on = __ballot_sync(0xffffffffu, myon);
    int pos[8];
    float wj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      pos[j] = __shfl_sync(0xffffffffu, myp, j);
      wj[j] = __shfl_sync(0xffffffffu, myw, j);
    }
    const int v0 = c * kCombineChunkVec + lane, v1 = v0 + 32;
    const bool ok0 = v0 < nvec, ok1 = v1 < nvec;
    uint4 r0[8], r1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      r0[j] = r1[j] = make_uint4(0u, 0u, 0u, 0u);
      const bool use = j < k && ((on >> j) & 1u);
      if (use && ok0) r0[j] = __ldcs(O + (size_t)pos[j] * nvec + v0);
      if (use && ok1) r1[j] = __ldcs(O + (size_t)pos[j] * nvec + v1);
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (half == 0 ? !ok0 : !ok1) continue;
      const uint4* r = half == 0 ? r0 : r1;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && ((on >> j) & 1u)) {
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&r[j]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            acc[2 * i] = fmaf(wj[j], f.x, acc[2 * i]);
            acc[2 * i + 1] = fmaf(wj[j], f.y, acc[2 * i + 1]);
          }
        }
      }
      const size_t vi = (size_t)t * nvec + (half == 0 ? v0 : v1);
      if (F32OUT) {
        float4* yo = static_cast<float4*>(y_out) + 2 * vi;
        yo[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        yo[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
        uint4 out;
        out.x = pack_bf16x2(acc[0], acc[1]);
        out.y = pack_bf16x2(acc[2], acc[3]);
        out.z = pack_bf16x2(acc[4], acc[5]);
        out.w = pack_bf16x2(acc[6], acc[7]);
        static_cast<uint4*>(y_out)[vi] = out;
      }
    }
  }
}

// Tile list of a grouped FFN over caller-given row segments (one CTA): segment i holds
// seg_rows[i] consecutive rows of local expert seg_expert[i], segments back to back from row
// 0.  Tiles of BM rows never cross a segment.  Also zeroes the FFN's counters.  A segment
// with an expert id outside [0, E) or a negative row count raises BAD_INDEX and gets no tiles;
// segments that add up to more than N rows (the rows the caller's buffers hold) raise
// BAD_INDEX and produce no tiles at all, so nothing is read or written past row N.
constexpr int kMaxSegments = 1024;
__global__ void __launch_bounds__(256) segment_tiles_kernel(
    const int32_t* __restrict__ seg_rows, const int32_t* __restrict__ seg_expert, int n_seg,
    int N, int E, int BM, int max_tiles, int32_t* __restrict__ tile_num,
    int32_t* __restrict__ tile_expert, int32_t* __restrict__ tile_row0,
    int32_t* __restrict__ tile_rows, int32_t* __restrict__ counters, int n_counters) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_start[kMaxSegments], s_tstart[kMaxSegments];
  for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
  if (threadIdx.x == 0) {
    // segments are few (ranks x local experts): a serial scan keeps the order obvious
    int row = 0, tt = 0;
    for (int i = 0; i < n_seg; ++i) {
      int n = __ldg(seg_rows + i);
      const int e = __ldg(seg_expert + i);
      if (n < 0 || (n > 0 && (unsigned)e >= (unsigned)E)) {
        raise_error(MOE_DEVERR_BAD_INDEX);
        n = -1;
      }
      s_start[i] = row;
      s_tstart[i] = n > 0 ? tt : -1;
      if (n > 0) {
        row += n;
        tt += (n + BM - 1) / BM;
      }
    }
    if (row > N || tt > max_tiles) {   // more rows than the caller's buffers hold
      raise_error(MOE_DEVERR_BAD_INDEX);
      tt = 0;
    }
    *tile_num = tt;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_seg; i += blockDim.x) {
    const int t0 = s_tstart[i];
    if (t0 < 0 || *tile_num == 0) continue;
    const int n = __ldg(seg_rows + i), e = __ldg(seg_expert + i);
    for (int m = 0; m * BM < n; ++m) {
      tile_expert[t0 + m] = e;
      tile_row0[t0 + m] = s_start[i] + m * BM;
      tile_rows[t0 + m] = min(BM, n - m * BM);
    }
  }
}

}  // namespace moe
