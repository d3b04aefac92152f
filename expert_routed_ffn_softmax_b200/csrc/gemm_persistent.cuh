// gemm_persistent.cuh -- persistent, warp-specialised grouped GEMM on tcgen05 (the expert
// FFN matmuls; the role SwiftGMM plays on Ascend in "MoE推理「王炸」组合：昇腾×盘古让推理性能
// 狂飙6-8倍", Group 4).  Same tiles, operand layouts and epilogues as grouped_gemm.cuh:
// 128 rows of one expert x 64*NSLAB MMA columns, K staged 64 at a time by TMA (A K-major,
// B MN-major slabs), fp32 accumulators in TMEM, GEGLU / bf16 / fp32 epilogues.
//
// One CTA per SM, 6 warps: warp 0 = TMA producer (lane 0) and TMEM owner, warp 1 = MMA
// issuer (lane 0), warps 2-5 = epilogue (warp w reads TMEM lanes 32*(w%4)..+31).  Two TMEM
// accumulators alternate between work items, so the epilogue of one item overlaps the
// mainloop of the next.  A gathering GEMM adds warps 6-7, which copy the A rows of each
// stage from the unpermuted activations with cp.async (TMA then loads only the weights).
// Eight warps put two on each SM sub-partition, whose 16K registers then allow up to 255
// per thread (ten warps would put three on one and cap every thread at 168).
//
// The warp roles, operand layouts and epilogue helpers here are shared with the default,
// dynamically scheduled expert FFN (ffn_dynamic.cuh).  This file's kernel is the statically
// scheduled form, run when a flag asks for it (one launch for both GEMMs, or two):
// Schedule over U = tiles x column blocks units of nk k-steps each, G CTAs:
//   * whole units, round robin (unit g + i*G), for all but the last one-to-two waves;
//   * the remaining R units (G <= R < 2G, or all of them when U < 2G) are cut into G equal
//     ranges of k-steps ("stream-K"), so every CTA streams the same number of weight bytes.
//     A unit split between CTAs is finished by the CTA that completes its piece last: each
//     epilogue warp stores its 32 rows of the fp32 partial tile and bumps that quadrant's
//     counter; the warp that counts last adds the pieces in piece order (deterministic)
//     and runs the epilogue.  Nothing waits on another CTA or another warp.
#pragma once
#include <cuda.h>
#include "ptx.cuh"
#include "grouped_gemm.cuh"

namespace moe {

constexpr int PG_THREADS = 192;
constexpr int PG_GATHER_THREADS = 64;
constexpr int PG_MAX_THREADS = PG_THREADS + PG_GATHER_THREADS;
constexpr int PG_EPI_THREADS = 128;

__host__ __device__ constexpr int pgemm_threads(bool gather) {
  return gather ? PG_MAX_THREADS : PG_THREADS;
}

// SMALL_A: every tile has at most 8 rows (batches of at most 8 tokens).  A stage then
// holds only 8 A rows (1 KB) and the MMA reads them as all 128 rows of its A operand (the
// descriptor's stride between 8-row groups is 0), so accumulator rows 8..127 repeat rows
// 0..7 and are never stored.  The stages shrink from 48 KB to 33 KB and 6 fit instead of 4:
// half as many weight bytes again in flight per SM, which is what a weight-streaming
// decode step needs.
constexpr int PG_SMALL_ROWS = 8;

template <int NSLAB, bool SMALL_A>
__host__ __device__ constexpr int pgemm_a_bytes() {
  return SMALL_A ? PG_SMALL_ROWS * GM_BK * 2 : GM_A_BYTES;
}

template <int NSLAB, bool SMALL_A>
__host__ __device__ constexpr int pgemm_stage_bytes() {
  return pgemm_a_bytes<NSLAB, SMALL_A>() + NSLAB * GM_SLAB_BYTES;
}

template <int STAGES, int NSLAB, bool SMALL_A = false>
__host__ __device__ constexpr int pgemm_smem_bytes() {
  return 1024 + STAGES * pgemm_stage_bytes<NSLAB, SMALL_A>() + 1024;   // + barriers, flags
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

struct PItem {
  int unit;     // 0 .. U-1
  int kb, ke;   // k-step range [kb, ke)
  int r;        // remainder-unit index (stream-K part), -1 for whole units
};

// The work items of CTA g, in order.  Every role walks the same sequence.
struct PSched {
  int g, G, U, nk, n_dp, i_dp, dp_units;
  long long c, e, Cr, Gs;   // Gs: CTAs sharing the stream-K part, each with >= 1 k-step

  __device__ void init(int g_, int G_, int U_, int nk_) {
    g = g_;
    G = G_;
    U = U_;
    nk = nk_;
    const int waves = U / G;
    dp_units = waves >= 2 ? (waves - 1) * G : 0;
    n_dp = dp_units / G;
    i_dp = 0;
    Cr = (long long)(U - dp_units) * nk;
    Gs = Cr < G ? Cr : G;
    if (g < Gs) {
      c = (long long)g * Cr / Gs;
      e = (long long)(g + 1) * Cr / Gs;
    } else {
      c = e = 0;
    }
  }
  __device__ bool next(PItem& it) {
    if (i_dp < n_dp) {
      it.unit = g + i_dp * G;
      it.kb = 0;
      it.ke = nk;
      it.r = -1;
      ++i_dp;
      return true;
    }
    if (c >= e) return false;
    const int r = (int)(c / nk);
    const int kb = (int)(c - (long long)r * nk);
    const int ke = (int)min((long long)nk, kb + (e - c));
    it.unit = dp_units + r;
    it.kb = kb;
    it.ke = ke;
    it.r = (kb == 0 && ke == nk) ? -1 : r;   // covered whole by this CTA: no partial
    c += ke - kb;
    return true;
  }
  // CTA that owns remainder chunk q (the Gs ranges are all non-empty, so the owners of a
  // unit's chunks are consecutive CTAs).
  __device__ int owner(long long q) const { return (int)(((q + 1) * Gs - 1) / Cr); }
  // Partial-tile slot of (CTA gg, remainder unit r): 2*gg for gg's first unit, else 2*gg+1.
  __device__ int slot(int gg, int r) const {
    const long long first = (long long)gg * Cr / Gs;
    return (first / nk == r) ? 2 * gg : 2 * gg + 1;
  }
};

template <int MODE, int NSLAB>
__device__ __forceinline__ void pg_tile_info(const TileList& tiles, int n_blocks, int unit,
                                             int& e, int& row0, int& rows, int& n0) {
  constexpr int BN = 64 * NSLAB;
  const int tile = unit / n_blocks;
  const int nb = unit - tile * n_blocks;
  if (tiles.uniform_rows > 0) {
    e = 0;
    row0 = tile * GM_BM;
    rows = min(GM_BM, tiles.uniform_rows - row0);
  } else {
    e = tiles.expert[tile];
    row0 = tiles.row0[tile];
    rows = tiles.rows[tile];
  }
  n0 = nb * (MODE == EPI_GEGLU ? BN / 2 : BN);
}

// Epilogue of 32 consecutive accumulator columns [c, c+32) (and, for GEGLU, the up columns
// [BN/2 + c, ...)) given as fp32 values, for one row.
template <int MODE, int NSLAB>
__device__ __forceinline__ void pg_store32(void* out_ptr, int ldo, int row, int n0, int c,
                                           int N_total, const float* g, const float* u) {
  if (MODE == EPI_F32) {
    float* orow = static_cast<float*>(out_ptr) + (size_t)row * ldo + n0 + c;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (n0 + c + 4 * i < N_total)
        reinterpret_cast<float4*>(orow)[i] = make_float4(g[4 * i], g[4 * i + 1], g[4 * i + 2],
                                                         g[4 * i + 3]);
    return;
  }
  if (n0 + c >= N_total) return;
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (MODE == EPI_GEGLU)
      pk[i] = pack_bf16x2(gelu_tanh_f(g[2 * i]) * u[2 * i], gelu_tanh_f(g[2 * i + 1]) * u[2 * i + 1]);
    else
      pk[i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
  }
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out_ptr) + (size_t)row * ldo +
                                        n0 + c);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

// One GEMM of a persistent launch.
struct PGemm {
  int n_blocks;      // output column blocks (BN/2 GEGLU features, or BN columns, each)
  int K;             // reduction depth, a multiple of 64
  int N_total;       // output columns
  void* out;         // output rows, ldo elements apart (bf16; fp32 for EPI_F32)
  int ldo;
  float* partials;   // stream-K partial tiles: 2 per CTA, 128 x BN fp32 each
  int* counters;     // stream-K counters, 4 per split unit; zero at launch, left zero
};

// Epilogue of one work item by one epilogue warp (accumulator rows 32*quad .. +31, in
// TMEM at trow).  Frees the TMEM buffer (arrives on tempty) once it has been read.
// Returns true (warp-uniform) when this warp stored the item's final rows: a whole unit,
// or the last piece of a split unit after adding the pieces in order.
template <int MODE, int NSLAB>
__device__ __forceinline__ bool pg_epilogue(const PGemm& g, const PSched& sch, const PItem& it,
                                            int row0, int rows, int n0, uint32_t trow,
                                            uint32_t tempty, int quad, int lane) {
  constexpr int BN = 64 * NSLAB;
  constexpr int NC = MODE == EPI_GEGLU ? BN / 2 : BN;
  const int r_local = quad * 32 + lane;
  const bool row_ok = r_local < rows;
  const int row = row0 + r_local;
  if (it.r < 0) {
    // whole unit: epilogue straight from TMEM
#pragma unroll 1
    for (int c = 0; c < NC; c += 32) {
      uint32_t gv[32], uv[32];
      tmem_ld_32x32b_x32(trow + c, gv);
      if (MODE == EPI_GEGLU) tmem_ld_32x32b_x32(trow + BN / 2 + c, uv);
      tmem_ld_wait();
      if (row_ok)
        pg_store32<MODE, NSLAB>(g.out, g.ldo, row, n0, c, g.N_total,
                                reinterpret_cast<const float*>(gv),
                                reinterpret_cast<const float*>(uv));
    }
    tc_fence_before();
    mbar_arrive(tempty);
    return true;
  }
  // piece of a split unit: store this warp's 32 rows of the fp32 partial, count the piece,
  // and let the warp that counts last add the pieces in order and finish.
  const int slot = sch.slot(blockIdx.x, it.r);
  float* prow = g.partials + ((size_t)slot * GM_BM + r_local) * BN;
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(trow + c, v);
    tmem_ld_wait();
    if (row_ok) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<uint4*>(prow + c)[i] =
            make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  }
  tc_fence_before();
  mbar_arrive(tempty);
  __threadfence();
  __syncwarp();
  const int nk = sch.nk;
  const long long cf = (long long)it.r * nk, cl = cf + nk - 1;
  const int g_first = sch.owner(cf), n_pieces = sch.owner(cl) - g_first + 1;
  int last = 0;
  if (lane == 0) {
    int* ctr = &g.counters[it.r * 4 + quad];
    last = atomicAdd(ctr, 1) == n_pieces - 1;
    if (last) *ctr = 0;   // ready for the next launch
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return false;
  __threadfence();
  if (row_ok) {
#pragma unroll 1
    for (int c = 0; c < NC; c += 32) {
      float gsum[32], usum[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) gsum[i] = usum[i] = 0.f;
      for (int p = 0; p < n_pieces; ++p) {
        const float* src = g.partials + ((size_t)sch.slot(g_first + p, it.r) * GM_BM + r_local) * BN;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 a = __ldcg(reinterpret_cast<const float4*>(src + c) + i);
          gsum[4 * i] += a.x;
          gsum[4 * i + 1] += a.y;
          gsum[4 * i + 2] += a.z;
          gsum[4 * i + 3] += a.w;
          if (MODE == EPI_GEGLU) {
            const float4 bq = __ldcg(reinterpret_cast<const float4*>(src + BN / 2 + c) + i);
            usum[4 * i] += bq.x;
            usum[4 * i + 1] += bq.y;
            usum[4 * i + 2] += bq.z;
            usum[4 * i + 3] += bq.w;
          }
        }
      }
      pg_store32<MODE, NSLAB>(g.out, g.ldo, row, n0, c, g.N_total, gsum, usum);
    }
  }
  return true;
}

// One launch runs one GEMM (g0), or with FUSED both expert GEMMs: phase 0 = GEMM-1 + GEGLU
// (g0: h = gelu(x Wg) * (x Wu), A gathered from x), then phase 1 = GEMM-2 (g1: O = h Wd, A
// = rows of h by TMA through tmA2, B through tmB2).  Every CTA runs all its phase-0 items
// before its phase-1 items; a phase-1 item waits until the four epilogue warps of every
// phase-0 column block of its tile have stored their h rows (h_ready[tile] = 4 n_blocks).
// Those are always items that run earlier on their CTAs, and every CTA is resident (one
// per SM), so the waits end.  h_ready[n_tiles] counts the same stores over all tiles: once
// a CTA has seen it complete, its later phase-1 items skip the per-tile check (a global
// acquire per item would stall the producer for a memory round trip each time).
//
// GATHER: row r of a tile's phase-0 A operand is tiles.src[perm[row0 + r] / k] (tmA is
// unused).  Rows past the tile's end are not loaded: their accumulator rows hold whatever
// the stage held before and are never stored.  (One TMA tile::gather4 per four rows was
// measured first; its per-instruction cost capped a 128-row tile at about a sixth of the
// MMA rate.)
template <int STAGES, int MODE, int NSLAB, bool GATHER = false, bool FUSED = false,
          bool SMALL_A = false>
__global__ void __launch_bounds__(PG_MAX_THREADS, 1)
    grouped_gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmA,
                                   const __grid_constant__ CUtensorMap tmB0,
                                   const __grid_constant__ CUtensorMap tmB1,
                                   const __grid_constant__ CUtensorMap tmA2,
                                   const __grid_constant__ CUtensorMap tmB2, TileList tiles,
                                   PGemm g0, PGemm g1, int* __restrict__ h_ready) {
  constexpr int BN = 64 * NSLAB;
  constexpr int A_BYTES = pgemm_a_bytes<NSLAB, SMALL_A>();
  constexpr int STAGE_BYTES = pgemm_stage_bytes<NSLAB, SMALL_A>();
  constexpr uint32_t A_SBO = SMALL_A ? 0u : 1024u;   // stride between 8-row groups of A
  constexpr uint32_t TMEM_COLS = 2 * BN;   // two accumulators
  constexpr int NPH = FUSED ? 2 : 1;
  static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1 KB alignment of swizzled tiles");
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of 2");
  static_assert(MODE != EPI_GEGLU || NSLAB % 2 == 0, "GEGLU pairs gate and up slabs");
  static_assert(!FUSED || (MODE == EPI_GEGLU && GATHER), "the fused launch is GEMM-1 then GEMM-2");

  pdl_trigger();

  extern __shared__ uint8_t psm_raw[];
  const uint32_t raw_addr = smem_u32(psm_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* psm = psm_raw + (base - raw_addr);
  const uint32_t bar_base = base + STAGES * STAGE_BYTES;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  uint8_t* misc = psm + STAGES * STAGE_BYTES + 8 * (2 * STAGES + 4);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* n_issued = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* n_consumed = reinterpret_cast<volatile int*>(misc + 12);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), GATHER ? 1 + PG_GATHER_THREADS : 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), PG_EPI_THREADS);
    }
    *abort_flag = 0;
    *n_issued = 0;
    *n_consumed = 0;
    fence_barrier_init();
    if (!GATHER) tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    if (FUSED) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prologue above overlaps the previous kernel; the tile list is its output.
  pdl_wait();
  int n_tiles = 0;
  if (!(*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT))
    n_tiles = tiles.uniform_rows > 0 ? (tiles.uniform_rows + GM_BM - 1) / GM_BM : *tiles.num;
  const int h_target = 4 * g0.n_blocks;
  // Phase p's schedule (every role walks the same sequence of items).
  auto sched = [&](int p) {
    const PGemm& g = p ? g1 : g0;
    PSched sc;
    sc.init(blockIdx.x, gridDim.x, n_tiles * g.n_blocks, g.K / GM_BK);
    return sc;
  };
  PItem it;

  if (warp == 0) {
    // -------------------------------------------------------------- TMA producer (lane 0)
    if (lane == 0) {
      int q = 0;
      bool stop = false, all_h_ready = false;
      for (int p = 0; p < NPH && !stop; ++p) {
        const PGemm& g = p ? g1 : g0;
        const bool a_tma = !(GATHER && p == 0);
        PSched sch = sched(p);
        while (!stop && sch.next(it)) {
          int e, row0, rows, n0;
          if (p == 0)
            pg_tile_info<MODE, NSLAB>(tiles, g.n_blocks, it.unit, e, row0, rows, n0);
          else
            pg_tile_info<EPI_STORE, NSLAB>(tiles, g.n_blocks, it.unit, e, row0, rows, n0);
          if (FUSED && p == 1 && !all_h_ready) {
            // this tile's h rows come from phase-0 items of (possibly) other CTAs
            if (ld_acquire_gpu(h_ready + n_tiles) >= h_target * n_tiles) {
              all_h_ready = true;
            } else if (!wait_counter_geq(h_ready + it.unit / g.n_blocks, h_target)) {
              *abort_flag = 1;
              stop = true;
              break;
            }
            fence_proxy_async_global();   // TMA reads of h after the generic acquire
          }
          for (int kc = it.kb; kc < it.ke; ++kc, ++q) {
            const int s = q % STAGES;
            if (*abort_flag ||
                (q >= STAGES && !mbar_wait(empty_bar(s), ((q / STAGES) - 1) & 1))) {
              *abort_flag = 1;
              stop = true;
              break;
            }
            const uint32_t sA = base + s * STAGE_BYTES;
            const uint32_t sB = sA + A_BYTES;
            mbar_arrive_expect_tx(full_bar(s), (a_tma ? A_BYTES : 0) + NSLAB * GM_SLAB_BYTES);
            // phase 1: the gather warps have left; arrive in their place
            if (FUSED && p == 1) mbar_arrive_cnt(full_bar(s), PG_GATHER_THREADS);
            if (a_tma) tma_load_2d(sA, p ? &tmA2 : &tmA, full_bar(s), kc * GM_BK, row0);
            // one load per projection: NSLAB/2 (gate, up) or NSLAB (down) 64-column slabs
            if (p == 0 && MODE == EPI_GEGLU) {
              tma_load_4d(sB, &tmB0, full_bar(s), 0, kc * GM_BK, n0 / 64, e);
              tma_load_4d(sB + (NSLAB / 2) * GM_SLAB_BYTES, &tmB1, full_bar(s), 0, kc * GM_BK,
                          n0 / 64, e);
            } else {
              tma_load_4d(sB, p ? &tmB2 : &tmB0, full_bar(s), 0, kc * GM_BK, n0 / 64, e);
            }
            *n_issued = q + 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(GM_BM, BN, false, true);
      int q = 0, j = 0;
      bool stop = false;
      for (int p = 0; p < NPH && !stop; ++p) {
        PSched sch = sched(p);
        while (!*abort_flag && sch.next(it)) {
          const int b = j & 1, use = j >> 1;
          if (use >= 1 && !mbar_wait(tempty_bar(b), (use - 1) & 1)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tmem + b * BN;
          bool ok = true;
          for (int kc = it.kb; kc < it.ke; ++kc, ++q) {
            const int s = q % STAGES;
            if (!mbar_wait(full_bar(s), (q / STAGES) & 1)) {
              ok = false;
              break;
            }
            *n_consumed = q + 1;
            if (GATHER && p == 0) fence_proxy_async_smem();   // A came through the generic proxy
            tc_fence_after();
            const uint32_t sA = base + s * STAGE_BYTES;
            const uint32_t sB = sA + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < GM_BK / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(sA + kk * 32, 16, A_SBO);
              const uint64_t bdesc = smem_desc_sw128(sB + kk * 2048, GM_SLAB_BYTES, 1024);
              umma_bf16(dt, adesc, bdesc, idesc, (kc != it.kb || kk != 0) ? 1u : 0u);
            }
            umma_commit(empty_bar(s));
          }
          umma_commit(tfull_bar(b));
          ++j;
          if (!ok) {
            *abort_flag = 1;
            stop = true;
            break;
          }
        }
      }
    }
  } else if (warp < 6) {
    // -------------------------------------------------------------- epilogue (warps 2-5)
    // Each warp owns 32 rows and works on its own: no barrier across the epilogue warps.
    const int quad = warp & 3;
    int j = 0;
    bool stop = false;
    for (int p = 0; p < NPH && !stop; ++p) {
      const PGemm& g = p ? g1 : g0;
      PSched sch = sched(p);
      while (sch.next(it)) {
        const int b = j & 1, use = j >> 1;
        bool got = mbar_wait(tfull_bar(b), use & 1);
        tc_fence_after();
        got = __all_sync(0xffffffffu, got && !*abort_flag);   // warp-uniform decision
        if (!got) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        int e, row0, rows, n0;
        const uint32_t trow = tmem + b * BN + (static_cast<uint32_t>(quad * 32) << 16);
        if (p == 0) {
          pg_tile_info<MODE, NSLAB>(tiles, g.n_blocks, it.unit, e, row0, rows, n0);
          const bool done = pg_epilogue<MODE, NSLAB>(g, sch, it, row0, rows, n0, trow,
                                                     tempty_bar(b), quad, lane);
          if (FUSED && done) {
            // publish this warp's h rows of the tile to the phase-1 TMA loads
            fence_proxy_async_global();
            __threadfence();
            __syncwarp();
            if (lane == 0) {
              red_release_add_gpu(h_ready + it.unit / g.n_blocks, 1);
              red_release_add_gpu(h_ready + n_tiles, 1);
            }
          }
        } else {
          pg_tile_info<EPI_STORE, NSLAB>(tiles, g.n_blocks, it.unit, e, row0, rows, n0);
          pg_epilogue<EPI_STORE, NSLAB>(g, sch, it, row0, rows, n0, trow, tempty_bar(b), quad,
                                        lane);
        }
        ++j;
      }
    }
  } else if (GATHER) {
    // -------------------------------------------------------------- A-row gather (warps 6-7)
    // Gather warp w' = warp - 6 copies tile rows 64w'..64w'+63, four rows per instruction:
    // lane = (sub-row lane/8, 16-byte chunk lane%8).  Chunk c of row r lands where a
    // 128-byte-swizzled TMA box of 64 columns puts it: byte 128 r + 16 (c ^ (r % 8)).
    // Phase 0 only: in phase 1 the TMA thread arrives for these warps.
    const int gw = warp - 6, sub = lane >> 3, ch = lane & 7;
    int q = 0;
    bool stop = false;
    PSched sch = sched(0);
    while (!stop && sch.next(it)) {
      constexpr int NI = GM_BM / (4 * (PG_GATHER_THREADS / 32));   // instructions per stage
      const __nv_bfloat16* src[NI];
      uint32_t doff[NI];
      int e, row0, rows, n0;
      pg_tile_info<MODE, NSLAB>(tiles, g0.n_blocks, it.unit, e, row0, rows, n0);
      if (SMALL_A && rows > PG_SMALL_ROWS) {   // the host never launches this; stay in the slot
        raise_error(MOE_DEVERR_BAD_INDEX);
        rows = PG_SMALL_ROWS;
      }
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const int r = gw * (4 * NI) + 4 * i + sub;
        src[i] = nullptr;
        if (r < rows) {
          const int t = __ldg(tiles.perm + row0 + r) / tiles.k;
          if (t >= 0 && t < tiles.src_rows)
            src[i] = tiles.src + (size_t)t * tiles.ld + 8 * ch;
          else
            raise_error(MOE_DEVERR_BAD_INDEX);   // row left uncopied
        }
        doff[i] = static_cast<uint32_t>(r * 128 + ((ch ^ (r & 7)) << 4));
      }
      for (int kc = it.kb; kc < it.ke; ++kc, ++q) {
        const int s = q % STAGES;
        bool ok = !*abort_flag && (q < STAGES || mbar_wait(empty_bar(s), ((q / STAGES) - 1) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        const uint32_t sA = base + s * STAGE_BYTES;
#pragma unroll
        for (int i = 0; i < NI; ++i)
          if (src[i] != nullptr) cp_async_16(sA + doff[i], src[i] + kc * GM_BK);
        cp_async_arrive_noinc(full_bar(s));
      }
    }
    cp_async_wait_all();   // nothing of ours lands in shared memory after this CTA ends
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    raise_error(MOE_DEVERR_TIMEOUT);
    for (int q = *n_consumed; q < *n_issued; ++q)
      mbar_wait_ns(full_bar(q % STAGES), (q / STAGES) & 1, kDrainLimitNs);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace moe
