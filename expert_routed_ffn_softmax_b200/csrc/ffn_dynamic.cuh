// ffn_dynamic.cuh -- the expert FFN (GEMM-1 + GEGLU, then GEMM-2) of a batch in one
// persistent launch whose CTAs take their work from a shared counter.
//
// The work is cut into units -- (row tile, 128 GEMM-1 features) and (row tile, 256 GEMM-2
// columns) -- handed out in order from one global counter: every GEMM-1 unit before any
// GEMM-2 unit, so a CTA never waits for work that is handed out after its own, and SMs that
// stream faster simply take more units (with a fixed split the slowest SM sets the end).
// Each unit is summed over its whole K in one TMEM accumulator (two alternate, so one
// unit's epilogue overlaps the next unit's mainloop) and its epilogue works straight from
// TMEM: GEGLU and a bf16 store of h (GEMM-1), a bf16 store of the expert output (GEMM-2).
// A GEMM-1 unit then publishes h_ready[tile]; a GEMM-2 unit issues its W_down loads for
// the first stages, waits for h_ready, then loads its h rows.
//
// Roles as in gemm_persistent.cuh (TMA thread, MMA thread, 4 epilogue warps, gather warps:
// 4 for 128-row slots, 2 otherwise), with A slots of R = 8 ... 128 rows (every tile has at most R rows).  The TMA
// thread takes unit ids and passes them to the other roles through a ring of descriptors
// in shared memory (full / empty mbarriers).  A tile list from the dispatch describes the
// routed rows (expert, first sorted row, rows; the A rows gathered from x through perm);
// without a list (TileList::uniform_rows) the rows of x form one "expert" in 128-row
// tiles, which is how the dense MLP beside the MoE runs.  Every wait is bounded.
#pragma once
#include "gemm_persistent.cuh"

namespace moe {

constexpr int DY_RING = 8;                           // unit descriptors in flight per CTA

// R = rows of a tile's A slot: 8, 16, 32 or 64 for batches of T <= R tokens (at most T
// rows per tile), 128 for any batch (tiles are at most 128 rows).  The MMA reads 128 rows
// of A; rows past R read the stage's weight bytes, which follow the slot, and their
// accumulator rows are never stored.
template <int R>
struct DyShape {
  static_assert(R == 8 || R == 16 || R == 32 || R == 64 || R == 128, "A slot rows");
  static constexpr int A_BYTES = R * GM_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + 4 * GM_SLAB_BYTES;
  static constexpr int STAGES = R <= 32 ? 6 : R == 64 ? 5 : 4;
  static constexpr int ROW_WARPS = (R + 31) / 32;    // epilogue warps holding rows
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 2048;
};

struct DyState {
  int* next;       // [1] next unit id; zero at launch
};

template <int R>
__host__ __device__ inline int dy_smem_bytes() {
  return DyShape<R>::SMEM;
}

// Gather warps: four for 128-row slots (large batches, where GEMM-1 waits on its gathered
// rows), two otherwise.  The kernel's threads: TMA, MMA, 4 epilogue warps, the gather warps.
template <int R>
__host__ __device__ constexpr int dy_gather_warps() {
  return R == 128 ? 4 : 2;
}
template <int R>
__host__ __device__ constexpr int dy_threads() {
  return PG_THREADS + 32 * dy_gather_warps<R>();
}

// A unit: phase 0 = GEMM-1, 1 = GEMM-2; unit index within its GEMM; k-steps [kb, ke).
struct DyChunk {
  int phase, unit, kb, ke;
};
__device__ __forceinline__ DyChunk dy_decode(int c, int U1, int nk1, int nk2) {
  DyChunk d;
  d.phase = c < U1 ? 0 : 1;
  d.unit = c < U1 ? c : c - U1;
  d.kb = 0;
  d.ke = c < U1 ? nk1 : nk2;
  return d;
}

// A GEMM-1 column block covers 128 features: 128 gate and 128 up columns in one N = 256
// MMA.  When I % 128 == 64 the last block has 64 features; it runs an N = 128 MMA (gate in
// slab 0, up in slab 1, loaded with the one-slab maps tmWg1 / tmWu1) instead of computing
// 128 zero-filled columns.
__device__ __forceinline__ bool dy_narrow_block(const DyChunk& d, const PGemm& g1) {
  return d.phase == 0 && (g1.N_total & 127) != 0 && d.unit % g1.n_blocks == g1.n_blocks - 1;
}

// tmH: h rows, box R rows x 64 columns.  tmWg / tmWu: two-slab boxes; tmWg1 / tmWu1: one-slab
// boxes (the narrow last GEMM-1 block).  tmX: GEMM-1's A rows when tiles.a_tma (box R rows x
// 64 columns of a contiguous row-major tensor), else unused.
template <int R>
__global__ void __launch_bounds__(PG_THREADS + 128, 1)
    expert_ffn_dynamic_kernel(const __grid_constant__ CUtensorMap tmWg,
                              const __grid_constant__ CUtensorMap tmWu,
                              const __grid_constant__ CUtensorMap tmWg1,
                              const __grid_constant__ CUtensorMap tmWu1,
                              const __grid_constant__ CUtensorMap tmX,
                              const __grid_constant__ CUtensorMap tmH,
                              const __grid_constant__ CUtensorMap tmWd, TileList tiles,
                              PGemm g1, PGemm g2, int* __restrict__ h_ready, DyState dy) {
  using SH = DyShape<R>;
  constexpr int NSLAB = 4, BN = 256;
  constexpr int A_BYTES = SH::A_BYTES;
  constexpr int STAGE_BYTES = SH::STAGE_BYTES;
  constexpr int DY_STAGES = SH::STAGES;
  constexpr int NRW = SH::ROW_WARPS;
  constexpr uint32_t TMEM_COLS = 2 * BN;

  pdl_trigger();
  extern __shared__ uint8_t dsm_raw[];
  const uint32_t raw_addr = smem_u32(dsm_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* dsm = dsm_raw + (base - raw_addr);
  const uint32_t bar_base = base + DY_STAGES * STAGE_BYTES;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (DY_STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * DY_STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * DY_STAGES + 2 + b); };
  auto dfull_bar = [&](int r) { return bar_base + 8u * (2 * DY_STAGES + 4 + r); };
  auto dempty_bar = [&](int r) { return bar_base + 8u * (2 * DY_STAGES + 4 + DY_RING + r); };
  uint8_t* misc = dsm + DY_STAGES * STAGE_BYTES + 8 * (2 * DY_STAGES + 4 + 2 * DY_RING);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* n_issued = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* n_consumed = reinterpret_cast<volatile int*>(misc + 12);
  volatile int* ring = reinterpret_cast<volatile int*>(misc + 16);   // [DY_RING] unit ids

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // arrivals that release a descriptor: MMA thread, 4 epilogue warps, 2 gather warps
  constexpr int NGW = dy_gather_warps<R>(), GATHER_THREADS = 32 * NGW;
  constexpr int kDescReaders = 1 + 4 + NGW;
  if (tid == 0) {
    for (int s = 0; s < DY_STAGES; ++s) {
      mbar_init(full_bar(s), 1 + GATHER_THREADS);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), PG_EPI_THREADS);
    }
    for (int r = 0; r < DY_RING; ++r) {
      mbar_init(dfull_bar(r), 1);
      mbar_init(dempty_bar(r), kDescReaders);
    }
    *abort_flag = 0;
    *n_issued = 0;
    *n_consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmWg);
    tma_prefetch_desc(&tmWu);
    if (g1.N_total & 127) {
      tma_prefetch_desc(&tmWg1);
      tma_prefetch_desc(&tmWu1);
    }
    if (tiles.a_tma) tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmWd);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();   // the tile list, counters and x come from the previous kernels
  int n_tiles = 0;
  if (!(*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT))
    n_tiles = tiles.uniform_rows > 0 ? (tiles.uniform_rows + GM_BM - 1) / GM_BM : *tiles.num;
  const int U1 = n_tiles * g1.n_blocks, U2 = n_tiles * g2.n_blocks;
  const int nk1 = g1.K / GM_BK, nk2 = g2.K / GM_BK;
  const int total = U1 + U2;
  const int h_target = NRW * g1.n_blocks;   // one release per (GEMM-1 unit, row warp)

  // Read descriptor i (bounded wait); every reader then releases it.  -1 = no more work,
  // -2 = a wait ran out.
  auto read_desc = [&](int i) -> int {
    const int r = i % DY_RING;
    if (!mbar_wait(dfull_bar(r), (i / DY_RING) & 1)) return -2;
    return ring[r];
  };

  if (warp == 0) {
    // -------------------------------------------------------------- TMA producer (lane 0)
    if (lane == 0) {
      int q = 0, i = 0;
      bool all_h_ready = false;
      int c = atomicAdd(dy.next, 1);
      while (true) {
        const int r = i % DY_RING;
        if (i >= DY_RING && !mbar_wait(dempty_bar(r), ((i / DY_RING) - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        const bool stop = *abort_flag || c >= total;
        ring[r] = stop ? -1 : c;
        mbar_arrive(dfull_bar(r));
        if (stop) break;
        const int cnext = atomicAdd(dy.next, 1);   // claimed one unit ahead
        const DyChunk d = dy_decode(c, U1, nk1, nk2);
        int e, row0, rows, n0;
        if (d.phase == 0)
          pg_tile_info<EPI_GEGLU, NSLAB>(tiles, g1.n_blocks, d.unit, e, row0, rows, n0);
        else
          pg_tile_info<EPI_STORE, NSLAB>(tiles, g2.n_blocks, d.unit, e, row0, rows, n0);
        const bool narrow = dy_narrow_block(d, g1);
        // Issue stage `kc` of the unit: wait for the slot; B (and, unless deferred, A).
        auto stage_in = [&](int kc, int qq, bool with_a) -> bool {
          const int s = qq % DY_STAGES;
          if (*abort_flag ||
              (qq >= DY_STAGES && !mbar_wait(empty_bar(s), ((qq / DY_STAGES) - 1) & 1))) {
            *abort_flag = 1;
            return false;
          }
          const uint32_t sA = base + s * STAGE_BYTES;
          const uint32_t sB = sA + A_BYTES;
          if (d.phase == 0) {
            const uint32_t b_bytes = (narrow ? 2 : NSLAB) * GM_SLAB_BYTES;
            if (tiles.a_tma) {
              mbar_arrive_expect_tx(full_bar(s), b_bytes + A_BYTES);
              mbar_arrive_cnt(full_bar(s), GATHER_THREADS);   // in place of the gather warps
              tma_load_2d(sA, &tmX, full_bar(s), kc * GM_BK, row0);
            } else {
              mbar_arrive_expect_tx(full_bar(s), b_bytes);
            }
            if (narrow) {
              tma_load_4d(sB, &tmWg1, full_bar(s), 0, kc * GM_BK, n0 / 64, e);
              tma_load_4d(sB + GM_SLAB_BYTES, &tmWu1, full_bar(s), 0, kc * GM_BK, n0 / 64, e);
            } else {
              tma_load_4d(sB, &tmWg, full_bar(s), 0, kc * GM_BK, n0 / 64, e);
              tma_load_4d(sB + (NSLAB / 2) * GM_SLAB_BYTES, &tmWu, full_bar(s), 0, kc * GM_BK,
                          n0 / 64, e);
            }
          } else {
            mbar_arrive_expect_tx(full_bar(s), A_BYTES + NSLAB * GM_SLAB_BYTES);
            mbar_arrive_cnt(full_bar(s), GATHER_THREADS);   // in place of the gather warps
            tma_load_4d(sB, &tmWd, full_bar(s), 0, kc * GM_BK, n0 / 64, e);
            if (with_a) tma_load_2d(sA, &tmH, full_bar(s), kc * GM_BK, row0);
          }
          *n_issued = qq + 1;
          return true;
        };
        bool ok = true;
        int kc = d.kb;
        if (d.phase == 1 && !all_h_ready) {
          // GEMM-2 needs this tile's h rows (GEMM-1 units of any CTA).  The W_down tiles do
          // not: load them for the first stages, then wait for h, then load its rows.
          const int pre = min(d.ke - d.kb, DY_STAGES);
          for (int t2 = 0; t2 < pre && ok; ++t2) ok = stage_in(d.kb + t2, q + t2, false);
          if (ok) {
            if (!wait_counter_geq(h_ready + d.unit / g2.n_blocks, h_target)) {
              *abort_flag = 1;
              ok = false;
            } else {
              all_h_ready = ld_acquire_gpu(h_ready + n_tiles) >= h_target * n_tiles;
              fence_proxy_async_global();   // TMA reads of h after the generic acquire
              for (int t2 = 0; t2 < pre; ++t2) {
                const int s = (q + t2) % DY_STAGES;
                tma_load_2d(base + s * STAGE_BYTES, &tmH, full_bar(s), (d.kb + t2) * GM_BK, row0);
              }
            }
          }
          kc += pre;
          q += pre;
        }
        for (; ok && kc < d.ke; ++kc, ++q) ok = stage_in(kc, q, true);
        if (!ok) break;
        c = cnext;
        ++i;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_full = idesc_bf16_f32(GM_BM, BN, false, true);
      constexpr uint32_t idesc_narrow = idesc_bf16_f32(GM_BM, BN / 2, false, true);
      int q = 0;
      for (int i = 0;; ++i) {
        const int c = read_desc(i);
        mbar_arrive(dempty_bar(i % DY_RING));
        if (c < 0) {
          if (c == -2) *abort_flag = 1;
          break;
        }
        const DyChunk d = dy_decode(c, U1, nk1, nk2);
        const uint32_t idesc = dy_narrow_block(d, g1) ? idesc_narrow : idesc_full;
        const int b = i & 1, use = i >> 1;
        if (use >= 1 && !mbar_wait(tempty_bar(b), (use - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem + b * BN;
        bool ok = true;
        for (int kc = d.kb; kc < d.ke; ++kc, ++q) {
          const int s = q % DY_STAGES;
          if (!mbar_wait(full_bar(s), (q / DY_STAGES) & 1)) {
            ok = false;
            break;
          }
          *n_consumed = q + 1;
          if (d.phase == 0 && !tiles.a_tma) fence_proxy_async_smem();   // A came by cp.async
          tc_fence_after();
          const uint32_t sA = base + s * STAGE_BYTES;
          const uint32_t sB = sA + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < GM_BK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sA + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sB + kk * 2048, GM_SLAB_BYTES, 1024);
            umma_bf16(dt, adesc, bdesc, idesc, (kc != d.kb || kk != 0) ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
        }
        umma_commit(tfull_bar(b));
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp < 6) {
    // -------------------------------------------------------------- epilogue (warps 2-5)
    // Warp w reads TMEM lanes 32 (w % 4) .. +31; the rows of a tile (< R) sit in the first
    // NRW of those quadrants.  The other warps only keep the accumulator hand-off going.
    const int quad = warp & 3;
    const bool rows_warp = quad < NRW;
    for (int i = 0;; ++i) {
      int c = 0;
      if (lane == 0) c = read_desc(i);
      c = __shfl_sync(0xffffffffu, c, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty_bar(i % DY_RING));
      if (c < 0) {
        if (c == -2) *abort_flag = 1;
        break;
      }
      const DyChunk d = dy_decode(c, U1, nk1, nk2);
      const int b = i & 1, use = i >> 1;
      bool got = mbar_wait(tfull_bar(b), use & 1);
      tc_fence_after();
      got = __all_sync(0xffffffffu, got && !*abort_flag);
      if (!got) {
        *abort_flag = 1;
        break;
      }
      const PGemm& g = d.phase == 0 ? g1 : g2;
      int e, row0, rows, n0;
      if (d.phase == 0)
        pg_tile_info<EPI_GEGLU, NSLAB>(tiles, g.n_blocks, d.unit, e, row0, rows, n0);
      else
        pg_tile_info<EPI_STORE, NSLAB>(tiles, g.n_blocks, d.unit, e, row0, rows, n0);
      const int r_local = quad * 32 + lane;
      const bool row_ok = rows_warp && r_local < rows && r_local < R;
      const uint32_t trow = tmem + b * BN + (static_cast<uint32_t>(quad * 32) << 16);
      // epilogue straight from TMEM
      if (rows_warp) {
        // GEMM-1: gate columns [0, NC), up columns [NC, 2 NC) of the accumulator
        const bool narrow = dy_narrow_block(d, g1);
        const int NC = d.phase == 0 ? (narrow ? BN / 4 : BN / 2) : BN;
#pragma unroll 1
        for (int cc = 0; cc < NC; cc += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld_32x32b_x32(trow + cc, gv);
          if (d.phase == 0) tmem_ld_32x32b_x32(trow + NC + cc, uv);
          tmem_ld_wait();
          if (row_ok) {
            if (d.phase == 0)
              pg_store32<EPI_GEGLU, NSLAB>(g.out, g.ldo, row0 + r_local, n0, cc, g.N_total,
                                           reinterpret_cast<const float*>(gv),
                                           reinterpret_cast<const float*>(uv));
            else
              pg_store32<EPI_STORE, NSLAB>(g.out, g.ldo, row0 + r_local, n0, cc, g.N_total,
                                           reinterpret_cast<const float*>(gv),
                                           reinterpret_cast<const float*>(uv));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(b));
      if (d.phase == 0 && rows_warp) {
        // publish this warp's h rows of the unit to the GEMM-2 TMA loads
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) {
          red_release_add_gpu(h_ready + d.unit / g1.n_blocks, 1);
          red_release_add_gpu(h_ready + n_tiles, 1);
        }
      }
    }
  } else {
    // -------------------------------------------------------------- A-row gather (warps 6..)
    // GEMM-1 units: the <= R rows of the tile, 16-byte cp.async into the 128-byte-swizzled
    // slot (chunk c of row r at byte 128 r + 16 (c ^ r)).  GEMM-2 units, and GEMM-1 units
    // whose A rows come by TMA: nothing (the TMA thread arrives in their place), but the
    // stage count must follow.
    const int gw = warp - 6, sub = lane >> 3, ch = lane & 7;
    int q = 0;
    for (int i = 0;; ++i) {
      int c = 0;
      if (lane == 0) c = read_desc(i);
      c = __shfl_sync(0xffffffffu, c, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty_bar(i % DY_RING));
      if (c < 0) {
        if (c == -2) *abort_flag = 1;
        break;
      }
      const DyChunk d = dy_decode(c, U1, nk1, nk2);
      if (d.phase == 1 || tiles.a_tma) {
        q += d.ke - d.kb;
        continue;
      }
      int e, row0, rows, n0;
      pg_tile_info<EPI_GEGLU, NSLAB>(tiles, g1.n_blocks, d.unit, e, row0, rows, n0);
      if (rows > R) {   // never launched so; stay inside the slot
        raise_error(MOE_DEVERR_BAD_INDEX);
        rows = R;
      }
      // gather warp gw copies rows gw R/NGW .. (gw + 1) R/NGW - 1, four rows per instruction
      constexpr int NI = R / (4 * NGW);
      const __nv_bfloat16* src[NI];
      uint32_t doff[NI];
#pragma unroll
      for (int u = 0; u < NI; ++u) {
        const int r = gw * (R / NGW) + 4 * u + sub;
        src[u] = nullptr;
        if (r < rows) {
          // the routed pair's token, or (no permutation: one dense layer) the row itself
          const int t = tiles.perm ? __ldg(tiles.perm + row0 + r) / tiles.k : row0 + r;
          if (t >= 0 && t < tiles.src_rows)
            src[u] = tiles.src + (size_t)t * tiles.ld + 8 * ch;
          else
            raise_error(MOE_DEVERR_BAD_INDEX);
        }
        doff[u] = static_cast<uint32_t>(r * 128 + ((ch ^ (r & 7)) << 4));
      }
      bool stop = false;
      for (int kc = d.kb; kc < d.ke; ++kc, ++q) {
        const int s = q % DY_STAGES;
        bool ok = !*abort_flag &&
                  (q < DY_STAGES || mbar_wait(empty_bar(s), ((q / DY_STAGES) - 1) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        const uint32_t sA = base + s * STAGE_BYTES;
#pragma unroll
        for (int u = 0; u < NI; ++u)
          if (src[u] != nullptr) cp_async_16(sA + doff[u], src[u] + kc * GM_BK);
        cp_async_arrive_noinc(full_bar(s));
      }
      if (stop) break;
    }
    cp_async_wait_all();
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    raise_error(MOE_DEVERR_TIMEOUT);
    for (int q = *n_consumed; q < *n_issued; ++q)
      mbar_wait_ns(full_bar(q % DY_STAGES), (q / DY_STAGES) & 1, kDrainLimitNs);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace moe
