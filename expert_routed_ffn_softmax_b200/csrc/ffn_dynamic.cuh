// ffn_dynamic.cuh -- the expert FFN (GEMM-1 + GEGLU, then GEMM-2) of a batch of at most 8
// tokens in one persistent launch whose CTAs take their work from a shared counter.
//
// A decode step streams the weights of every chosen expert once; the layer's time is that
// stream.  With a fixed split of the work each CTA streams the same bytes, but SMs do not
// stream at the same rate, so the slowest CTA sets the end, and GEMM-2 can only start a tile
// once GEMM-1 has stored it.  Here the work is cut into chunks of a few 64-deep k-steps
// (CH1 chunks per GEMM-1 unit = (tile, 128 features), CH2 per GEMM-2 unit = (tile, 256
// columns)), handed out in order from one global counter: every GEMM-1 chunk before any
// GEMM-2 chunk, so a CTA never waits for work that is handed out after its own.  A chunk's
// fp32 partial (at most R rows x 256 columns) goes to global memory; the CTA that completes
// a unit's last chunk adds the unit's partials in chunk order (deterministic whatever the
// timing), applies GEGLU (GEMM-1) or rounds (GEMM-2) and stores the rows.  GEMM-1 units
// publish h_ready[tile]; a GEMM-2 chunk's TMA load of h waits for it.
//
// Roles as in gemm_persistent.cuh (TMA thread, MMA thread, 4 epilogue warps, 2 gather
// warps), with A slots of R <= 64 rows (batches of T <= R tokens).  The TMA thread takes chunk ids and
// passes them to the other roles through a ring of descriptors in shared memory (full /
// empty mbarriers).  Every wait is bounded.
#pragma once
#include "gemm_persistent.cuh"

namespace moe {

constexpr int DY_RING = 8;                           // chunk descriptors in flight per CTA
constexpr int DY_CH1 = 1;                            // chunks per GEMM-1 unit
constexpr int DY_CH2 = 1;                            // chunks per GEMM-2 unit

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
  static constexpr int PART_FLOATS = R * 256;        // one chunk's partial tile
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 2048;
};

struct DyState {
  int* next;       // [1] next chunk id; zero at launch
  int* done1;      // [U1][ROW_WARPS] finished chunks per GEMM-1 unit; zero at launch
  int* done2;      // [U2][ROW_WARPS] finished chunks per GEMM-2 unit; zero at launch
  float* part1;    // [U1 * CH1][R][256] (unused when CH1 == 1)
  float* part2;    // [U2 * CH2][R][256] (unused when CH2 == 1)
};

template <int R>
__host__ __device__ inline int dy_smem_bytes() {
  return DyShape<R>::SMEM;
}

// A chunk: phase 0 = GEMM-1, 1 = GEMM-2; unit; chunk index j within the unit; k-steps
// [kb, ke).  A unit of nk k-steps has ch = min(CH, nk) chunks, none empty.
struct DyChunk {
  int phase, unit, j, kb, ke;
};
__device__ __forceinline__ DyChunk dy_decode(int c, int U1, int nk1, int nk2, int ch1,
                                             int ch2) {
  DyChunk d;
  const int total1 = U1 * ch1;
  if (c < total1) {
    d.phase = 0;
    d.unit = c / ch1;
    d.j = c - d.unit * ch1;
    d.kb = d.j * nk1 / ch1;
    d.ke = (d.j + 1) * nk1 / ch1;
  } else {
    d.phase = 1;
    const int c2 = c - total1;
    d.unit = c2 / ch2;
    d.j = c2 - d.unit * ch2;
    d.kb = d.j * nk2 / ch2;
    d.ke = (d.j + 1) * nk2 / ch2;
  }
  return d;
}

// tmH: h rows, box R rows x 64 columns.
template <int R>
__global__ void __launch_bounds__(PG_MAX_THREADS, 1)
    expert_ffn_dynamic_kernel(const __grid_constant__ CUtensorMap tmWg,
                              const __grid_constant__ CUtensorMap tmWu,
                              const __grid_constant__ CUtensorMap tmH,
                              const __grid_constant__ CUtensorMap tmWd, TileList tiles,
                              PGemm g1, PGemm g2, int* __restrict__ h_ready, DyState dy) {
  using SH = DyShape<R>;
  constexpr int NSLAB = 4, BN = 256;
  constexpr int A_BYTES = SH::A_BYTES;
  constexpr int STAGE_BYTES = SH::STAGE_BYTES;
  constexpr int DY_STAGES = SH::STAGES;
  constexpr int NRW = SH::ROW_WARPS;
  constexpr int PARTF = SH::PART_FLOATS;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  static_assert(DY_CH1 >= 1 && DY_CH2 >= 1, "chunks");

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
  volatile int* ring = reinterpret_cast<volatile int*>(misc + 16);   // [DY_RING] chunk ids

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // arrivals that release a descriptor: MMA thread, 4 epilogue warps, 2 gather warps
  constexpr int kDescReaders = 1 + 4 + PG_GATHER_THREADS / 32;
  if (tid == 0) {
    for (int s = 0; s < DY_STAGES; ++s) {
      mbar_init(full_bar(s), 1 + PG_GATHER_THREADS);
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
  const int ch1 = min(DY_CH1, nk1), ch2 = min(DY_CH2, nk2);
  const int total = U1 * ch1 + U2 * ch2;
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
        const int cnext = atomicAdd(dy.next, 1);   // claimed one chunk ahead
        const DyChunk d = dy_decode(c, U1, nk1, nk2, ch1, ch2);
        int e, row0, rows, n0;
        if (d.phase == 0)
          pg_tile_info<EPI_GEGLU, NSLAB>(tiles, g1.n_blocks, d.unit, e, row0, rows, n0);
        else
          pg_tile_info<EPI_STORE, NSLAB>(tiles, g2.n_blocks, d.unit, e, row0, rows, n0);
        // Issue stage `kc` of the chunk: wait for the slot; B (and, unless deferred, A).
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
            mbar_arrive_expect_tx(full_bar(s), NSLAB * GM_SLAB_BYTES);
            tma_load_4d(sB, &tmWg, full_bar(s), 0, kc * GM_BK, n0 / 64, e);
            tma_load_4d(sB + (NSLAB / 2) * GM_SLAB_BYTES, &tmWu, full_bar(s), 0, kc * GM_BK,
                        n0 / 64, e);
          } else {
            mbar_arrive_expect_tx(full_bar(s), A_BYTES + NSLAB * GM_SLAB_BYTES);
            mbar_arrive_cnt(full_bar(s), PG_GATHER_THREADS);   // in place of the gather warps
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
      constexpr uint32_t idesc = idesc_bf16_f32(GM_BM, BN, false, true);
      int q = 0;
      for (int i = 0;; ++i) {
        const int c = read_desc(i);
        mbar_arrive(dempty_bar(i % DY_RING));
        if (c < 0) {
          if (c == -2) *abort_flag = 1;
          break;
        }
        const DyChunk d = dy_decode(c, U1, nk1, nk2, ch1, ch2);
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
          if (d.phase == 0) fence_proxy_async_smem();   // A came through the generic proxy
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
      const DyChunk d = dy_decode(c, U1, nk1, nk2, ch1, ch2);
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
      const int nch = d.phase == 0 ? ch1 : ch2;
      const int r_local = quad * 32 + lane;
      const bool row_ok = rows_warp && r_local < rows && r_local < R;
      const uint32_t trow = tmem + b * BN + (static_cast<uint32_t>(quad * 32) << 16);
      if (nch == 1) {
        // the whole unit in one chunk: epilogue straight from TMEM
        if (rows_warp) {
          const int NC = d.phase == 0 ? BN / 2 : BN;
#pragma unroll 1
          for (int cc = 0; cc < NC; cc += 32) {
            uint32_t gv[32], uv[32];
            tmem_ld_32x32b_x32(trow + cc, gv);
            if (d.phase == 0) tmem_ld_32x32b_x32(trow + BN / 2 + cc, uv);
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
      } else {
        float* part = (d.phase == 0 ? dy.part1 + (size_t)d.unit * DY_CH1 * PARTF
                                    : dy.part2 + (size_t)d.unit * DY_CH2 * PARTF);
        if (rows_warp) {
          // this chunk's partial rows -> global
          float* prow = part + (size_t)d.j * PARTF + (size_t)r_local * 256;
#pragma unroll 1
          for (int cc = 0; cc < BN; cc += 32) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(trow + cc, v);
            tmem_ld_wait();
            if (row_ok) {
#pragma unroll
              for (int k4 = 0; k4 < 8; ++k4)
                reinterpret_cast<uint4*>(prow + cc)[k4] =
                    make_uint4(v[4 * k4], v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(b));
        if (!rows_warp) continue;
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          int* ctr = (d.phase == 0 ? dy.done1 : dy.done2) + d.unit * NRW + quad;
          last = atomicAdd(ctr, 1) == nch - 1;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        // the unit's last chunk: add the partials in chunk order and finish the rows
        __threadfence();
        if (row_ok) {
          constexpr int NC1 = BN / 2;
          const int NC = d.phase == 0 ? NC1 : BN;
#pragma unroll 1
          for (int cc = 0; cc < NC; cc += 32) {
            float gsum[32], usum[32];
#pragma unroll
            for (int k2 = 0; k2 < 32; ++k2) gsum[k2] = usum[k2] = 0.f;
            for (int jj = 0; jj < nch; ++jj) {
              const float* src = part + (size_t)jj * PARTF + (size_t)r_local * 256;
#pragma unroll
              for (int k4 = 0; k4 < 8; ++k4) {
                const float4 a4 = __ldcg(reinterpret_cast<const float4*>(src + cc) + k4);
                gsum[4 * k4] += a4.x;
                gsum[4 * k4 + 1] += a4.y;
                gsum[4 * k4 + 2] += a4.z;
                gsum[4 * k4 + 3] += a4.w;
                if (d.phase == 0) {
                  const float4 bq = __ldcg(reinterpret_cast<const float4*>(src + NC1 + cc) + k4);
                  usum[4 * k4] += bq.x;
                  usum[4 * k4 + 1] += bq.y;
                  usum[4 * k4 + 2] += bq.z;
                  usum[4 * k4 + 3] += bq.w;
                }
              }
            }
            if (d.phase == 0)
              pg_store32<EPI_GEGLU, NSLAB>(g.out, g.ldo, row0 + r_local, n0, cc, g.N_total, gsum,
                                           usum);
            else
              pg_store32<EPI_STORE, NSLAB>(g.out, g.ldo, row0 + r_local, n0, cc, g.N_total, gsum,
                                           usum);
          }
        }
      }
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
    // -------------------------------------------------------------- A-row gather (warps 6-7)
    // GEMM-1 chunks: the <= R rows of the tile, 16-byte cp.async into the 128-byte-swizzled
    // slot (chunk c of row r at byte 128 r + 16 (c ^ r)).  GEMM-2 chunks: nothing (the TMA
    // thread arrives in their place), but the stage count must follow.
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
      const DyChunk d = dy_decode(c, U1, nk1, nk2, ch1, ch2);
      if (d.phase == 1) {
        q += d.ke - d.kb;
        continue;
      }
      int e, row0, rows, n0;
      pg_tile_info<EPI_GEGLU, NSLAB>(tiles, g1.n_blocks, d.unit, e, row0, rows, n0);
      if (rows > R) {   // never launched so; stay inside the slot
        raise_error(MOE_DEVERR_BAD_INDEX);
        rows = R;
      }
      // warp 6 copies rows 0 .. R/2-1, warp 7 rows R/2 .. R-1, four rows per instruction
      constexpr int NI = R / 8;
      const __nv_bfloat16* src[NI];
      uint32_t doff[NI];
#pragma unroll
      for (int u = 0; u < NI; ++u) {
        const int r = gw * (R / 2) + 4 * u + sub;
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
