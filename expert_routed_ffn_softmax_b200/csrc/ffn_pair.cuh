// ffn_pair.cuh -- the expert FFN of a large batch on CTA pairs: GEMM-1 + GEGLU and GEMM-2 in
// one persistent launch of 2-CTA clusters, every MMA a tcgen05.mma.cta_group::2 of M = 256
// rows (the role SwiftGMM's grouped matmul plays on Ascend, "MoE推理「王炸」组合：昇腾×盘古让推理
// 性能狂飙6-8倍", Group 4).
//
// Why pairs: a single-CTA unit of 128 rows x 256 columns streams 16 KB of A and 32 KB of B
// through shared memory per 64-deep k-step, for 512 cycles of MMA -- about as many bytes per
// cycle as shared memory and L2 deliver, so the tensor pipe idles on operands.  A pair computes
// a 256 x 256 tile: each CTA loads its own 128 A rows and half of the B columns (16 + 16 KB per
// k-step), and the MMA of M = 256 reads the peer's half of A and B from the peer's shared
// memory.  Operand bytes per FLOP drop by a third, and six stages fit instead of four.
//
// Work units are (pair tile, column block): a pair tile is up to 256 sorted rows of one
// expert (the dispatch cuts tiles of 256), rank 0 of the cluster takes rows [0, 128) of it
// and rank 1 rows [128, 256).  GEMM-1 blocks put 128 gate columns in rank 0 and the same 128
// up columns in rank 1, so each CTA's TMEM row holds g and u of every feature of the block
// (columns [0,128) and [128,256)), exactly as in the single-CTA kernel; a narrow last block
// (I % 128 == 64) runs N = 128.  GEMM-2 blocks are 256 output columns, 128 per CTA.
//
// Roles (both CTAs, 8 warps):
//   warp 0 lane 0  TMA producer.  Rank 0 also takes unit ids from the global counter and
//                  writes each into both CTAs' descriptor rings.  Both producers load their
//                  half of B (and, for GEMM-2, their 128 h rows) with the cta_group::2 TMA
//                  form, whose byte count lands on rank 0's full barrier; rank 0 announces
//                  the bytes of both.  No load uses cluster multicast.
//   warp 1 lane 0  rank 0: MMA issuer (tcgen05.mma.cta_group::2; commits arrive on both
//                  CTAs' barriers).  Rank 1: forwards "A rows landed" for the stages whose A
//                  rows its gather warps copy -- they complete a local barrier, this thread
//                  then arrives on rank 0's full barrier (cp.async cannot signal another CTA's
//                  barrier).  Stages loaded by TMA alone need no forward: their bytes count on
//                  rank 0's barrier and rank 0's producer arrives for rank 1.
//   warps 2-5      epilogue from this CTA's TMEM (its 128 rows): GEGLU + bf16 h, or bf16 O;
//                  releases the accumulator to rank 0 and publishes h_ready.
//   warps 6-7      GEMM-1 A-row gather of this CTA's 128 rows from x through perm (cp.async
//                  into the 128-byte-swizzled layout).
// Every wait is bounded; a wait that runs out sets the error word, and every path still
// reaches the closing cluster barrier, so neither CTA leaves while the other can touch it.
#pragma once
#include "ffn_dynamic.cuh"

namespace moe {

constexpr int PR_ROWS = 2 * GM_BM;                     // rows of a pair tile
constexpr int PR_STAGES = 6;
constexpr int PR_A_BYTES = GM_BM * GM_BK * 2;          // 16 KB: this CTA's 128 rows
constexpr int PR_B_BYTES = 2 * GM_SLAB_BYTES;          // 16 KB: this CTA's 128 MMA columns
constexpr int PR_STAGE_BYTES = PR_A_BYTES + PR_B_BYTES;
constexpr int PR_SMEM = 1024 + PR_STAGES * PR_STAGE_BYTES + 2048;
// ring readers: rank 0 MMA thread, 4 epilogue warps, 2 gather warps; rank 1 TMA thread,
// forwarder, 4 epilogue warps, 2 gather warps
constexpr int PR_DESC_READERS = 7 + 8;
constexpr int PR_EPI_WARPS = 8;                        // accumulator releases per unit (both CTAs)


// (expert, first sorted row, rows <= 256, first output column) of pair unit `unit`.
__device__ __forceinline__ void pr_tile_info(const TileList& tiles, int n_blocks, int unit,
                                             bool geglu, int& e, int& row0, int& rows, int& n0) {
  const int tile = unit / n_blocks;
  const int nb = unit - tile * n_blocks;
  if (tiles.uniform_rows > 0) {
    e = 0;
    row0 = tile * PR_ROWS;
    rows = min(PR_ROWS, tiles.uniform_rows - row0);
  } else {
    e = tiles.expert[tile];
    row0 = tiles.row0[tile];
    rows = tiles.rows[tile];
  }
  n0 = nb * (geglu ? 128 : 256);
}

// tmWg / tmWu: two-slab boxes of W_gate / W_up; tmWg1 / tmWu1: one-slab boxes (narrow last
// GEMM-1 block); tmX: 128 rows x 64 columns of GEMM-1's A rows when tiles.a_tma; tmH: 128
// rows x 64 columns of h; tmWd: two-slab boxes of W_down.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PG_MAX_THREADS, 1)
    expert_ffn_pair_kernel(const __grid_constant__ CUtensorMap tmWg,
                           const __grid_constant__ CUtensorMap tmWu,
                           const __grid_constant__ CUtensorMap tmWg1,
                           const __grid_constant__ CUtensorMap tmWu1,
                           const __grid_constant__ CUtensorMap tmX,
                           const __grid_constant__ CUtensorMap tmH,
                           const __grid_constant__ CUtensorMap tmWd, TileList tiles, PGemm g1,
                           PGemm g2, int* __restrict__ h_ready, DyState dy) {
  constexpr int BN = 256;
  constexpr int S = PR_STAGES;
  constexpr uint32_t TMEM_COLS = 2 * BN;

  pdl_trigger();
  extern __shared__ uint8_t psm_raw[];
  const uint32_t raw_addr = smem_u32(psm_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* psm = psm_raw + (base - raw_addr);
  const uint32_t bar_base = base + S * PR_STAGE_BYTES;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };
  auto afull_bar = [&](int s) { return bar_base + 8u * (2 * S + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (3 * S + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (3 * S + 2 + b); };
  auto dfull_bar = [&](int r) { return bar_base + 8u * (3 * S + 4 + r); };
  auto dempty_bar = [&](int r) { return bar_base + 8u * (3 * S + 4 + DY_RING + r); };
  uint8_t* misc = psm + S * PR_STAGE_BYTES + 8 * (3 * S + 4 + 2 * DY_RING);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* n_issued = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* n_consumed = reinterpret_cast<volatile int*>(misc + 12);
  volatile int* ring = reinterpret_cast<volatile int*>(misc + 16);   // [DY_RING] unit ids
  const uint32_t ring_addr = smem_u32(misc + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();   // 0 issues the MMAs, 1 is its peer
  const bool leader = rank == 0;
  const int half0 = leader ? 0 : GM_BM;     // this CTA's first row within a pair tile
  auto at_leader = [&](uint32_t a) { return mapa_shared(a, 0); };
  auto at_peer = [&](uint32_t a) { return mapa_shared(a, 1); };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      // rank 0: its TMA thread (bytes of both CTAs), its 64 gather threads (or the TMA
      // thread for them), rank 1's forwarder
      mbar_init(full_bar(s), 1 + PG_GATHER_THREADS + 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(afull_bar(s), PG_GATHER_THREADS);   // rank 1: its gather threads (per
                                                     // gathered stage, in gather order)
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), PR_EPI_WARPS);
    }
    for (int r = 0; r < DY_RING; ++r) {
      mbar_init(dfull_bar(r), 1);
      mbar_init(dempty_bar(r), PR_DESC_READERS);
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
  cluster_sync();   // both CTAs' barriers exist before any remote arrival or TMA names them
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();   // the tile list, counters and x come from the previous kernels
  int n_tiles = 0;
  if (!(*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT))
    n_tiles = tiles.uniform_rows > 0 ? (tiles.uniform_rows + PR_ROWS - 1) / PR_ROWS : *tiles.num;
  const int U1 = n_tiles * g1.n_blocks, U2 = n_tiles * g2.n_blocks;
  const int nk1 = g1.K / GM_BK, nk2 = g2.K / GM_BK;
  const int total = U1 + U2;
  const int h_target = PR_EPI_WARPS * g1.n_blocks;   // one release per (GEMM-1 unit, warp)

  auto read_desc = [&](int i) -> int {
    const int r = i % DY_RING;
    if (!mbar_wait_cl(dfull_bar(r), (i / DY_RING) & 1)) return -2;
    return ring[r];
  };
  auto release_desc = [&](int i) {
    const uint32_t b = dempty_bar(i % DY_RING);
    if (leader)
      mbar_arrive(b);
    else
      mbar_arrive_remote(at_leader(b));
  };

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- TMA producers
      int q = 0, i = 0;
      bool all_h_ready = false;
      int c = leader ? atomicAdd(dy.next, 1) : 0;
      while (true) {
        if (leader) {
          const int r = i % DY_RING;
          if (i >= DY_RING && !mbar_wait(dempty_bar(r), ((i / DY_RING) - 1) & 1)) {
            *abort_flag = 1;
            break;
          }
          const bool stop = *abort_flag || c >= total;
          const int v = stop ? -1 : c;
          ring[r] = v;
          st_cluster_u32(at_peer(ring_addr + 4u * r), static_cast<uint32_t>(v));
          mbar_arrive(dfull_bar(r));
          mbar_arrive_remote_publish(at_peer(dfull_bar(r)));   // after the ring store
          if (stop) break;
        } else {
          c = read_desc(i);
          release_desc(i);
          if (c < 0) {
            if (c == -2) *abort_flag = 1;
            break;
          }
        }
        const int cnext = leader ? atomicAdd(dy.next, 1) : 0;   // claimed one unit ahead
        const DyChunk d = dy_decode(c, U1, nk1, nk2);
        int e, row0, rows, n0;
        pr_tile_info(tiles, d.phase == 0 ? g1.n_blocks : g2.n_blocks, d.unit, d.phase == 0, e,
                     row0, rows, n0);
        const bool narrow = dy_narrow_block(d, g1);
        // Issue stage `kc` of the unit into slot qq % S: this CTA's half of B (and, unless
        // deferred, its h rows); the bytes count on rank 0's full barrier.
        auto stage_in = [&](int kc, int qq, bool with_a) -> bool {
          const int s = qq % S;
          if (*abort_flag || (qq >= S && !mbar_wait(empty_bar(s), ((qq / S) - 1) & 1))) {
            *abort_flag = 1;
            return false;
          }
          const uint32_t sA = base + s * PR_STAGE_BYTES;
          const uint32_t sB = sA + PR_A_BYTES;
          const uint32_t fb = leader ? full_bar(s) : at_leader(full_bar(s));
          // Rank 0 announces the bytes of both CTAs; on a stage without gathered rows it
          // also arrives for both CTAs' gather warps and for rank 1's forwarder.
          if (d.phase == 0) {
            const uint32_t b_bytes = narrow ? 2 * GM_SLAB_BYTES : 2 * PR_B_BYTES;
            if (leader) {
              if (tiles.a_tma) {
                mbar_arrive_expect_tx(fb, b_bytes + 2 * PR_A_BYTES);
                mbar_arrive_cnt(fb, PG_GATHER_THREADS + 1);
              } else {
                mbar_arrive_expect_tx(fb, b_bytes);
              }
            }
            if (tiles.a_tma) tma_load_2d_pair(sA, &tmX, fb, kc * GM_BK, row0 + half0);
            const CUtensorMap* m = narrow ? (leader ? &tmWg1 : &tmWu1) : (leader ? &tmWg : &tmWu);
            tma_load_4d_pair(sB, m, fb, 0, kc * GM_BK, n0 / 64, e);
          } else {
            if (leader) {
              mbar_arrive_expect_tx(fb, 2 * (PR_A_BYTES + PR_B_BYTES));
              mbar_arrive_cnt(fb, PG_GATHER_THREADS + 1);
            }
            tma_load_4d_pair(sB, &tmWd, fb, 0, kc * GM_BK, n0 / 64 + (leader ? 0 : 2), e);
            if (with_a) tma_load_2d_pair(sA, &tmH, fb, kc * GM_BK, row0 + half0);
          }
          *n_issued = qq + 1;
          return true;
        };
        bool ok = true;
        int kc = d.kb;
        if (d.phase == 1 && !all_h_ready) {
          // GEMM-2 needs this tile's h rows (GEMM-1 units of any pair).  The W_down tiles do
          // not: load them for the first stages, then wait for h, then load its rows.
          const int pre = min(d.ke - d.kb, S);
          for (int t2 = 0; t2 < pre && ok; ++t2) ok = stage_in(d.kb + t2, q + t2, false);
          if (ok) {
            if (!wait_counter_geq(h_ready + d.unit / g2.n_blocks, h_target)) {
              *abort_flag = 1;
              ok = false;
            } else {
              all_h_ready = ld_acquire_gpu(h_ready + n_tiles) >= h_target * n_tiles;
              fence_proxy_async_global();   // TMA reads of h after the generic acquire
              for (int t2 = 0; t2 < pre; ++t2) {
                const int s = (q + t2) % S;
                const uint32_t fb = leader ? full_bar(s) : at_leader(full_bar(s));
                tma_load_2d_pair(base + s * PR_STAGE_BYTES, &tmH, fb, (d.kb + t2) * GM_BK,
                                 row0 + half0);
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
      // Wait until the MMAs have released the last stages this CTA filled: their commits
      // arrive on this CTA's empty barriers, and none may still be in flight at exit.
      if (!*abort_flag) {
        const int qe = *n_issued;
        for (int qq = max(0, qe - S); qq < qe; ++qq)
          if (!mbar_wait(empty_bar(qq % S), (qq / S) & 1)) {
            *abort_flag = 1;
            break;
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (rank 0)
      constexpr uint32_t idesc_full = idesc_bf16_f32(PR_ROWS, BN, false, true);
      constexpr uint32_t idesc_narrow = idesc_bf16_f32(PR_ROWS, BN / 2, false, true);
      int q = 0;
      for (int i = 0;; ++i) {
        const int c = read_desc(i);
        release_desc(i);
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
          const int s = q % S;
          if (!mbar_wait(full_bar(s), (q / S) & 1)) {
            ok = false;
            break;
          }
          *n_consumed = q + 1;
          if (d.phase == 0 && !tiles.a_tma) fence_proxy_async_smem();   // A came by cp.async
          tc_fence_after();
          const uint32_t sA = base + s * PR_STAGE_BYTES;
          const uint32_t sB = sA + PR_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < GM_BK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sA + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sB + kk * 2048, GM_SLAB_BYTES, 1024);
            umma_bf16_pair(dt, adesc, bdesc, idesc, (kc != d.kb || kk != 0) ? 1u : 0u);
          }
          umma_commit_pair(empty_bar(s), 0x3);
        }
        umma_commit_pair(tfull_bar(b), 0x3);
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
    } else if (lane == 0) {
      // ------------------------------------------------ A-rows-landed forwarder (rank 1)
      // q: stage (shared-memory slot q % S); qa: gathered stage (A barrier qa % S)
      int q = 0, qa = 0;
      for (int i = 0;; ++i) {
        const int c = read_desc(i);
        release_desc(i);
        if (c < 0) {
          if (c == -2) *abort_flag = 1;
          break;
        }
        const DyChunk d = dy_decode(c, U1, nk1, nk2);
        if (d.phase == 1 || tiles.a_tma) {
          q += d.ke - d.kb;
          continue;
        }
        bool ok = true;
        for (int kc = d.kb; kc < d.ke; ++kc, ++q, ++qa) {
          const int s = q % S;
          if (!mbar_wait(afull_bar(qa % S), (qa / S) & 1)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();   // the gathered rows, for the pair MMA's reads
          mbar_arrive_remote(at_leader(full_bar(s)));
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp < 6) {
    // -------------------------------------------------------------- epilogue (warps 2-5)
    // Warp w reads TMEM lanes 32 (w % 4) .. +31 of this CTA: rows half0 + 32 (w % 4) + lane.
    const int quad = warp & 3;
    for (int i = 0;; ++i) {
      int c = 0;
      if (lane == 0) c = read_desc(i);
      c = __shfl_sync(0xffffffffu, c, 0);
      __syncwarp();
      if (lane == 0) release_desc(i);
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
      pr_tile_info(tiles, g.n_blocks, d.unit, d.phase == 0, e, row0, rows, n0);
      const int r_local = half0 + quad * 32 + lane;
      const bool row_ok = r_local < rows && r_local < PR_ROWS;
      const uint32_t trow = tmem + b * BN + (static_cast<uint32_t>(quad * 32) << 16);
      if (__any_sync(0xffffffffu, row_ok)) {
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
              pg_store32<EPI_GEGLU, 4>(g.out, g.ldo, row0 + r_local, n0, cc, g.N_total,
                                       reinterpret_cast<const float*>(gv),
                                       reinterpret_cast<const float*>(uv));
            else
              pg_store32<EPI_STORE, 4>(g.out, g.ldo, row0 + r_local, n0, cc, g.N_total,
                                       reinterpret_cast<const float*>(gv),
                                       reinterpret_cast<const float*>(uv));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(tempty_bar(b));
        else
          mbar_arrive_remote(at_leader(tempty_bar(b)));
      }
      if (d.phase == 0) {
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
    // GEMM-1 units: this CTA's <= 128 rows of the pair tile, 16-byte cp.async into the
    // 128-byte-swizzled slot (chunk c of row r at byte 128 r + 16 (c ^ r)); rank 0's complete
    // its full barrier, rank 1's its local A barrier (forwarded by warp 1).  GEMM-2 units,
    // and GEMM-1 units whose A rows come by TMA: nothing (rank 0's TMA thread arrives in
    // their place), but the stage count must follow.
    const int gw = warp - 6, sub = lane >> 3, ch = lane & 7;
    int q = 0, qa = 0;   // stage, gathered stage (rank 1's A barrier qa % S)
    for (int i = 0;; ++i) {
      int c = 0;
      if (lane == 0) c = read_desc(i);
      c = __shfl_sync(0xffffffffu, c, 0);
      __syncwarp();
      if (lane == 0) release_desc(i);
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
      pr_tile_info(tiles, g1.n_blocks, d.unit, true, e, row0, rows, n0);
      if (rows > PR_ROWS) {   // never launched so; stay inside the slots
        raise_error(MOE_DEVERR_BAD_INDEX);
        rows = PR_ROWS;
      }
      const int my_rows = min(GM_BM, max(0, rows - half0));
      // warp 6 copies rows 0 .. 63, warp 7 rows 64 .. 127 of this CTA, four per instruction
      constexpr int NI = GM_BM / 8;
      const __nv_bfloat16* src[NI];
      uint32_t doff[NI];
#pragma unroll
      for (int u = 0; u < NI; ++u) {
        const int r = gw * (GM_BM / 2) + 4 * u + sub;
        src[u] = nullptr;
        if (r < my_rows) {
          const int sr = row0 + half0 + r;
          const int t = tiles.perm ? __ldg(tiles.perm + sr) / tiles.k : sr;
          if (t >= 0 && t < tiles.src_rows)
            src[u] = tiles.src + (size_t)t * tiles.ld + 8 * ch;
          else
            raise_error(MOE_DEVERR_BAD_INDEX);
        }
        doff[u] = static_cast<uint32_t>(r * 128 + ((ch ^ (r & 7)) << 4));
      }
      bool stop = false;
      for (int kc = d.kb; kc < d.ke; ++kc, ++q, ++qa) {
        const int s = q % S;
        bool ok = !*abort_flag && (q < S || mbar_wait(empty_bar(s), ((q / S) - 1) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        const uint32_t sA = base + s * PR_STAGE_BYTES;
#pragma unroll
        for (int u = 0; u < NI; ++u)
          if (src[u] != nullptr) cp_async_16(sA + doff[u], src[u] + kc * GM_BK);
        cp_async_arrive_noinc(leader ? full_bar(s) : afull_bar(qa % S));
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
    if (leader)   // the copies of both CTAs count on rank 0's full barriers
      for (int q = *n_consumed; q < *n_issued; ++q)
        mbar_wait_ns(full_bar(q % S), (q / S) & 1, kDrainLimitNs);
  }
  cluster_sync();   // neither CTA touches the other after this
  tc_fence_after();
  if (warp == 0) tmem_dealloc_pair(tmem, TMEM_COLS);
}

}  // namespace moe
