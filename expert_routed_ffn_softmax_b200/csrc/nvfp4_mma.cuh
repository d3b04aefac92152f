// nvfp4_mma.cuh -- the expert FFN with NVFP4 weights and activations on the tensor cores
// (tcgen05.mma kind::mxf4nvf4: E2M1 operands, one E4M3 scale per 16 elements along K,
// fp32 accumulation), for decode batches (every expert tile holds at most 16 rows).
//
// Swapped operands, as in the bf16 decode tiles: the weights are A (M = 128 rows of a
// projection: gate/up features or down columns), the tile's routed rows are B (N = 16).  So
// the whole kernel is a weight stream: per 256-deep K stage, a TMA load of 128 rows x 128
// bytes of codes per projection, one bulk copy of the projection's 2 KB of scale blocks
// (the blocked layout of nvfp4_scale_offset), a TMA load of the 16 activation rows and their
// scale lines.  The MMA thread copies each stage's scale blocks into tensor memory
// (tcgen05.cp 32x128b.warpx4: 32 lanes x 16 bytes, repeated in the four lane quarters) and
// issues one MMA per 64-deep K block and projection.
//
// Work units -- (tile, 128 GEMM-1 features: gate and up) and (tile, 128 output columns of
// GEMM-2) -- come from one global counter, every GEMM-1 unit before any GEMM-2 unit.  A
// GEMM-1 epilogue applies the tensor scales and GEGLU, quantises h to NVFP4 in groups of 16
// features (16 TMEM lanes) and publishes h_ready[tile]; a GEMM-2 unit waits for its tile's
// count before it loads h.  A GEMM-2 epilogue writes the expert output rows in bf16.
//
// Roles: warp 0 producer (lane 0 issues; lanes 0-15 write the activation scale lines),
// warp 1 MMA issuer, warps 2-5 epilogue.  Every wait is bounded.
#pragma once
#include <cuda.h>
#include "ptx.cuh"
#include "grouped_gemm.cuh"
#include "gemm_decode.cuh"
#include "nvfp4.cuh"

namespace moe {

constexpr int F4_THREADS = 192;
constexpr int F4_STAGES = 5;
constexpr int F4_BN = 16;                        // token columns = max rows of a tile
constexpr int F4_KS = 256;                       // K elements per stage (128 bytes per row)
constexpr int F4_A_BYTES = 128 * 128;            // one projection's codes per stage
constexpr int F4_SF_BYTES = 4 * 512;             // 4 scale blocks (4 K blocks of 64)
constexpr int F4_B_BYTES = F4_BN * 128;          // activation codes per stage
// stage: A0 | A1 | SFA0 | SFA1 | B | SFB  (A and B 1024-aligned for the 128-byte swizzle)
constexpr int F4_OFF_A1 = F4_A_BYTES;
constexpr int F4_OFF_SFA0 = 2 * F4_A_BYTES;
constexpr int F4_OFF_SFA1 = F4_OFF_SFA0 + F4_SF_BYTES;
constexpr int F4_OFF_B = F4_OFF_SFA1 + F4_SF_BYTES;
constexpr int F4_OFF_SFB = F4_OFF_B + F4_B_BYTES;
constexpr int F4_STAGE = F4_OFF_SFB + F4_SF_BYTES;   // 40 KB
constexpr int F4_RING = 8;
constexpr int F4_SMEM = 1024 + F4_STAGES * F4_STAGE + 1024;
// tensor memory: two accumulators of 32 columns (gate 16 | up 16), then the scale columns
// of one stage: SFA0, SFA1, SFB (4 K blocks x 4 columns each)
constexpr uint32_t F4_TMEM_COLS = 128;
constexpr uint32_t F4_COL_SFA0 = 64, F4_COL_SFA1 = 80, F4_COL_SFB = 96;

struct Fp4Ffn {
  const uint8_t *sfa_g, *sfa_u, *sfa_d;   // blocked weight scales
  const float *ts_g, *ts_u, *ts_d;        // weight tensor scales [E]
  const uint8_t* xsf;                     // [P][H/16] scales of the sorted x rows
  uint8_t* hq;                            // [P][I/2] codes of h
  uint8_t* hsf;                           // [P][I/16] scales of h
  __nv_bfloat16* O;                       // [P][H] expert outputs, sorted rows
  const int32_t *tile_num, *tile_expert, *tile_row0, *tile_rows;
  int* next;                              // unit counter, zero at launch
  int* h_ready;                           // [max tiles] GEMM-1 epilogue warps done, zero at launch
  int H, I;
  float sx, sh;                           // activation tensor scales
};

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 ([7,10) and [10,13) = 1), both
// K-major, N >> 3 at [17,23), scale format UE4M3 (bit 23 = 0), M >> 4 at [24,29), scale
// factor ids 0, K = 64.
__host__ __device__ constexpr uint32_t idesc_nvfp4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= (A * scale A) (B * scale B)^T over 64 K elements, block scale per 16.
__device__ __forceinline__ void umma_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared -> tensor memory: 32 rows of 16 bytes (a 512-byte scale block) into 32 lanes x 4
// columns, repeated in each of the four 32-lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Descriptor of a 512-byte block read as 32 rows of 16 bytes (no swizzle, K-major): core
// matrices of 8 rows x 16 bytes, 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sf_block(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// A unit: phase 0 = GEMM-1 (tile, 128 features), 1 = GEMM-2 (tile, 128 columns).
struct F4Unit {
  int phase, tile, rb;
};
__device__ __forceinline__ F4Unit f4_decode(int c, int U1, int nb1, int nb2) {
  F4Unit u;
  u.phase = c < U1 ? 0 : 1;
  const int v = c < U1 ? c : c - U1;
  const int nb = c < U1 ? nb1 : nb2;
  u.tile = v / nb;
  u.rb = v - u.tile * nb;
  return u;
}

// tmWg / tmWu: codes [E][I][H/2] as (H/2 bytes, I rows, E), box 128 x 128 x 1.  tmWd: codes
// [E][H][I/2], same box.  tmXq: sorted x codes [P][H/2], box 128 bytes x 16 rows.  tmHq: h
// codes [P][I/2], same box.
__global__ void __launch_bounds__(F4_THREADS, 1)
    nvfp4_ffn_kernel(const __grid_constant__ CUtensorMap tmWg,
                     const __grid_constant__ CUtensorMap tmWu,
                     const __grid_constant__ CUtensorMap tmWd,
                     const __grid_constant__ CUtensorMap tmXq,
                     const __grid_constant__ CUtensorMap tmHq, Fp4Ffn a) {
  pdl_trigger();
  extern __shared__ uint8_t fsm_raw[];
  const uint32_t raw_addr = smem_u32(fsm_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* fsm = fsm_raw + (base - raw_addr);
  const uint32_t bar_base = base + F4_STAGES * F4_STAGE;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (F4_STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * F4_STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * F4_STAGES + 2 + b); };
  auto dfull_bar = [&](int r) { return bar_base + 8u * (2 * F4_STAGES + 4 + r); };
  auto dempty_bar = [&](int r) { return bar_base + 8u * (2 * F4_STAGES + 4 + F4_RING + r); };
  const uint32_t done_bar = bar_base + 8u * (2 * F4_STAGES + 4 + 2 * F4_RING);
  uint8_t* misc = fsm + F4_STAGES * F4_STAGE + 8 * (2 * F4_STAGES + 5 + 2 * F4_RING);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* n_issued = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* n_consumed = reinterpret_cast<volatile int*>(misc + 12);
  volatile int* ring = reinterpret_cast<volatile int*>(misc + 16);   // [F4_RING] unit ids

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kDescReaders = 1 + 4;   // MMA thread, 4 epilogue warps
  // The activation scale lines (rows 0-15, 4 bytes each) are rewritten every stage; the
  // rest of every SFB block stays zero (the rows >= 16 of the 128-row scale layout).
  for (int s = 0; s < F4_STAGES; ++s) {
    uint4* p = reinterpret_cast<uint4*>(fsm + s * F4_STAGE + F4_OFF_SFB);
    for (int i = tid; i < F4_SF_BYTES / 16; i += blockDim.x) p[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    for (int s = 0; s < F4_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 128);
    }
    for (int r = 0; r < F4_RING; ++r) {
      mbar_init(dfull_bar(r), 1);
      mbar_init(dempty_bar(r), kDescReaders);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *n_issued = 0;
    *n_consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmWg);
    tma_prefetch_desc(&tmWu);
    tma_prefetch_desc(&tmWd);
    tma_prefetch_desc(&tmXq);
    tma_prefetch_desc(&tmHq);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), F4_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();   // tile list, sorted x codes and zeroed counters come from earlier kernels
  int n_tiles = 0;
  if (!(*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT))
    n_tiles = *a.tile_num;
  const int H = a.H, I = a.I;
  const int nb1 = (I + 127) / 128, nb2 = (H + 127) / 128;
  const int U1 = n_tiles * nb1, total = U1 + n_tiles * nb2;
  const int kb1 = H / 64, kb2 = I / 64;   // 64-deep K blocks
  const int h_target = 4 * nb1;           // one release per (GEMM-1 unit, epilogue warp)

  auto read_desc = [&](int i) -> int {
    const int r = i % F4_RING;
    if (!mbar_wait(dfull_bar(r), (i / F4_RING) & 1)) return -2;
    return ring[r];
  };
  auto tile_rows = [&](int tile) {
    int rows = a.tile_rows[tile];
    if (rows > F4_BN || rows < 0) {   // never produced so; keep every access in bounds
      raise_error(MOE_DEVERR_BAD_INDEX);
      rows = rows < 0 ? 0 : F4_BN;
    }
    return rows;
  };

  if (warp == 0) {
    // -------------------------------------------------------------- producer (warp 0)
    int q = 0;
    int c = 0;
    if (lane == 0) c = atomicAdd(a.next, 1);
    c = __shfl_sync(0xffffffffu, c, 0);
    for (int i = 0;; ++i) {
      const int r = i % F4_RING;
      int ok = 1;
      if (lane == 0 && i >= F4_RING) ok = mbar_wait(dempty_bar(r), ((i / F4_RING) - 1) & 1);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      const bool stop = *abort_flag || c >= total;
      if (lane == 0) {
        ring[r] = stop ? -1 : c;
        mbar_arrive(dfull_bar(r));
      }
      if (stop) break;
      int cnext = 0;
      if (lane == 0) cnext = atomicAdd(a.next, 1);   // claimed one unit ahead
      cnext = __shfl_sync(0xffffffffu, cnext, 0);
      const F4Unit u = f4_decode(c, U1, nb1, nb2);
      const int e = a.tile_expert[u.tile], row0 = a.tile_row0[u.tile];
      const int rows = tile_rows(u.tile);
      const bool g1 = u.phase == 0;
      const int kbt = g1 ? kb1 : kb2, nk = (kbt + 3) / 4;
      const int ldsf = (g1 ? H : I) / 16;   // activation scale bytes per row
      const uint8_t* act_sf = g1 ? a.xsf : a.hsf;
      if (!g1) {
        // this tile's h: every GEMM-1 epilogue warp of its units has published
        if (lane == 0) {
          ok = wait_counter_geq(a.h_ready + u.tile, h_target);
          fence_proxy_async_global();   // TMA reads of h after the generic acquire
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
      const uint8_t* sfa0 = g1 ? a.sfa_g : a.sfa_d;
      const size_t blk0 = ((size_t)e * (g1 ? nb1 : nb2) + u.rb) * kbt;   // first scale block
      bool stopped = false;
      for (int kc = 0; kc < nk; ++kc, ++q) {
        const int s = q % F4_STAGES;
        ok = 1;
        if (lane == 0 && q >= F4_STAGES) ok = mbar_wait(empty_bar(s), ((q / F4_STAGES) - 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok || *abort_flag) {
          *abort_flag = 1;
          stopped = true;
          break;
        }
        const int nkb = min(4, kbt - 4 * kc);
        const uint32_t sA = base + s * F4_STAGE;
        // activation scale lines: row `lane`, K blocks 4 kc .. 4 kc + nkb - 1 (4 bytes each)
        if (lane < F4_BN) {
          uint8_t* sfb = fsm + s * F4_STAGE + F4_OFF_SFB + 16 * lane;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t v = 0;
            if (lane < rows && j < nkb)
              v = __ldcg(reinterpret_cast<const unsigned int*>(act_sf + (size_t)(row0 + lane) * ldsf +
                                                               16 * kc + 4 * j));
            *reinterpret_cast<uint32_t*>(sfb + 512 * j) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const uint32_t sf_bytes = 512u * nkb;
          mbar_arrive_expect_tx(full_bar(s), (g1 ? 2 : 1) * (F4_A_BYTES + sf_bytes) + F4_B_BYTES);
          tma_load_3d(sA, g1 ? &tmWg : &tmWd, full_bar(s), kc * 128, u.rb * 128, e);
          bulk_load(sA + F4_OFF_SFA0, sfa0 + (blk0 + 4 * kc) * 512, sf_bytes, full_bar(s));
          if (g1) {
            tma_load_3d(sA + F4_OFF_A1, &tmWu, full_bar(s), kc * 128, u.rb * 128, e);
            bulk_load(sA + F4_OFF_SFA1, a.sfa_u + (blk0 + 4 * kc) * 512, sf_bytes, full_bar(s));
          }
          tma_load_2d(sA + F4_OFF_B, g1 ? &tmXq : &tmHq, full_bar(s), kc * 128, row0);
          *n_issued = q + 1;
        }
      }
      if (stopped) break;
      c = cnext;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_nvfp4(128, F4_BN);
      int q = 0;
      for (int i = 0;; ++i) {
        const int c = read_desc(i);
        mbar_arrive(dempty_bar(i % F4_RING));
        if (c < 0) {
          if (c == -2) *abort_flag = 1;
          break;
        }
        const F4Unit u = f4_decode(c, U1, nb1, nb2);
        const bool g1 = u.phase == 0;
        const int kbt = g1 ? kb1 : kb2, nk = (kbt + 3) / 4;
        const int b = i & 1, use = i >> 1;
        if (use >= 1 && !mbar_wait(tempty_bar(b), (use - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem + b * 32, d1 = d0 + 16;
        bool ok = true;
        for (int kc = 0; kc < nk; ++kc, ++q) {
          const int s = q % F4_STAGES;
          if (!mbar_wait(full_bar(s), (q / F4_STAGES) & 1)) {
            ok = false;
            break;
          }
          *n_consumed = q + 1;
          tc_fence_after();
          const int nkb = min(4, kbt - 4 * kc);
          const uint32_t sA = base + s * F4_STAGE;
          // this stage's scales into tensor memory (ordered before the MMAs below, after the
          // previous stage's MMAs that read the same columns)
          for (int j = 0; j < nkb; ++j) {
            tmem_cp_32x128b_warpx4(tmem + F4_COL_SFA0 + 4 * j, smem_desc_sf_block(sA + F4_OFF_SFA0 + 512 * j));
            if (g1)
              tmem_cp_32x128b_warpx4(tmem + F4_COL_SFA1 + 4 * j,
                                     smem_desc_sf_block(sA + F4_OFF_SFA1 + 512 * j));
            tmem_cp_32x128b_warpx4(tmem + F4_COL_SFB + 4 * j, smem_desc_sf_block(sA + F4_OFF_SFB + 512 * j));
          }
          for (int j = 0; j < nkb; ++j) {
            const uint64_t bdesc = smem_desc_sw128(sA + F4_OFF_B + 32 * j, 16, 1024);
            const uint32_t acc = (kc != 0 || j != 0) ? 1u : 0u;
            umma_nvfp4(d0, smem_desc_sw128(sA + 32 * j, 16, 1024), bdesc, idesc,
                       tmem + F4_COL_SFA0 + 4 * j, tmem + F4_COL_SFB + 4 * j, acc);
            if (g1)
              umma_nvfp4(d1, smem_desc_sw128(sA + F4_OFF_A1 + 32 * j, 16, 1024), bdesc, idesc,
                         tmem + F4_COL_SFA1 + 4 * j, tmem + F4_COL_SFB + 4 * j, acc);
          }
          umma_commit(empty_bar(s));
        }
        umma_commit(tfull_bar(b));
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
      // every MMA and copy this thread issued has completed before the teardown
      umma_commit(done_bar);
      if (!mbar_wait_ns(done_bar, 0, kDrainLimitNs)) *abort_flag = 1;
    }
  } else {
    // -------------------------------------------------------------- epilogue (warps 2-5)
    const int quad = warp & 3;
    for (int i = 0;; ++i) {
      int c = 0;
      if (lane == 0) c = read_desc(i);
      c = __shfl_sync(0xffffffffu, c, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty_bar(i % F4_RING));
      if (c < 0) {
        if (c == -2) *abort_flag = 1;
        break;
      }
      const F4Unit u = f4_decode(c, U1, nb1, nb2);
      const int b = i & 1, use = i >> 1;
      bool got = mbar_wait(tfull_bar(b), use & 1);
      tc_fence_after();
      got = __all_sync(0xffffffffu, got && !*abort_flag);
      if (!got) {
        *abort_flag = 1;
        break;
      }
      const int e = a.tile_expert[u.tile], row0 = a.tile_row0[u.tile];
      const int rows = tile_rows(u.tile);
      const uint32_t trow = tmem + b * 32 + (static_cast<uint32_t>(quad * 32) << 16);
      const int n = u.rb * 128 + quad * 32 + lane;   // feature (GEMM-1) or column (GEMM-2)
      uint32_t v0[16], v1[16];
      tmem_ld_32x32b_x16(trow, v0);
      if (u.phase == 0) tmem_ld_32x32b_x16(trow + 16, v1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(tempty_bar(b));
      if (u.phase == 0) {
        const float cg = __fmul_rn(a.sx, a.ts_g[e]), cu = __fmul_rn(a.sx, a.ts_u[e]);
        const float sh = a.sh;
#pragma unroll
        for (int t = 0; t < F4_BN; ++t) {
          if (t < rows) {   // uniform across the warp
            const float hv = n < I ? gelu_tanh_f(__uint_as_float(v0[t]) * cg) *
                                         (__uint_as_float(v1[t]) * cu)
                                   : 0.f;
            // NVFP4 of h over 16 consecutive features = 16 lanes
            float amax = fabsf(hv);
#pragma unroll
            for (int off = 1; off < 16; off <<= 1)
              amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float s = __fdiv_rn(__fdiv_rn(amax, 6.0f), sh);
            const uint32_t s8 = e4m3_round_sat(s);
            const float S = __fmul_rn(e4m3_to_f32(s8), sh);
            const uint32_t code = S == 0.f ? 0u : (e2m1x2_round_sat(__fdiv_rn(hv, S), 0.f) & 15u);
            const uint32_t nb = __shfl_down_sync(0xffffffffu, code, 1);
            if (n < I) {
              if ((lane & 1) == 0)
                a.hq[(size_t)(row0 + t) * (I / 2) + n / 2] = static_cast<uint8_t>(code | (nb << 4));
              if ((lane & 15) == 0)
                a.hsf[(size_t)(row0 + t) * (I / 16) + n / 16] = static_cast<uint8_t>(s8);
            }
          }
        }
        // publish this warp's part of the tile's h to the GEMM-2 loads (TMA and generic)
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add_gpu(a.h_ready + u.tile, 1);
      } else {
        const float cd = __fmul_rn(a.sh, a.ts_d[e]);
#pragma unroll
        for (int t = 0; t < F4_BN; ++t)
          if (t < rows && n < H)
            a.O[(size_t)(row0 + t) * H + n] = __float2bfloat16_rn(__uint_as_float(v0[t]) * cd);
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    raise_error(MOE_DEVERR_TIMEOUT);
    for (int qq = *n_consumed; qq < *n_issued; ++qq)
      mbar_wait_ns(full_bar(qq % F4_STAGES), (qq / F4_STAGES) & 1, kDrainLimitNs);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, F4_TMEM_COLS);
}

}  // namespace moe
