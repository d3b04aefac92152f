// nvfp4_mma.cuh -- the expert FFN with NVFP4 weights and activations on the tensor cores
// (tcgen05.mma kind::mxf4nvf4: E2M1 operands, one E4M3 scale per 16 elements along K,
// fp32 accumulation), for decode batches (every expert tile holds at most 16 rows).
//
// Swapped operands, as in the bf16 decode tiles: the weights are A (M = 128 rows of a
// projection: gate/up features or down columns), the tile's routed rows are B (N = 16).  So
// the whole kernel is a weight stream: per 256-deep K stage, a TMA load of 128 rows x 128
// bytes of codes per projection, one bulk copy of the projection's 2 KB of scale blocks
// (the blocked layout of nvfp4_scale_offset), a TMA load of the 16 activation rows and a
// 256-byte bulk copy of their scale lines per K block (rows 0-15 of that block's scales).  The MMA thread copies each stage's scale blocks into tensor memory
// (tcgen05.cp 32x128b.warpx4: 32 lanes x 16 bytes, repeated in the four lane quarters) and
// issues one MMA per 64-deep K block and projection.
//
// Work units -- (tile, 128 GEMM-1 features: gate and up rows) and (tile, 256 output columns
// of GEMM-2: two 128-row blocks of W_down) -- so that every unit streams two A operands per
// stage into two accumulators -- come from one global counter, every GEMM-1 unit before any
// GEMM-2 unit.  A
// GEMM-1 epilogue applies the tensor scales and GEGLU, quantises h to NVFP4 in groups of 16
// features (16 TMEM lanes) and publishes h_ready[tile]; a GEMM-2 unit waits for its tile's
// count before it loads h.  A GEMM-2 epilogue writes the expert output rows in bf16.
//
// Roles: warp 0 weight producer, warp 6 activation producer, warp 1 MMA issuer, warps 2-5
// epilogue.  Every wait is bounded.
#pragma once
#include <cuda.h>
#include "ptx.cuh"
#include "grouped_gemm.cuh"
#include "gemm_decode.cuh"
#include "nvfp4.cuh"

namespace moe {

constexpr int F4_THREADS = 224;
constexpr int F4_STAGES = 5;
constexpr int F4_BN = 16;                        // token columns = max rows of a tile
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
constexpr int F4_MAX_TILES = 128;                // tiles of a batch: at most min(E, 16 k)
// after the stages: barriers and flags (512 bytes), then the tile table (32 bytes a tile)
constexpr int F4_SMEM = 1024 + F4_STAGES * F4_STAGE + 512 + 32 * F4_MAX_TILES;
// tensor memory: two accumulators of 32 columns (gate 16 | up 16), then one set of scale
// columns per pipeline stage (SFA0, SFA1, SFB: 4 K blocks x 4 columns each), so that a
// stage's copies never overwrite scales that MMAs still in flight read
constexpr uint32_t F4_TMEM_COLS = 512;
constexpr uint32_t F4_SF_SET = 48;
constexpr uint32_t F4_COL_SFA0 = 64, F4_COL_SFA1 = 80, F4_COL_SFB = 96;
static_assert(F4_COL_SFA0 + F4_STAGES * F4_SF_SET <= F4_TMEM_COLS, "scale columns");

struct Fp4Ffn {
  const uint8_t *sfa_g, *sfa_u, *sfa_d;   // blocked weight scales
  const float *ts_g, *ts_u, *ts_d;        // weight tensor scales [E]
  const uint8_t* x_lines;                 // [H/64][Pp][16] scale lines of the sorted x rows
  uint8_t* hq;                            // [P][I/2] codes of h
  uint8_t* h_lines;                       // [I/64][Pp][16] scale lines of h (zero at launch)
  __nv_bfloat16* O;                       // [P][H] expert outputs, sorted rows
  const int32_t *tile_num, *tile_expert, *tile_row0, *tile_rows;
  int* next;                              // unit counter, zero at launch
  int* h_ready;                           // [max tiles] GEMM-1 epilogue warps done, zero at launch
  int H, I, E, Pp;                        // Pp = T k + 16 rows of scale lines
  float sx, sh;                           // activation tensor scales
};

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 ([7,10) and [10,13) = 1), both
// K-major, N >> 3 at [17,23), scale format UE4M3 (bit 23 = 0), M >> 4 at [24,29), scale
// factor ids 0, K = 64.
__host__ __device__ constexpr uint32_t idesc_nvfp4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// 1 in exactly one lane of the converged warp (the same lane at every call), else 0.  As a
// predicate of a tcgen05 or TMA instruction this keeps the instruction on its fast issue
// path; a predicate computed from the lane index does not (measured: several times slower).
__device__ __forceinline__ uint32_t elect_lane() {
  uint32_t e;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(e));
  return e;
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

// Predicated forms: executed by the whole (converged) warp, the instruction issues only in
// lanes whose `p` is non-zero.  A stage's copies and MMAs are issued as one branch-free
// sequence predicated by elect_lane(): a few tens of cycles per instruction, where a branch
// around each instruction costs several times that (measured).
// D[tmem] (+)= (A * scale A) (B * scale B)^T over 64 K elements, E4M3 block scale per 16.
__device__ __forceinline__ void umma_nvfp4_p(uint32_t p, uint32_t d_tmem, uint64_t adesc,
                                             uint64_t bdesc, uint32_t idesc, uint32_t sfa_tmem,
                                             uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, a;\n\t"
      "setp.ne.b32 p, %0, 0;\n\t"
      "setp.ne.b32 a, %5, 0;\n\t"
      "@p tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%1], %2, %3, %4, [%6], [%7], a;"
      "\n\t}" ::"r"(p),
      "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// Shared -> tensor memory: 32 rows of 16 bytes (a 512-byte scale block) into 32 lanes x 4
// columns, repeated in each of the four 32-lane quarters (the layout the MMA reads scales in).
__device__ __forceinline__ void tmem_cp_sf_p(uint32_t p, uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p tcgen05.cp.cta_group::1.32x128b.warpx4 [%1], %2;\n\t}" ::"r"(p),
      "r"(taddr), "l"(sdesc)
      : "memory");
}
__device__ __forceinline__ void umma_commit_p(uint32_t p, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%1];\n\t}" ::"r"(p),
      "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_p(uint32_t p, uint32_t dst, const void* desc,
                                              uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%1], [%2, {%4, %5, %6}], [%3];\n\t}" ::"r"(p),
      "r"(dst), "l"(reinterpret_cast<uint64_t>(desc)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_p(uint32_t p, uint32_t dst, const void* desc,
                                              uint32_t bar, int c0, int c1) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%1], [%2, {%4, %5}], [%3];\n\t}" ::"r"(p),
      "r"(dst), "l"(reinterpret_cast<uint64_t>(desc)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_load_p(uint32_t p, uint32_t dst, const void* src,
                                            uint32_t bytes, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%1], [%2], %3, [%4];"
      "\n\t}" ::"r"(p),
      "r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void mbar_expect_tx_p(uint32_t p, uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %2;\n\t}" ::"r"(p),
      "r"(bar), "r"(bytes)
      : "memory");
}

// A unit: phase 0 = GEMM-1 (tile, 128 features), 1 = GEMM-2 (tile, 256 columns).
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
// codes [P][I/2], same box.  tmXl / tmHl: scale lines [K/64][Pp][16] as (16 bytes, Pp rows,
// K/64), box 16 x 32 x 4: one load is a stage's 4 activation scale blocks (rows 16-31 of a
// block belong to no B row of an N = 16 MMA and are never read).
__global__ void __launch_bounds__(F4_THREADS, 1)
    nvfp4_ffn_kernel(const __grid_constant__ CUtensorMap tmWg,
                     const __grid_constant__ CUtensorMap tmWu,
                     const __grid_constant__ CUtensorMap tmWd,
                     const __grid_constant__ CUtensorMap tmXq,
                     const __grid_constant__ CUtensorMap tmHq,
                     const __grid_constant__ CUtensorMap tmXl,
                     const __grid_constant__ CUtensorMap tmHl, Fp4Ffn a) {
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

  int4* tile_tab = reinterpret_cast<int4*>(fsm + F4_STAGES * F4_STAGE + 512);   // e, row0, rows
  float4* ts_tab = reinterpret_cast<float4*>(tile_tab + F4_MAX_TILES);          // g, u, d scales

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kDescReaders = 1 + 4 + 1;   // MMA warp, 4 epilogue warps, activation warp
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
    tma_prefetch_desc(&tmXl);
    tma_prefetch_desc(&tmHl);
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
  if (n_tiles > F4_MAX_TILES || n_tiles < 0) {   // never produced so (T <= 16)
    if (tid == 0) raise_error(MOE_DEVERR_BAD_INDEX);
    n_tiles = 0;
  }
  // the tile table, once: expert, first sorted row, rows (at most 16), tensor scales
  for (int t = tid; t < n_tiles; t += blockDim.x) {
    int e = a.tile_expert[t], rows = a.tile_rows[t], row0 = a.tile_row0[t];
    if ((unsigned)e >= (unsigned)a.E || rows > F4_BN || rows < 0 || row0 < 0 ||
        row0 + rows > a.Pp - 16) {   // never produced so; keep every access in bounds
      raise_error(MOE_DEVERR_BAD_INDEX);
      e = 0;
      rows = 0;
      row0 = 0;
    }
    tile_tab[t] = make_int4(e, row0, rows, 0);
    ts_tab[t] = make_float4(a.ts_g[e], a.ts_u[e], a.ts_d[e], 0.f);
  }
  __syncthreads();
  const int H = a.H, I = a.I;
  // GEMM-1 units: 128 features (gate rows and up rows); GEMM-2 units: 256 columns (two
  // 128-row blocks of W_down, the second absent past H)
  const int nb1 = (I + 127) / 128, nbh = (H + 127) / 128, nb2 = (nbh + 1) / 2;
  const int U1 = n_tiles * nb1, total = U1 + n_tiles * nb2;
  const int kb1 = H / 64, kb2 = I / 64;   // 64-deep K blocks
  const int h_target = 4 * nb1;           // one release per (GEMM-1 unit, epilogue warp)

  auto read_desc = [&](int i) -> int {
    const int r = i % F4_RING;
    if (!mbar_wait(dfull_bar(r), (i / F4_RING) & 1)) return -2;
    return ring[r];
  };
  if (warp == 0) {
    // -------------------------------------------------------------- weight producer (warp 0)
    // Warp-uniform loop as in the MMA warp: lane 0 waits and claims units, the elected lane
    // issues the copies (predicated).  The next unit is claimed when a unit starts and read
    // when it ends, so the claim's round trip overlaps the unit's issue.  The weights never
    // wait for h: a GEMM-2 unit's W_down streams while warp 6 waits for the tile's h.
    int q = 0;
    int c = 0;
    if (lane == 0) c = atomicAdd(a.next, 1);
    c = __shfl_sync(0xffffffffu, c, 0);
    for (int i = 0;; ++i) {
      const int r = i % F4_RING;
      int ok = 1;
      if (lane == 0 && i >= F4_RING) ok = mbar_wait(dempty_bar(r), ((i / F4_RING) - 1) & 1);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        *abort_flag = 1;
        break;
      }
      const bool stop = *abort_flag || c >= total;
      int cnext = 0;
      if (lane == 0) {
        ring[r] = stop ? -1 : c;
        mbar_arrive(dfull_bar(r));
        if (!stop) cnext = atomicAdd(a.next, 1);   // claimed one unit ahead
      }
      if (__shfl_sync(0xffffffffu, stop ? 1 : 0, 0)) break;
      const F4Unit u = f4_decode(c, U1, nb1, nb2);
      const int e = tile_tab[u.tile].x;
      const bool g1 = u.phase == 0;
      const int kbt = g1 ? kb1 : kb2, nk = (kbt + 3) / 4;
      // the unit's two A operands: rows (row block rA of matrix 0) and (rB of matrix 1)
      const int rA = g1 ? u.rb : 2 * u.rb, rB = g1 ? u.rb : 2 * u.rb + 1;
      const bool two = g1 || rB < nbh;
      const uint8_t* sfa0 = g1 ? a.sfa_g : a.sfa_d;
      const uint8_t* sfa1 = g1 ? a.sfa_u : a.sfa_d;
      const size_t blkA = ((size_t)e * (g1 ? nb1 : nbh) + rA) * kbt;   // first scale blocks
      const size_t blkB = ((size_t)e * (g1 ? nb1 : nbh) + rB) * kbt;
      // Stage kc's weights (A + scales); the stage's byte count includes the activations,
      // which warp 6 loads into the same stage.
      auto weights_in = [&](int kc, int qq) -> bool {
        const int s = qq % F4_STAGES;
        int okw = !*abort_flag;
        if (lane == 0 && okw && qq >= F4_STAGES)
          okw = mbar_wait(empty_bar(s), ((qq / F4_STAGES) - 1) & 1);
        if (!__shfl_sync(0xffffffffu, okw, 0)) {
          *abort_flag = 1;
          return false;
        }
        const int nkb = min(4, kbt - 4 * kc);
        const uint32_t sA = base + s * F4_STAGE, sf_bytes = 512u * nkb;
        const uint32_t lead = elect_lane(), up = lead & (two ? 1u : 0u);
        mbar_expect_tx_p(lead, full_bar(s),
                         (two ? 2 : 1) * (F4_A_BYTES + sf_bytes) + F4_B_BYTES + F4_SF_BYTES);
        tma_load_3d_p(lead, sA, g1 ? &tmWg : &tmWd, full_bar(s), kc * 128, rA * 128, e);
        bulk_load_p(lead, sA + F4_OFF_SFA0, sfa0 + (blkA + 4 * kc) * 512, sf_bytes, full_bar(s));
        tma_load_3d_p(up, sA + F4_OFF_A1, g1 ? &tmWu : &tmWd, full_bar(s), kc * 128, rB * 128, e);
        bulk_load_p(up, sA + F4_OFF_SFA1, sfa1 + (blkB + 4 * kc) * 512, sf_bytes, full_bar(s));
        if (lane == 0) *n_issued = qq + 1;
        __syncwarp();
        return true;
      };
      bool okp = true;
      for (int kc = 0; okp && kc < nk; ++kc, ++q) okp = weights_in(kc, q);
      if (!okp) break;
      c = __shfl_sync(0xffffffffu, cnext, 0);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer (warp 1)
    // The whole warp runs the loop, so descriptors and tensor-memory addresses stay
    // warp-uniform; lane 0 does the waits, the elected lane issues every tcgen05 instruction.
    constexpr uint32_t idesc = idesc_nvfp4(128, F4_BN);
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    // descriptors of stage 0; a stage s, K block jb adds (address offset >> 4) to the start
    // address field (every address stays below 256 KB, so the 14-bit field cannot carry)
    const uint64_t dA0 = smem_desc_sw128(base, 16, 1024);
    const uint64_t dA1 = smem_desc_sw128(base + F4_OFF_A1, 16, 1024);
    const uint64_t dB = smem_desc_sw128(base + F4_OFF_B, 16, 1024);
    const uint64_t dS0 = smem_desc_sf_block(base + F4_OFF_SFA0);
    const uint64_t dS1 = smem_desc_sf_block(base + F4_OFF_SFA1);
    const uint64_t dSB = smem_desc_sf_block(base + F4_OFF_SFB);
    int q = 0;
    for (int i = 0;; ++i) {
      int c = 0;
      if (lane == 0) {
        c = read_desc(i);
        mbar_arrive(dempty_bar(i % F4_RING));
      }
      c = __shfl_sync(0xffffffffu, c, 0);
      if (c < 0) {
        if (c == -2) *abort_flag = 1;
        break;
      }
      const F4Unit u = f4_decode(c, U1, nb1, nb2);
      const bool g1 = u.phase == 0;
      const int kbt = g1 ? kb1 : kb2, nk = (kbt + 3) / 4;
      const int b = i & 1, use = i >> 1;
      int ok = 1;
      if (lane == 0 && use >= 1) ok = mbar_wait(tempty_bar(b), (use - 1) & 1);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d0 = tm + b * 32, d1 = d0 + 16;
      for (int kc = 0; kc < nk; ++kc, ++q) {
        const int s = q % F4_STAGES;
        if (lane == 0) {
          ok = mbar_wait(full_bar(s), (q / F4_STAGES) & 1);
          *n_consumed = q + 1;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const int nkb = min(4, kbt - 4 * kc);
        const uint32_t sA = base + s * F4_STAGE;
        const uint32_t ts = tm + s * F4_SF_SET;   // this stage's scale columns
        // this stage's scales into tensor memory (their columns were last read by the MMAs
        // of stage q - F4_STAGES, which completed before the stage's buffers were refilled)
        const uint32_t lead = elect_lane();
        const bool two = g1 || 2 * u.rb + 1 < nbh;   // second A operand
        const uint64_t so = static_cast<uint64_t>((s * F4_STAGE) >> 4);
        if (nkb == 4 && two) {
          // the common stage: every instruction predicated by the elected lane alone
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            tmem_cp_sf_p(lead, ts + F4_COL_SFA0 + 4 * jb, dS0 + so + 32 * jb);
            tmem_cp_sf_p(lead, ts + F4_COL_SFA1 + 4 * jb, dS1 + so + 32 * jb);
            tmem_cp_sf_p(lead, ts + F4_COL_SFB + 4 * jb, dSB + so + 32 * jb);
          }
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            const uint32_t acc = (kc != 0 || jb != 0) ? 1u : 0u;
            umma_nvfp4_p(lead, d0, dA0 + so + 2 * jb, dB + so + 2 * jb, idesc,
                         ts + F4_COL_SFA0 + 4 * jb, ts + F4_COL_SFB + 4 * jb, acc);
            umma_nvfp4_p(lead, d1, dA1 + so + 2 * jb, dB + so + 2 * jb, idesc,
                         ts + F4_COL_SFA1 + 4 * jb, ts + F4_COL_SFB + 4 * jb, acc);
          }
        } else {
          // a stage with fewer K blocks, or one A operand
          const uint32_t up = lead & (two ? 1u : 0u);
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            const uint32_t v = jb < nkb ? 1u : 0u;
            tmem_cp_sf_p(lead & v, ts + F4_COL_SFA0 + 4 * jb,
                         smem_desc_sf_block(sA + F4_OFF_SFA0 + 512 * jb));
            tmem_cp_sf_p(up & v, ts + F4_COL_SFA1 + 4 * jb,
                         smem_desc_sf_block(sA + F4_OFF_SFA1 + 512 * jb));
            tmem_cp_sf_p(lead & v, ts + F4_COL_SFB + 4 * jb,
                         smem_desc_sf_block(sA + F4_OFF_SFB + 512 * jb));
          }
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            const uint32_t v = jb < nkb ? 1u : 0u;
            const uint64_t bdesc = smem_desc_sw128(sA + F4_OFF_B + 32 * jb, 16, 1024);
            const uint32_t acc = (kc != 0 || jb != 0) ? 1u : 0u;
            umma_nvfp4_p(lead & v, d0, smem_desc_sw128(sA + 32 * jb, 16, 1024), bdesc, idesc,
                         ts + F4_COL_SFA0 + 4 * jb, ts + F4_COL_SFB + 4 * jb, acc);
            umma_nvfp4_p(up & v, d1, smem_desc_sw128(sA + F4_OFF_A1 + 32 * jb, 16, 1024), bdesc,
                         idesc, ts + F4_COL_SFA1 + 4 * jb, ts + F4_COL_SFB + 4 * jb, acc);
          }
        }
        umma_commit_p(lead, empty_bar(s));
      }
      umma_commit_p(elect_lane(), tfull_bar(b));
      if (!ok) {
        *abort_flag = 1;
        break;
      }
    }
    // every MMA and copy issued here (by the elected lane) has completed before the teardown
    umma_commit_p(elect_lane(), done_bar);
    if (lane == 0 && !mbar_wait_ns(done_bar, 0, kDrainLimitNs)) *abort_flag = 1;
    __syncwarp();
  } else if (warp == 6) {
    // -------------------------------------------------------------- activation producer
    // The same units and stages as warp 0: per stage, the tile's 16 activation rows (x's
    // codes for GEMM-1, h's for GEMM-2) and their scale lines, into the stage warp 0 filled
    // or is filling (the stage's byte count, set by warp 0, covers both).  A GEMM-2 unit
    // first waits until every GEMM-1 epilogue warp of its tile has published h.
    int q = 0;
    for (int i = 0;; ++i) {
      int c = 0;
      if (lane == 0) {
        c = read_desc(i);
        mbar_arrive(dempty_bar(i % F4_RING));
      }
      c = __shfl_sync(0xffffffffu, c, 0);
      if (c < 0) {
        if (c == -2) *abort_flag = 1;
        break;
      }
      const F4Unit u = f4_decode(c, U1, nb1, nb2);
      const int row0 = tile_tab[u.tile].y;
      const bool g1 = u.phase == 0;
      const int kbt = g1 ? kb1 : kb2, nk = (kbt + 3) / 4;
      if (!g1) {
        int okh = 1;
        if (lane == 0) okh = wait_counter_geq(a.h_ready + u.tile, h_target);
        // every lane (whichever issues the loads) acquires the count, then orders its
        // async-proxy reads of h after it
        okh = __shfl_sync(0xffffffffu, okh, 0);
        (void)ld_acquire_gpu(a.h_ready + u.tile);
        fence_proxy_async_global();
        if (!okh) {
          *abort_flag = 1;
          break;
        }
      }
      bool ok = true;
      for (int kc = 0; kc < nk; ++kc, ++q) {
        const int s = q % F4_STAGES;
        int okw = !*abort_flag;
        if (lane == 0 && okw && q >= F4_STAGES)
          okw = mbar_wait(empty_bar(s), ((q / F4_STAGES) - 1) & 1);
        if (!__shfl_sync(0xffffffffu, okw, 0)) {
          ok = false;
          break;
        }
        const uint32_t sA = base + s * F4_STAGE;
        const uint32_t lead = elect_lane();
        tma_load_2d_p(lead, sA + F4_OFF_B, g1 ? &tmXq : &tmHq, full_bar(s), kc * 128, row0);
        tma_load_3d_p(lead, sA + F4_OFF_SFB, g1 ? &tmXl : &tmHl, full_bar(s), 0, row0, 4 * kc);
        __syncwarp();
      }
      if (!ok) {
        *abort_flag = 1;
        break;
      }
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
      const int4 tt = tile_tab[u.tile];
      const float4 tsc = ts_tab[u.tile];
      const int row0 = tt.y, rows = tt.z;
      const uint32_t trow = tmem + b * 32 + (static_cast<uint32_t>(quad * 32) << 16);
      // feature (GEMM-1: gate in v0, up in v1) or column (GEMM-2: n in v0, n + 128 in v1)
      const int n = (u.phase == 0 ? u.rb * 128 : u.rb * 256) + quad * 32 + lane;
      uint32_t v0[16], v1[16];
      tmem_ld_32x32b_x16(trow, v0);
      tmem_ld_32x32b_x16(trow + 16, v1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(tempty_bar(b));
      if (u.phase == 0) {
        const float cg = __fmul_rn(a.sx, tsc.x), cu = __fmul_rn(a.sx, tsc.y);
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
              if ((lane & 15) == 0)   // group g = n / 16: line (g / 4, row), byte g % 4
                a.h_lines[((size_t)(n / 64) * a.Pp + row0 + t) * 16 + (n / 16) % 4] =
                    static_cast<uint8_t>(s8);
            }
          }
        }
        // publish this warp's part of the tile's h to the GEMM-2 loads (TMA and generic)
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add_gpu(a.h_ready + u.tile, 1);
      } else {
        const float cd = __fmul_rn(a.sh, tsc.z);
#pragma unroll
        for (int t = 0; t < F4_BN; ++t) {
          if (t < rows) {
            __nv_bfloat16* orow = a.O + (size_t)(row0 + t) * H;
            if (n < H) orow[n] = __float2bfloat16_rn(__uint_as_float(v0[t]) * cd);
            if (n + 128 < H) orow[n + 128] = __float2bfloat16_rn(__uint_as_float(v1[t]) * cd);
          }
        }
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
