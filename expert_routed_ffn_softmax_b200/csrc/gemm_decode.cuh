// gemm_decode.cuh -- the expert matmuls for small batches (T <= 16 tokens, so every expert
// holds at most 16 rows): "small-M decode tiles".  Reading the active experts' weights is
// all the work, so the kernel is built to stream them at HBM speed:
//
//   * swapped operands: D^T[f, t] = sum_k W[e][k][f] * X[row0 + t][k].  The weights are the
//     MMA's A operand (M = 128 output features, MN-major slabs of 64 features), the <= 16
//     rows of the expert are B (N = 16, K-major, 32-byte swizzle);
//   * one pipeline stage = 16 K-rows of the expert's weights across ALL its output features
//     (every row contiguous in memory) plus the matching 16 x 16 activation block, so the
//     TMA reads whole weight rows;
//   * one fp32 TMEM accumulator of 16 columns per 128-feature M-tile (gate and up tiles side
//     by side for GEGLU);
//   * the K-steps of all tiles are split into equal ranges over the CTAs; each CTA stores
//     an fp32 partial per (tile, range) and the warp that completes a (tile, row quadrant)
//     last adds the pieces in order and runs the epilogue (GEGLU -> Hbuf, or -> O).
// Roles as in the persistent kernel: warp 0 TMA, warp 1 MMA, warps 2-5 epilogue.  All
// waits are bounded.
#pragma once
#include <cuda.h>
#include "ptx.cuh"
#include "grouped_gemm.cuh"

namespace moe {

constexpr int DG_THREADS = 192;
constexpr int DG_BN = 16;                  // token columns (max rows per expert tile)
constexpr int DG_KS = 16;                  // K rows per stage
constexpr int DG_SLAB = DG_KS * 64 * 2;    // 2 KB: 16 K rows x 64 features
constexpr int DG_BBYTES = DG_BN * DG_KS * 2;   // 512 B activation block
constexpr int DG_MAX_STAGES = 8;
constexpr int DG_SMEM_BUDGET = 200 * 1024;

// Layout of one launch, from the output width N_out and the mode.
struct DecodeShape {
  int mt;        // 128-feature M-tiles per projection
  int nm;        // accumulators (2*mt for GEGLU)
  int nsl;       // 64-feature slabs that hold data, per projection
  int stage;     // bytes per stage (A slabs + B block)
  int stages;
  int tmem_cols;
};

__host__ __device__ inline DecodeShape decode_shape(int N_out, bool geglu) {
  DecodeShape s;
  s.mt = (N_out + 127) / 128;
  s.nm = geglu ? 2 * s.mt : s.mt;
  s.nsl = (N_out + 63) / 64;
  s.stage = s.nm * 2 * DG_SLAB + 1024;   // B block padded to keep stages 1024-aligned
  s.stages = DG_SMEM_BUDGET / s.stage;
  if (s.stages > DG_MAX_STAGES) s.stages = DG_MAX_STAGES;
  int cols = 32;
  while (cols < s.nm * DG_BN) cols *= 2;
  s.tmem_cols = cols;
  return s;
}

__host__ __device__ inline int decode_smem_bytes(int N_out, bool geglu) {
  const DecodeShape s = decode_shape(N_out, geglu);
  return 1024 + s.stages * s.stage + 256;
}

// The kernel supports it when the accumulators fit TMEM and two stages fit shared memory.
__host__ __device__ inline bool decode_shape_ok(int N_out, bool geglu) {
  const DecodeShape s = decode_shape(N_out, geglu);
  return s.nm * DG_BN <= 512 && s.stages >= 2;
}

// Shared-memory descriptor, 32-byte swizzle, K-major (rows of 16 bf16): SBO = 256 B.
__device__ __forceinline__ uint64_t smem_desc_sw32_kmajor(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1) << 16;                       // LBO (unused)
  d |= static_cast<uint64_t>((256u >> 4) & 0x3FFFu) << 32;   // SBO: next 8-row group
  d |= static_cast<uint64_t>(1) << 46;                       // version
  d |= static_cast<uint64_t>(6) << 61;                       // SWIZZLE_32B
  return d;
}

// 32 lanes x 16 consecutive fp32 columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

struct DItem {
  int tile, kb, ke;
};

// Equal ranges of the C = tiles * nk K-steps over Gs = min(G, C) CTAs (each range non-empty,
// so the owners of one tile's steps are consecutive CTAs).
struct DSched {
  long long c, e, C, Gs;
  int nk;
  __device__ void init(int g, int G, int n_tiles, int nk_) {
    nk = nk_;
    C = (long long)n_tiles * nk;
    Gs = C < G ? C : G;
    if (g < Gs) {
      c = (long long)g * C / Gs;
      e = (long long)(g + 1) * C / Gs;
    } else {
      c = e = 0;
    }
  }
  __device__ bool next(DItem& it) {
    if (c >= e) return false;
    it.tile = (int)(c / nk);
    it.kb = (int)(c - (long long)it.tile * nk);
    it.ke = (int)min((long long)nk, it.kb + (e - c));
    c += it.ke - it.kb;
    return true;
  }
  __device__ int owner(long long q) const { return (int)(((q + 1) * Gs - 1) / C); }
  __device__ int slot(int gg, int tile) const {
    const long long first = (long long)gg * C / Gs;
    return (first / nk == tile) ? 2 * gg : 2 * gg + 1;
  }
};

template <int MODE>
__global__ void __launch_bounds__(DG_THREADS, 1)
    grouped_gemm_decode_kernel(const __grid_constant__ CUtensorMap tmX,   // activations, box 16x16
                               const __grid_constant__ CUtensorMap tmW0,  // weights, 16 rows x all slabs
                               const __grid_constant__ CUtensorMap tmW1,  // (up weights for GEGLU)
                               TileList tiles, int K, int N_out, void* __restrict__ out_ptr,
                               int ldo, float* __restrict__ partials,
                               int* __restrict__ counters) {
  constexpr bool GEGLU = MODE == EPI_GEGLU;
  pdl_trigger();
  const DecodeShape sh = decode_shape(N_out, GEGLU);
  const int STAGES = sh.stages;
  const int nk = K / DG_KS;
  const int prow = sh.nm * 128;   // floats per token row of a partial tile

  extern __shared__ uint8_t dsm_raw[];
  const uint32_t raw_addr = smem_u32(dsm_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* dsm = dsm_raw + (base - raw_addr);
  const uint32_t bar_base = base + STAGES * sh.stage;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (DG_MAX_STAGES + s); };
  const uint32_t tfull = bar_base + 8u * (2 * DG_MAX_STAGES);
  const uint32_t tempty = tfull + 8u;
  uint8_t* misc = dsm + STAGES * sh.stage + 8 * (2 * DG_MAX_STAGES + 2);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* n_issued = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* n_consumed = reinterpret_cast<volatile int*>(misc + 12);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Slabs past the output width are never loaded: zero them once in every stage.
  {
    const int proj = GEGLU ? 2 : 1;
    const int zslabs = 2 * sh.mt - sh.nsl;
    for (int s = 0; s < STAGES; ++s)
      for (int pj = 0; pj < proj; ++pj)
        for (int z = 0; z < zslabs; ++z) {
          uint4* p = reinterpret_cast<uint4*>(dsm + s * sh.stage +
                                              (pj * 2 * sh.mt + sh.nsl + z) * DG_SLAB);
          for (int i = tid; i < DG_SLAB / 16; i += blockDim.x) p[i] = make_uint4(0, 0, 0, 0);
        }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 128);
    *abort_flag = 0;
    *n_issued = 0;
    *n_consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW0);
    tma_prefetch_desc(&tmW1);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), sh.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prologue above overlaps the previous kernel; the tile list is its output.
  pdl_wait();
  const int n_tiles =
      (*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT) ? 0 : *tiles.num;

  DSched sch;
  sch.init(blockIdx.x, gridDim.x, n_tiles, nk);
  DItem it;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const uint32_t tx = sh.nsl * (GEGLU ? 2 : 1) * DG_SLAB + DG_BBYTES;
      int q = 0;
      while (!*abort_flag && sch.next(it)) {
        const int e = tiles.expert[it.tile], row0 = tiles.row0[it.tile];
        for (int ks = it.kb; ks < it.ke; ++ks, ++q) {
          const int s = q % STAGES;
          if (q >= STAGES && !mbar_wait(empty_bar(s), ((q / STAGES) - 1) & 1)) {
            *abort_flag = 1;
            break;
          }
          const uint32_t sA = base + s * sh.stage;
          const uint32_t sB = sA + sh.nm * 2 * DG_SLAB;
          mbar_arrive_expect_tx(full_bar(s), tx);
          tma_load_2d(sB, &tmX, full_bar(s), ks * DG_KS, row0);
          // one load per projection: 16 K-rows x all nsl slabs of the expert
          tma_load_4d(sA, &tmW0, full_bar(s), 0, ks * DG_KS, 0, e);
          if (GEGLU) tma_load_4d(sA + 2 * sh.mt * DG_SLAB, &tmW1, full_bar(s), 0, ks * DG_KS, 0, e);
          *n_issued = q + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(128, DG_BN, true, false);
      int q = 0, j = 0;
      while (!*abort_flag && sch.next(it)) {
        if (j >= 1 && !mbar_wait(tempty, (j - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int ks = it.kb; ks < it.ke; ++ks, ++q) {
          const int s = q % STAGES;
          if (!mbar_wait(full_bar(s), (q / STAGES) & 1)) {
            ok = false;
            break;
          }
          *n_consumed = q + 1;
          tc_fence_after();
          const uint32_t sA = base + s * sh.stage;
          const uint64_t bdesc = smem_desc_sw32_kmajor(sA + sh.nm * 2 * DG_SLAB);
          for (int m = 0; m < sh.nm; ++m) {
            const uint64_t adesc = smem_desc_sw128(sA + 2 * m * DG_SLAB, DG_SLAB, 1024);
            umma_bf16(tmem + m * DG_BN, adesc, bdesc, idesc, ks != it.kb ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
        }
        umma_commit(tfull);
        ++j;
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (warps 2-5)
    const int quad = warp & 3;
    const int fl = quad * 32 + lane;   // feature within an M-tile
    int j = 0;
    while (sch.next(it)) {
      bool got = mbar_wait(tfull, j & 1);
      tc_fence_after();
      got = __all_sync(0xffffffffu, got && !*abort_flag);
      if (!got) {
        *abort_flag = 1;
        break;
      }
      const int rows = tiles.rows[it.tile], row0 = tiles.row0[it.tile];
      const int slot = sch.slot(blockIdx.x, it.tile);
      float* pbase = partials + (size_t)slot * DG_BN * prow;
      const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
      for (int m = 0; m < sh.nm; ++m) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(trow + m * DG_BN, v);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < DG_BN; ++t)
          if (t < rows) pbase[(size_t)t * prow + m * 128 + fl] = __uint_as_float(v[t]);
      }
      tc_fence_before();
      mbar_arrive(tempty);
      __threadfence();
      __syncwarp();
      const long long cf = (long long)it.tile * nk, cl = cf + nk - 1;
      const int g_first = sch.owner(cf), n_pieces = sch.owner(cl) - g_first + 1;
      int last = 0;
      if (lane == 0) {
        int* ctr = &counters[it.tile * 4 + quad];
        last = atomicAdd(ctr, 1) == n_pieces - 1;
        if (last) *ctr = 0;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        // (m, t) pairs of this thread, 4 at a time, with the loads of up to 8 pieces each
        // issued before they are added (in piece order)
        const int npair = sh.mt * rows;
        for (int q0 = 0; q0 < npair; q0 += 4) {
          float g[4], u[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) g[a] = u[a] = 0.f;
          for (int p0 = 0; p0 < n_pieces; p0 += 8) {
            float gp[4][8], up[4][8];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const int qq = q0 + a, m = qq / rows, t = qq - m * rows;
#pragma unroll
              for (int b = 0; b < 8; ++b) {
                gp[a][b] = up[a][b] = 0.f;
                if (qq < npair && p0 + b < n_pieces && m * 128 + fl < N_out) {
                  const float* src = partials +
                                     (size_t)sch.slot(g_first + p0 + b, it.tile) * DG_BN * prow +
                                     (size_t)t * prow;
                  gp[a][b] = __ldcg(src + m * 128 + fl);
                  if (GEGLU) up[a][b] = __ldcg(src + (sh.mt + m) * 128 + fl);
                }
              }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
              for (int b = 0; b < 8; ++b)
                if (p0 + b < n_pieces) {
                  g[a] += gp[a][b];
                  u[a] += up[a][b];
                }
          }
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const int qq = q0 + a, m = qq / rows, t = qq - m * rows;
            const int f = m * 128 + fl;
            if (qq < npair && f < N_out) {
              const float o = GEGLU ? gelu_tanh_f(g[a]) * u[a] : g[a];
              static_cast<__nv_bfloat16*>(out_ptr)[(size_t)(row0 + t) * ldo + f] =
                  __float2bfloat16_rn(o);
            }
          }
        }
      }
      ++j;
    }
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
  if (warp == 0) tmem_dealloc(tmem, sh.tmem_cols);
}

}  // namespace moe
