// grouped_gemm.cuh -- the expert FFN as grouped matmuls on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM, operands staged in shared memory by TMA).  This is
// the role SwiftGMM plays on Ascend ("MoE推理「王炸」组合：昇腾×盘古让推理性能狂飙6-8倍",
// Group 4), rebuilt for sm_100a.
//
//   GEMM-1 (EPI_GEGLU):  for each expert tile, D = Xp[rows, :] x [W_gate | W_up][e][:, f0:f0+128]
//            one MMA of N = 256 covers 128 gate columns and the same 128 up columns, so the
//            epilogue holds g and u of a feature in the same thread and writes
//            h = gelu_tanh(g) * u  (GEGLU, optimisation report §1; gelu_pytorch_tanh,
//            verification report §2.1) as bf16.
//   GEMM-2 (EPI_STORE):  O[rows, n0:n0+256] = Hbuf[rows, :] x W_down[e][:, n0:n0+256], bf16.
//
// Tile: 128 rows (sorted pairs of one expert) x 256 MMA columns, K staged 64 at a time
// (one 128-byte swizzle row of bf16).  A (activations) is K-major; B (weights, stored
// [K][N] with N contiguous) is MN-major, loaded as 64-column slabs.  Rows past the end of
// the expert's segment are computed and not stored; slabs past N are zero-filled by TMA.
//
// Roles (128 threads): warp 0 allocates TMEM and its lane 0 issues TMA; warp 1 lane 0
// issues the MMAs; all four warps run the epilogue, warp w reading TMEM lanes 32w..32w+31.
// Every mbarrier wait is bounded; on a failure the CTA drains the copies it issued, frees
// its TMEM and returns, and the host sees MOE_ERR_TIMEOUT from moe_sync_status().
#pragma once
#include <cuda.h>
#include "ptx.cuh"

namespace moe {

constexpr int GM_BM = 128;
constexpr int GM_BK = 64;
constexpr int GM_A_BYTES = GM_BM * GM_BK * 2;          // 16 KB
constexpr int GM_SLAB_BYTES = GM_BK * 64 * 2;          // 8 KB: 64 K rows x 64 columns

// EPI_GEGLU: B = [gate | up] slabs, h = gelu_tanh(g) * u stored bf16 (N/2 columns out)
// EPI_STORE: bf16 store of all N columns;  EPI_F32: fp32 store of all N columns.
enum { EPI_GEGLU = 0, EPI_STORE = 1, EPI_F32 = 2 };

struct TileList {
  const int32_t* num;     // [1] tiles in use
  const int32_t* expert;  // [cap]
  const int32_t* row0;    // [cap] first sorted row
  const int32_t* rows;    // [cap] rows in tile (1..128)
  int uniform_rows;       // > 0: no list; tile m covers rows [128m, min(128m+128, uniform_rows)) of expert 0
  // Gathering GEMMs: sorted row r of the A operand is row perm[r] / k of src (row stride ld
  // elements), i.e. x[t] for the pair (t, j) = divmod(perm[r], k).
  const int32_t* perm = nullptr;
  int k = 1;
  const __nv_bfloat16* src = nullptr;
  int ld = 0;         // row stride of src (elements; a multiple of 8)
  int src_rows = 0;   // rows of src
  // 1: the A rows of GEMM-1 are rows row0.. of a contiguous row-major tensor (the tile's rows
  // already in sorted order), loaded by TMA like GEMM-2's h rows; the gather warps idle.
  int a_tma = 0;
};

template <int NSLAB>
__host__ __device__ constexpr int gemm_stage_bytes() {
  return GM_A_BYTES + NSLAB * GM_SLAB_BYTES;
}
template <int STAGES, int NSLAB>
__host__ __device__ constexpr int gemm_smem_bytes() {
  return 1024 /*alignment slack*/ + STAGES * gemm_stage_bytes<NSLAB>() + 256 /*barriers*/;
}

__device__ __forceinline__ float gelu_tanh_f(float g) {
  const float inner = 0.7978845608028654f * fmaf(0.044715f * g, g * g, g);
  return 0.5f * g * (1.0f + tanh_approx(inner));
}

template <int STAGES, int MODE, int NSLAB>
__global__ void __launch_bounds__(128, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, TileList tiles, int n_blocks,
                        int K, int N_total, void* __restrict__ out_ptr, int ldo) {
  pdl_trigger();
  pdl_wait();
  constexpr int BN = 64 * NSLAB;                       // MMA N
  constexpr int STAGE_BYTES = gemm_stage_bytes<NSLAB>();
  constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  static_assert(MODE != EPI_GEGLU || NSLAB % 2 == 0, "GEGLU pairs gate and up slabs");
  // 1-D grid: n_blocks column blocks per row tile, column block fastest so that the CTAs
  // sharing one activation tile run together.
  const int tile = blockIdx.x / n_blocks;
  const int nb = blockIdx.x - tile * n_blocks;
  int e, row0, rows;
  if (tiles.uniform_rows > 0) {
    if (tile * GM_BM >= tiles.uniform_rows) return;
    e = 0;
    row0 = tile * GM_BM;
    rows = min(GM_BM, tiles.uniform_rows - row0);
  } else {
    if (tile >= *tiles.num) return;
    e = tiles.expert[tile];
    row0 = tiles.row0[tile];
    rows = tiles.rows[tile];
  }
  // After a device-side timeout anywhere, skip the work until the host clears the word.
  if (*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT) return;
  // GEGLU: BN/2 output features per CTA; otherwise BN output columns per CTA.
  const int n0 = nb * (MODE == EPI_GEGLU ? BN / 2 : BN);

  extern __shared__ uint8_t gsm_raw[];
  const uint32_t raw_addr = smem_u32(gsm_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* gsm = gsm_raw + (base - raw_addr);
  const uint32_t bar_base = base + STAGES * STAGE_BYTES;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  const uint32_t done_bar = bar_base + 8u * (2 * STAGES);
  volatile uint32_t* tmem_slot =
      reinterpret_cast<volatile uint32_t*>(gsm + STAGES * STAGE_BYTES + 8 * (2 * STAGES + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(
      gsm + STAGES * STAGE_BYTES + 8 * (2 * STAGES + 1) + 4);
  volatile int* n_issued = abort_flag + 1;
  volatile int* n_consumed = abort_flag + 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *n_issued = 0;
    *n_consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // K may be split over gridDim.y CTAs (EPI_F32 only): this CTA sums k-blocks [kb0, kb1)
  // and stores its partial tile in slice blockIdx.y of the output
  const int nk_all = K / GM_BK;
  const int kb0 = (int)((long long)nk_all * blockIdx.y / gridDim.y);
  const int nk = (int)((long long)nk_all * (blockIdx.y + 1) / gridDim.y) - kb0;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int kc = 0;
    for (; kc < nk; ++kc) {
      const int s = kc % STAGES;
      if (kc >= STAGES && !mbar_wait(empty_bar(s), ((kc / STAGES) - 1) & 1)) {
        *abort_flag = 1;
        break;
      }
      if (*abort_flag) break;
      const uint32_t sA = base + s * STAGE_BYTES;
      const uint32_t sB = sA + GM_A_BYTES;
      mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES);
      const int kx = (kb0 + kc) * GM_BK;
      tma_load_2d(sA, &tmA, full_bar(s), kx, row0);
      if (MODE == EPI_GEGLU) {
#pragma unroll
        for (int j = 0; j < NSLAB / 2; ++j) {
          tma_load_3d(sB + j * GM_SLAB_BYTES, &tmB0, full_bar(s), n0 + 64 * j, kx, e);
          tma_load_3d(sB + (NSLAB / 2 + j) * GM_SLAB_BYTES, &tmB1, full_bar(s), n0 + 64 * j,
                      kx, e);
        }
      } else {
#pragma unroll
        for (int j = 0; j < NSLAB; ++j)
          tma_load_3d(sB + j * GM_SLAB_BYTES, &tmB0, full_bar(s), n0 + 64 * j, kx, e);
      }
      *n_issued = kc + 1;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(GM_BM, BN, false, true);
    int kc = 0;
    for (; kc < nk; ++kc) {
      const int s = kc % STAGES;
      if (!mbar_wait(full_bar(s), (kc / STAGES) & 1)) {
        *abort_flag = 1;
        break;
      }
      *n_consumed = kc + 1;
      tc_fence_after();
      const uint32_t sA = base + s * STAGE_BYTES;
      const uint32_t sB = sA + GM_A_BYTES;
#pragma unroll
      for (int kk = 0; kk < GM_BK / 16; ++kk) {
        const uint64_t adesc = smem_desc_sw128(sA + kk * 32, 16, 1024);
        const uint64_t bdesc = smem_desc_sw128(sB + kk * 2048, GM_SLAB_BYTES, 1024);
        umma_bf16(tmem, adesc, bdesc, idesc, (kc | kk) != 0 ? 1u : 0u);
      }
      umma_commit(empty_bar(s));
    }
    umma_commit(done_bar);
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  const bool done_ok = mbar_wait(done_bar, 0);
  tc_fence_after();
  const bool store = done_ok && (*abort_flag == 0);
  const int r = warp * 32 + lane;
  const bool row_ok = store && r < rows;
  const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  if (MODE == EPI_GEGLU) {
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(out_ptr) + (size_t)(row0 + r) * ldo;
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 32) {
      uint32_t g[32], u[32];
      tmem_ld_32x32b_x32(trow + c, g);
      tmem_ld_32x32b_x32(trow + BN / 2 + c, u);
      tmem_ld_wait();
      if (row_ok && n0 + c < N_total) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float h0 = gelu_tanh_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
          const float h1 =
              gelu_tanh_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
          pk[i] = pack_bf16x2(h0, h1);
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + n0 + c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
  } else if (MODE == EPI_STORE) {
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(out_ptr) + (size_t)(row0 + r) * ldo;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(trow + c, v);
      tmem_ld_wait();
      if (row_ok && n0 + c < N_total) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        uint4* dst = reinterpret_cast<uint4*>(orow + n0 + c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
  } else {
    float* orow = static_cast<float*>(out_ptr) +
                  ((size_t)blockIdx.y * tiles.uniform_rows + row0 + r) * ldo;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(trow + c, v);
      tmem_ld_wait();
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (n0 + c + 4 * i < N_total)
            reinterpret_cast<uint4*>(orow + n0 + c)[i] =
                make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    // Copies issued but never consumed must land before this CTA's smem is released.
    for (int c = *n_consumed; c < *n_issued; ++c)
      mbar_wait_ns(full_bar(c % STAGES), (c / STAGES) & 1, kDrainLimitNs);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace moe
