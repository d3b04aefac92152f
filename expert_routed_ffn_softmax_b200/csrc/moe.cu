// moe.cu -- the C ABI of include/moe.h: argument checks, workspace layout, TMA tensor
// maps and the launch sequence router -> dispatch -> GEMM-1 (+GEGLU) -> GEMM-2 -> combine.
// All kernels live in this one translation unit so that they share the device error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "moe.h"
#include "ptx.cuh"
#include "router.cuh"
#include "dispatch.cuh"
#include "grouped_gemm.cuh"
#include "gemm_persistent.cuh"
#include "ffn_dynamic.cuh"
#include "ffn_pair.cuh"
#include "decode_front.cuh"
#include "gemm_decode.cuh"
#include "nvfp4.cuh"
#include "nvfp4_mma.cuh"

namespace moe {
namespace {

constexpr int kGemmStages = 4;
constexpr int kMaxDevices = 64;
constexpr int kScreenMinTokens = 256;            // default router path switch
constexpr int kMaxGemmCtas = 256;                // >= SMs per GPU (148 on B200)
constexpr int kStreamKCounters = 4 * 2 * kMaxGemmCtas;   // per GEMM: 4 per split unit
constexpr int kFrontSmemMax = 200 * 1024;        // decode front kernel's dynamic smem cap

constexpr double kScreenC = 1.0 / 1024.0;        // screen error bound / (|x| |w|)
constexpr int kRouterStats = 5;                  // words of moe_aux_t::router_stats
constexpr int kFusedDispatchMaxChunks = 32;      // one-launch dispatch up to this many chunks
constexpr unsigned kKnownFlags = MOE_FLAG_NO_RENORM | MOE_FLAG_ROUTER_FP64 |
                                 MOE_FLAG_ROUTER_SCREEN | MOE_FLAG_PROFILE_STAGES |
                                 MOE_FLAG_DECODE_TILES | MOE_FLAG_PREFILL_TILES |
                                 MOE_FLAG_UNFUSED_FFN | MOE_FLAG_FUSED_FFN |
                                 MOE_FLAG_FFN_PAIRS | MOE_FLAG_FFN_SINGLE |
                                 MOE_FLAG_FFN_ROWS_COPY | MOE_FLAG_FFN_ROWS_GATHER;
// Default tile form of the routed layer's expert FFN: single CTAs at every batch size.
// Measured on B200 (FFN stage, T = 32768): single CTAs 3.14 ms with the in-kernel row gather;
// CTA pairs 3.78 ms with it -- the second CTA's gathered rows must be forwarded to the MMA's
// barrier -- and 2.96 ms (single CTAs 3.01 ms) when the rows are first copied in expert order
// and loaded by TMA, but that copy costs 0.58 ms.  The dense MLP, whose rows need no copy,
// runs on pairs from kDensePairMinTokens tokens (T = 32768: 0.85 ms, 0.83 of the bf16 peak).
constexpr int kPairMinTokens = 1 << 30;
constexpr int kDensePairMinTokens = 2048;

#define GEMM_GEGLU grouped_gemm_persistent_kernel<kGemmStages, EPI_GEGLU, 4, true>
#define GEMM_FFN grouped_gemm_persistent_kernel<kGemmStages, EPI_GEGLU, 4, true, true>
// batches of at most 8 tokens (<= 8 rows per tile): 1 KB A slots, 6 stages
constexpr int kSmallStages = 6;
#define GEMM_FFN_SMALL grouped_gemm_persistent_kernel<kSmallStages, EPI_GEGLU, 4, true, true, true>
#define GEMM_STORE grouped_gemm_persistent_kernel<kGemmStages, EPI_STORE, 4>
#define GEMM_SCREEN grouped_gemm_kernel<kGemmStages, EPI_F32, 2>

bool flags_ok(unsigned flags) {
  if (flags & ~kKnownFlags) return false;
  if ((flags & MOE_FLAG_ROUTER_FP64) && (flags & MOE_FLAG_ROUTER_SCREEN)) return false;
  if ((flags & MOE_FLAG_DECODE_TILES) && (flags & MOE_FLAG_PREFILL_TILES)) return false;
  if ((flags & MOE_FLAG_UNFUSED_FFN) && (flags & MOE_FLAG_FUSED_FFN)) return false;
  const unsigned tiles = MOE_FLAG_FFN_PAIRS | MOE_FLAG_FFN_SINGLE;
  const unsigned rows = MOE_FLAG_FFN_ROWS_COPY | MOE_FLAG_FFN_ROWS_GATHER;
  if ((flags & tiles) == tiles || (flags & rows) == rows) return false;
  if ((flags & (tiles | rows)) &&
      (flags & (MOE_FLAG_FUSED_FFN | MOE_FLAG_UNFUSED_FFN | MOE_FLAG_DECODE_TILES)))
    return false;
  return true;
}

// Tensor-core screen + fp64 recheck, or fp64 logits for every expert.
// The screen's TMA map over W_router [H][E] needs 16-byte rows: E % 8 == 0.
bool screen_shape_ok(int E) { return E % 8 == 0; }

// A forced screen path needs a shape the screen supports.
bool forced_path_ok(int E, unsigned flags) {
  return !(flags & MOE_FLAG_ROUTER_SCREEN) || screen_shape_ok(E);
}

bool router_uses_screen(int T, int E, unsigned flags) {
  if (flags & (MOE_FLAG_NO_RENORM | MOE_FLAG_ROUTER_FP64)) return false;
  if (!screen_shape_ok(E)) return false;
  if (flags & MOE_FLAG_ROUTER_SCREEN) return true;
  return T >= kScreenMinTokens;
}

// The dynamically scheduled expert FFN unless a flag asks for another form (0 = not used).
// Its A slot holds R = 8, 16, 32, 64 or 128 rows: a tile never has more rows than T.
// Measured on B200 it beat the static schedules at every T from 1 to 32768.
int dy_rows(int T, unsigned flags) {
  if (flags & (MOE_FLAG_FUSED_FFN | MOE_FLAG_UNFUSED_FFN | MOE_FLAG_DECODE_TILES)) return 0;
  return T <= 8 ? 8 : T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128;
}

// The dynamic FFN on CTA pairs (256-row tiles, tcgen05 cta_group::2): batches of more than
// 64 tokens, when asked for (kPairMinTokens sets the default).
bool use_pair_ffn(int T, unsigned flags) {
  if (dy_rows(T, flags) != 128 || (flags & MOE_FLAG_FFN_SINGLE)) return false;
  return (flags & MOE_FLAG_FFN_PAIRS) || T >= kPairMinTokens;
}

// GEMM-1's A rows for the dynamic FFN of more than 64 tokens: copied into an expert-sorted
// buffer and loaded by TMA, or gathered inside the kernel (the default: see kPairMinTokens).
constexpr int kRowCopyMinTokens = 1 << 30;
bool use_row_copy(int T, unsigned flags) {
  if (dy_rows(T, flags) != 128 || (flags & MOE_FLAG_FFN_ROWS_GATHER)) return false;
  return (flags & MOE_FLAG_FFN_ROWS_COPY) || T >= kRowCopyMinTokens;
}

// Batches of at most 16 tokens (so at most 16 rows per expert) use the decode GEMMs.
constexpr int kDecodeMaxTokens = 16;
bool decode_gemm_ok(int T, int H, int I) {
  return T <= kDecodeMaxTokens && decode_shape_ok(I, true) && decode_shape_ok(H, false);
}
// Decode tiles only on request: measured on B200 the persistent 128-row tiles stream the
// weights faster at every batch size so far.
bool use_decode_gemm(int T, int H, int I, unsigned flags) {
  return (flags & MOE_FLAG_DECODE_TILES) && decode_gemm_ok(T, H, I);
}

// Batches of at most 8 tokens take the fused router + dispatch + gather launch.
bool use_decode_front(int T, int H, int E, unsigned flags) {
  return T <= kFrontMaxTokens && E <= 128 && !router_uses_screen(T, E, flags) &&
         H % (kFrontRanks * kFrontWarps) == 0 &&
         decode_front_smem_bytes(H, E) <= (size_t)kFrontSmemMax;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// K split of the screen GEMM: enough (row tile, K slice) CTAs to cover the SMs of a B200
// (148), at most 8 slices and at least one 64-wide k-block per slice.
int screen_ksplit(int T, int H) {
  const int mt = (T + 127) / 128;
  return std::max(1, std::min({kMaxScreenSplit, 148 / std::max(1, mt), H / 64}));
}

bool shape_supported(int T, int H, int E, int I, int k, bool need_I) {
  if (T < 1 || T > 1048576) return false;
  if (H < 64 || H > 16384 || H % 64) return false;
  if (need_I && (I < 64 || I > 8192 || I % 64)) return false;
  if (E < 4 || E > 256 || E % 4 || (E > 128 && E % 8)) return false;
  if (k < 1 || k > 8 || k > E) return false;
  return true;
}

// Split of the router's H axis over CTAs: a divisor d of H/32 (so every warp's share is a
// whole number of 8-element vectors) with 64 <= H/d <= 1408 (the per-CTA x stage stays
// within 88 KB), the smallest one that gives ~2 CTAs per SM.
int router_ksplit(int T, int H) {
  const int ntg = (T + kRouterTokens - 1) / kRouterTokens;
  const int target = (296 + ntg - 1) / ntg;
  int first = -1, largest = -1;
  for (int d = 1; d <= H / 32; ++d) {
    if ((H / 32) % d) continue;
    const int hs = H / d;
    if (hs < 64 || hs > 1408) continue;
    largest = d;
    if (first < 0 && d >= target) first = d;
  }
  return first > 0 ? first : largest;
}

struct Layout {
  bool screen = false;
  int ks = 0, hs = 0, nchunks = 0, max_tiles = 0, bm = 0;
  size_t part_logit = 0, part_xn2 = 0, part_wn2 = 0, stats = 0, ids = 0, wts = 0;
  size_t scr = 0, wrT = 0, wn = 0;
  int screen_ks = 1;   // K split of the screen GEMM (partial-sum slices in scr)
  size_t chunk_counts = 0, chunk_base = 0, counts = 0, offsets = 0, perm = 0, inv = 0;
  size_t dsync = 0;   // one-launch dispatch: arrivals, flag
  size_t tile_num = 0, tile_expert = 0, tile_row0 = 0, tile_rows = 0;
  size_t xp = 0, hbuf = 0, obuf = 0;
  size_t partials = 0, partials2 = 0, counters = 0;
  int dy_ctr = 0;   // dynamic FFN: offset of its unit counter among the counters
  int n_counters = 0;
  size_t total = 0;
};

Layout make_layout(int T, int H, int E, int I, int k, unsigned flags, bool forward) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const size_t P = (size_t)T * k;
  L.screen = router_uses_screen(T, E, flags);
  L.stats = take(8 * sizeof(unsigned));   // router statistics [5]; [7] front-end counter
  if (L.screen) {
    L.screen_ks = screen_ksplit(T, H);
    L.scr = take(sizeof(float) * (size_t)L.screen_ks * T * E);
    L.wrT = take(2 * (size_t)E * H);
    L.wn = take(sizeof(double) * E);
  } else {
    L.ks = router_ksplit(T, H);
    L.hs = H / L.ks;
    L.part_logit = take(sizeof(double) * L.ks * (size_t)T * E);
    L.part_xn2 = take(sizeof(double) * L.ks * (size_t)T);
    L.part_wn2 = take(sizeof(double) * L.ks * (size_t)E);
  }
  if (forward) {
    L.nchunks = (int)((P + kDispatchChunk - 1) / kDispatchChunk);
    L.bm = use_decode_gemm(T, H, I, flags) ? DG_BN : use_pair_ffn(T, flags) ? PR_ROWS : GM_BM;
    L.max_tiles = (int)(P / L.bm) + E;
    L.ids = take(sizeof(int32_t) * P);
    L.wts = take(sizeof(float) * P);
    L.chunk_counts = take(sizeof(int32_t) * (size_t)L.nchunks * E);
    L.chunk_base = take(sizeof(int32_t) * (size_t)L.nchunks * E);
    L.dsync = take(2 * sizeof(int32_t));
    L.counts = take(sizeof(int32_t) * E);
    L.offsets = take(sizeof(int32_t) * (E + 1));
    L.perm = take(sizeof(int32_t) * P);
    L.inv = take(sizeof(int32_t) * P);
    L.tile_num = take(sizeof(int32_t));
    L.tile_expert = take(sizeof(int32_t) * L.max_tiles);
    L.tile_row0 = take(sizeof(int32_t) * L.max_tiles);
    L.tile_rows = take(sizeof(int32_t) * L.max_tiles);
    // Xp (expert-sorted copies of the x rows) only for the decode tiles; the prefill tiles
    // gather the rows straight from x
    if (L.bm == DG_BN || use_row_copy(T, flags)) L.xp = take(2 * P * H);
    L.hbuf = take(2 * P * I);
    L.obuf = take(2 * P * H);
    // stream-K split tiles of the statically scheduled GEMMs: two fp32 tile slots per CTA
    // and per-(split unit, row quadrant) counters, one set per GEMM (the fused launch runs
    // both at once); then one h-ready counter per tile for the single-launch forms
    const int R = dy_rows(T, flags);
    if (R == 0) {
      L.partials = take(sizeof(float) * 2 * (size_t)kMaxGemmCtas * GM_BM * 256);
      L.partials2 = take(sizeof(float) * 2 * (size_t)kMaxGemmCtas * GM_BM * 256);
    }
    L.n_counters = 2 * kStreamKCounters + L.max_tiles + 1;
    if (R > 0) {
      // dynamic FFN: its unit counter
      L.dy_ctr = L.n_counters;
      L.n_counters += 1;
    }
    L.counters = take(sizeof(int32_t) * L.n_counters);
  }
  L.total = off;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// --------------------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major [rows][cols] bf16, box = box_cols x box_rows (64 columns with the 128-byte
// swizzle, or 16 columns with the 32-byte swizzle).
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                 uint32_t box_cols = 64) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = box_cols == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bytes [rows][cols] (cols contiguous, cols % 16 == 0), box = 128 bytes x box_rows rows,
// 128-byte swizzle: NVFP4 codes (two per byte) as a K-major MMA operand.
bool make_map_u8_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                    uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// Scale lines [kb][rows][16 bytes] as (16, rows, kb), box 16 bytes x 32 rows x 4 kb, no
// swizzle: one load fills four 512-byte scale blocks.
bool make_map_lines(CUtensorMap* m, const void* base, uint64_t rows, uint64_t kb) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {16, rows, kb};
  cuuint64_t strides[2] = {16, 16 * rows};
  cuuint32_t box[3] = {16, 32, 4};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// Stacked bytes [E][rows][cols], box = 128 bytes x 128 rows x 1 expert, 128-byte swizzle.
bool make_map_u8_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, E};
  cuuint64_t strides[2] = {cols, cols * rows};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stacked [E][rows][cols] bf16 (cols contiguous), box = 64 columns x box_rows rows x 1 expert.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E,
                 uint32_t box_rows = 64) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, E};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stacked [E][rows][cols] bf16 viewed as (64 columns, rows, cols/64 slabs, E), box = 64 columns
// x box_rows rows x box_slabs slabs x 1: one load fills box_slabs consecutive 64-column slabs
// of box_rows rows each (slab-major in shared memory, 128-byte swizzle), the layout of the
// MN-major MMA operand.  Every in-bounds coordinate addresses memory inside the tensor.
bool make_map_slabs(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E,
                    uint32_t box_rows, uint32_t box_slabs) {
  auto fn = encode_fn();
  if (!fn || cols % 64) return false;
  cuuint64_t dims[4] = {64, rows, cols / 64, E};
  cuuint64_t strides[3] = {cols * 2, 128, cols * rows * 2};
  cuuint32_t box[4] = {64, box_rows, box_slabs, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// --------------------------------------------------------------------------- per device
struct DeviceState {
  bool attrs_set = false;
  int num_sms = 0;
  cudaEvent_t ev[8] = {};
  int n_profiled = -1;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

const char* kStageNames[] = {"router", "dispatch", "expert_ffn", "combine"};
constexpr int kNumStages = 4;

thread_local int t_last_cuda_error = 0;
thread_local int t_kernels = 0;   // kernels launched by this thread's current/last call

moe_status_t cuda_failed(int code) {
  t_last_cuda_error = code;
  return MOE_ERR_CUDA;
}

#define MOE_TRY_CUDA(call)                          \
  do {                                              \
    const cudaError_t e_ = (call);                  \
    if (e_ != cudaSuccess) return cuda_failed(e_);  \
  } while (0)

DeviceState* device_state(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceState& d = g_dev[dev];
  if (!d.attrs_set) {
    cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    const int gs = pgemm_smem_bytes<kGemmStages, 4>();   // both persistent variants
    const int gs2 = gemm_smem_bytes<kGemmStages, 2>();
    if (cudaFuncSetAttribute(GEMM_GEGLU, cudaFuncAttributeMaxDynamicSharedMemorySize, gs) !=
            cudaSuccess ||
        cudaFuncSetAttribute(GEMM_FFN, cudaFuncAttributeMaxDynamicSharedMemorySize, gs) !=
            cudaSuccess ||
        cudaFuncSetAttribute(expert_ffn_dynamic_kernel<8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, dy_smem_bytes<8>()) !=
            cudaSuccess ||
        cudaFuncSetAttribute(expert_ffn_dynamic_kernel<16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, dy_smem_bytes<16>()) !=
            cudaSuccess ||
        cudaFuncSetAttribute(expert_ffn_dynamic_kernel<32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, dy_smem_bytes<32>()) !=
            cudaSuccess ||
        cudaFuncSetAttribute(expert_ffn_dynamic_kernel<64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, dy_smem_bytes<64>()) !=
            cudaSuccess ||
        cudaFuncSetAttribute(expert_ffn_dynamic_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, dy_smem_bytes<128>()) !=
            cudaSuccess ||
        cudaFuncSetAttribute(expert_ffn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PR_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(nvfp4_ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             F4_SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(GEMM_FFN_SMALL, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pgemm_smem_bytes<kSmallStages, 4, true>()) != cudaSuccess ||
        cudaFuncSetAttribute(GEMM_STORE, cudaFuncAttributeMaxDynamicSharedMemorySize, gs) !=
            cudaSuccess ||
        cudaFuncSetAttribute(GEMM_SCREEN, cudaFuncAttributeMaxDynamicSharedMemorySize, gs2) !=
            cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_decode_kernel<EPI_GEGLU>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_decode_kernel<EPI_STORE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(decode_front_kernel<4>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kFrontSmemMax) !=
            cudaSuccess ||
        cudaFuncSetAttribute(router_partial_kernel<4>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 1408 * 8 * 8) !=
            cudaSuccess ||
        cudaFuncSetAttribute(router_partial_kernel<8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 1408 * 8 * 8) !=
            cudaSuccess) {
      cuda_failed(cudaGetLastError());
      return nullptr;
    }
    for (auto& e : d.ev)
      if (const cudaError_t err = cudaEventCreate(&e); err != cudaSuccess) {
        cuda_failed(err);
        return nullptr;
      }
    d.attrs_set = true;
  }
  return &d;
}

struct Profiler {
  DeviceState* d;
  cudaStream_t st;
  bool on;
  int n = 0;
  unsigned rec_flags = cudaEventRecordDefault;
  // External records become event nodes when the call is captured into a CUDA graph, so
  // every replay records the stage boundaries (a plain record would only be a capture
  // dependency and never fire).
  void mark() {
    if (!on) return;
    if (n == 0) {
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      cudaStreamIsCapturing(st, &cs);
      rec_flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                      : cudaEventRecordDefault;
    }
    cudaEventRecordWithFlags(d->ev[n++], st, rec_flags);
  }
  void finish() {
    if (on) d->n_profiled = n - 1;
  }
};

moe_status_t launched() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : cuda_failed(e);
}

// Kernel launch; with `dependent` the kernel may start launching while the previous kernel
// on the stream is still running (programmatic stream serialisation): it runs its prologue
// and then waits in pdl_wait() for that kernel's results.
struct Launch {
  cudaStream_t st;
  bool pdl;   // allowed for this call (off while stage events sit between kernels)
  template <typename... KArgs, typename... Args>
  void operator()(bool dependent, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                  Args... args) const {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (dependent && pdl) ? 1 : 0;
    cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    ++t_kernels;
  }
};

moe_status_t launch_router(const __nv_bfloat16* x, const __nv_bfloat16* wr, const float* bias,
                           int T, int H, int E, int k, unsigned flags, int32_t* ids, float* wts,
                           unsigned* stats, uint8_t* ws, const Layout& L, const DeviceState& d,
                           cudaStream_t st, bool pdl) {
  MOE_TRY_CUDA(cudaMemsetAsync(stats, 0, kRouterStats * sizeof(unsigned), st));
  const Launch launch{st, pdl};
  const double u = std::ldexp(1.0, -53);
  const double n = (double)H + 8.0;
  const double gamma = n * u / (1.0 - n * u);
  const double beta_scale = 2.0 * gamma * 1.01;
  const int renorm = (flags & MOE_FLAG_NO_RENORM) ? 0 : 1;
  const int warps_blocks = std::min((T + 7) / 8, std::max(1, d.num_sms) * 8);
  if (L.screen) {
    float* scr = reinterpret_cast<float*>(ws + L.scr);
    __nv_bfloat16* wrT = reinterpret_cast<__nv_bfloat16*>(ws + L.wrT);
    double* wn = reinterpret_cast<double*>(ws + L.wn);
    launch(false, router_transpose_kernel, dim3((H + 31) / 32, (E + 31) / 32), dim3(32, 8), 0, wr,
           H, E, wrT);
    launch(true, router_wnorm_kernel, dim3(E), dim3(256), 0, wrT, H, E, wn);
    CUtensorMap tm_x, tm_wr;
    if (!make_map_2d(&tm_x, x, H, T, GM_BM) || !make_map_3d(&tm_wr, wr, E, H, 1))
      return cuda_failed(-1);   // a tensor map could not be encoded
    const TileList tl{nullptr, nullptr, nullptr, nullptr, T};
    const int nb = (E + 127) / 128;
    const int mt = (T + GM_BM - 1) / GM_BM;
    launch(true, GEMM_SCREEN, dim3(nb * mt, L.screen_ks), dim3(128),
           gemm_smem_bytes<kGemmStages, 2>(), tm_x, tm_wr, tm_wr, tl, nb, H, E, (void*)scr, E);
    const long long kstride = (long long)T * E;
    // at least four waves of 2-per-SM CTAs: the 4-per-SM form (same arithmetic)
    const bool deep = (long long)T >= 8LL * std::max(1, d.num_sms) * kScreenWarps;
    if (E <= 128 && deep)
      launch(true, router_screen_select_kernel<4, 4>, dim3(warps_blocks),
             dim3(32 * kScreenWarps), 0, (const float*)scr, L.screen_ks, kstride, x,
             (const __nv_bfloat16*)wrT, (const double*)wn, bias, T, H, E, k, kScreenC,
             beta_scale, ids, wts, stats);
    else if (E <= 128)
      launch(true, router_screen_select_kernel<4>, dim3(warps_blocks), dim3(32 * kScreenWarps), 0,
             (const float*)scr, L.screen_ks, kstride, x, (const __nv_bfloat16*)wrT,
             (const double*)wn, bias, T, H, E, k, kScreenC, beta_scale, ids, wts, stats);
    else
      launch(true, router_screen_select_kernel<8>, dim3(warps_blocks), dim3(32 * kScreenWarps), 0,
             (const float*)scr, L.screen_ks, kstride, x, (const __nv_bfloat16*)wrT,
             (const double*)wn, bias, T, H, E, k, kScreenC, beta_scale, ids, wts, stats);
    return launched();
  }
  double* part_logit = reinterpret_cast<double*>(ws + L.part_logit);
  double* part_xn2 = reinterpret_cast<double*>(ws + L.part_xn2);
  double* part_wn2 = reinterpret_cast<double*>(ws + L.part_wn2);
  const dim3 g1((T + kRouterTokens - 1) / kRouterTokens, L.ks);
  const size_t sm1 = sizeof(double) * std::max<size_t>((size_t)L.hs * kRouterTokens,
                                                       (size_t)kRouterWarps * kRouterTokens * E);
  if (E <= 128)
    launch(false, router_partial_kernel<4>, g1, dim3(128), sm1, x, wr, T, H, E, L.hs, part_logit,
           part_xn2, part_wn2);
  else
    launch(false, router_partial_kernel<8>, g1, dim3(128), sm1, x, wr, T, H, E, L.hs, part_logit,
           part_xn2, part_wn2);
  if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
  if (E <= 128)
    launch(true, router_select_kernel<4>, dim3(warps_blocks), dim3(256), 0,
           (const double*)part_logit, (const double*)part_xn2, (const double*)part_wn2, L.ks, bias,
           x, wr, T, H, E, k, renorm, beta_scale, ids, wts, stats);
  else
    launch(true, router_select_kernel<8>, dim3(warps_blocks), dim3(256), 0,
           (const double*)part_logit, (const double*)part_xn2, (const double*)part_wn2, L.ks, bias,
           x, wr, T, H, E, k, renorm, beta_scale, ids, wts, stats);
  return launched();
}

// Steps 1 and 2 of the layer (router, dispatch) into the buffers of `b` and the workspace's
// tile list; with copy_rows also the copy of the routed rows into Xp in expert order.
struct RouteBufs {
  int32_t* ids;
  float* wts;
  unsigned* stats;
  int32_t *counts, *offsets, *perm, *inv;
};
moe_status_t route_and_dispatch(const void* x, const void* w_router, const float* router_bias,
                                int T, int H, int E, int k, unsigned flags, const RouteBufs& b,
                                uint8_t* ws, const Layout& L, const DeviceState& dv,
                                cudaStream_t st, Profiler& prof, bool copy_rows) {
  const DeviceState* d = &dv;
  int32_t *ids = b.ids, *counts = b.counts, *offsets = b.offsets, *perm = b.perm, *inv = b.inv;
  float* wts = b.wts;
  unsigned* stats = b.stats;
  const int P = T * k;
  int32_t* chunk_counts = reinterpret_cast<int32_t*>(ws + L.chunk_counts);
  int32_t* chunk_base = reinterpret_cast<int32_t*>(ws + L.chunk_base);
  int32_t* tile_num = reinterpret_cast<int32_t*>(ws + L.tile_num);
  int32_t* tile_expert = reinterpret_cast<int32_t*>(ws + L.tile_expert);
  int32_t* tile_row0 = reinterpret_cast<int32_t*>(ws + L.tile_row0);
  int32_t* tile_rows = reinterpret_cast<int32_t*>(ws + L.tile_rows);
  __nv_bfloat16* xp = reinterpret_cast<__nv_bfloat16*>(ws + L.xp);
  int32_t* gemm_counters = reinterpret_cast<int32_t*>(ws + L.counters);
  const int gsm = std::max(1, d->num_sms) * 8;
  // Dependent launches, except while stage events sit between the kernels.
  const Launch launch{st, !prof.on};
  if (use_decode_front(T, H, E, flags)) {
    // 1+2. router and dispatch in one launch: one 8-CTA cluster per token.  Word 7 of the
    // workspace statistics is the front end's token counter (zero at launch, left zero).
    unsigned* ws_stats = reinterpret_cast<unsigned*>(ws + L.stats);
    unsigned* front_done = ws_stats + 7;
    if (stats == ws_stats) {
      MOE_TRY_CUDA(cudaMemsetAsync(ws_stats, 0, 8 * sizeof(unsigned), st));
    } else {
      MOE_TRY_CUDA(cudaMemsetAsync(stats, 0, kRouterStats * sizeof(unsigned), st));
      MOE_TRY_CUDA(cudaMemsetAsync(front_done, 0, sizeof(unsigned), st));
    }
    const double u = std::ldexp(1.0, -53), n = (double)H + 8.0;
    const double beta_scale = 2.0 * (n * u / (1.0 - n * u)) * 1.01;
    launch(false, decode_front_kernel<4>, dim3(kFrontRanks * T), dim3(32 * kFrontWarps),
           decode_front_smem_bytes(H, E), static_cast<const __nv_bfloat16*>(x),
           static_cast<const __nv_bfloat16*>(w_router), router_bias, T, H, E, k,
           (flags & MOE_FLAG_NO_RENORM) ? 0 : 1, beta_scale, ids, wts, stats, counts, offsets, perm,
           inv, tile_num, tile_expert, tile_row0, tile_rows, gemm_counters, L.n_counters, L.bm,
           front_done);
    if (copy_rows)   // decode tiles read a gathered copy of the routed rows
      launch(true, gather_rows_kernel, dim3(std::min((P + 7) / 8, gsm)), dim3(256), 0,
             static_cast<const uint4*>(x), (const int32_t*)perm, P, k, P, H / 8,
             reinterpret_cast<uint4*>(xp));
    if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
    prof.mark();
    prof.mark();
  } else {
    // one-launch dispatch for 2..32 chunks (every chunk's CTA must be resident at once;
    // measured on B200: 2 us faster at 8 and 16 chunks, 5-12 us slower at 64 and 128)
    const bool fused_dispatch =
        L.nchunks > 1 && L.nchunks <= std::min(kFusedDispatchMaxChunks, d->num_sms);
    int32_t* dsync = reinterpret_cast<int32_t*>(ws + L.dsync);
    if (fused_dispatch) MOE_TRY_CUDA(cudaMemsetAsync(dsync, 0, 2 * sizeof(int32_t), st));
    // 1. router
    moe_status_t s = launch_router(static_cast<const __nv_bfloat16*>(x),
                                   static_cast<const __nv_bfloat16*>(w_router), router_bias, T, H,
                                   E, k, flags, ids, wts, stats, ws, L, *d, st, !prof.on);
    if (s != MOE_OK) return s;
    prof.mark();
    // 2. dispatch
    if (L.nchunks == 1) {
      launch(true, dispatch_small_kernel, dim3(1), dim3(256), 0, (const int32_t*)ids, P, E, L.bm,
             counts, offsets, perm, inv, tile_num, tile_expert, tile_row0, tile_rows,
             gemm_counters, L.n_counters);
    } else if (fused_dispatch) {
      launch(true, dispatch_fused_kernel, dim3(L.nchunks), dim3(32 * kRankWarps),
             (kRankWarps + 1) * E * sizeof(int), (const int32_t*)ids, P, E, L.bm, L.nchunks,
             chunk_counts, chunk_base, counts, offsets, perm, inv, tile_num, tile_expert,
             tile_row0, tile_rows, gemm_counters, L.n_counters, dsync);
    } else {
      launch(true, dispatch_count_kernel, dim3(L.nchunks), dim3(256), E * sizeof(int),
             (const int32_t*)ids, P, E, chunk_counts);
      launch(true, dispatch_scan_kernel, dim3(1), dim3(256), 0, (const int32_t*)chunk_counts,
             L.nchunks, E, P, L.bm, counts, offsets, chunk_base, tile_num, tile_expert, tile_row0,
             tile_rows, gemm_counters, L.n_counters);
      launch(true, dispatch_rank_kernel, dim3(L.nchunks), dim3(32 * kRankWarps),
             (kRankWarps + 1) * E * sizeof(int),
             (const int32_t*)ids, P, E, (const int32_t*)chunk_base, perm, inv);
    }
    if (copy_rows)   // the routed rows, in expert order
      launch(true, gather_rows_kernel, dim3(std::min((P + 7) / 8, gsm)), dim3(256), 0,
             static_cast<const uint4*>(x), (const int32_t*)perm, P, k, P, H / 8,
             reinterpret_cast<uint4*>(xp));
    if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
    prof.mark();
  }
  return MOE_OK;
}

// Scratch of moe_route_static: a file-scope device array (every GPU that loads this
// library holds it until the process exits).  Host code must not use the symbol itself as a
// device address; moe_route_static looks its address up once per device.
constexpr size_t kStaticScratchBytes = 4u << 20;
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];
void* g_static_scratch_ptr[kMaxDevices] = {};

__global__ void unsatisfied_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  mbar_wait(b, 0);  // nothing arrives: runs out after the wait limit and raises the error
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_NO_WORKSPACE: return "MOE_ERR_NO_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

size_t moe_route_workspace_size(int T, int H, int E, int k, unsigned flags) {
  if (!flags_ok(flags) || !shape_supported(T, H, E, 64, k, false) || !forced_path_ok(E, flags))
    return 0;
  return make_layout(T, H, E, 64, k, flags, false).total;
}

size_t moe_workspace_size(int T, int H, int E, int I, int k, unsigned flags) {
  if (!flags_ok(flags) || !shape_supported(T, H, E, I, k, true) || !forced_path_ok(E, flags))
    return 0;
  return make_layout(T, H, E, I, k, flags, true).total;
}

moe_status_t moe_route(const void* x, const void* w_router, const float* router_bias, int T,
                       int H, int E, int k, unsigned flags, int32_t* topk_ids,
                       float* topk_weights, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (T < 0 || H <= 0 || E <= 0 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (!flags_ok(flags)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !topk_ids || !topk_weights || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  if (!shape_supported(T, H, E, 64, k, false) || !forced_path_ok(E, flags))
    return MOE_ERR_UNSUPPORTED;
  const Layout L = make_layout(T, H, E, 64, k, flags, false);
  if (workspace_bytes < L.total) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return launch_router(static_cast<const __nv_bfloat16*>(x),
                       static_cast<const __nv_bfloat16*>(w_router), router_bias, T, H, E, k, flags,
                       topk_ids, topk_weights,
                       reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + L.stats),
                       static_cast<uint8_t*>(workspace), L, *d, st, true);
}

moe_status_t moe_forward(const void* x, const void* w_router, const float* router_bias,
                         const void* w_gate, const void* w_up, const void* w_down, int T, int H,
                         int E, int I, int k, unsigned flags, void* y, const moe_aux_t* aux,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0 || H <= 0 || E <= 0 || I <= 0 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (!flags_ok(flags)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !w_gate || !w_up || !w_down || !y || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w_gate) || !aligned16(w_up) ||
      !aligned16(w_down) || !aligned16(y) || !aligned16(workspace))
    return MOE_ERR_INVALID_ARG;
  if (x == y) return MOE_ERR_INVALID_ARG;
  if (!shape_supported(T, H, E, I, k, true) || !forced_path_ok(E, flags))
    return MOE_ERR_UNSUPPORTED;
  if ((flags & MOE_FLAG_DECODE_TILES) && !decode_gemm_ok(T, H, I)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(T, H, E, I, k, flags, true);
  if (workspace_bytes < L.total) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int P = T * k;

  int32_t* ids = (aux && aux->topk_ids) ? aux->topk_ids : reinterpret_cast<int32_t*>(ws + L.ids);
  float* wts = (aux && aux->topk_weights) ? aux->topk_weights : reinterpret_cast<float*>(ws + L.wts);
  int32_t* counts =
      (aux && aux->expert_counts) ? aux->expert_counts : reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = (aux && aux->expert_offsets) ? aux->expert_offsets
                                                  : reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm = (aux && aux->perm) ? aux->perm : reinterpret_cast<int32_t*>(ws + L.perm);
  unsigned* stats = (aux && aux->router_stats) ? aux->router_stats
                                               : reinterpret_cast<unsigned*>(ws + L.stats);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
  int32_t* tile_num = reinterpret_cast<int32_t*>(ws + L.tile_num);
  int32_t* tile_expert = reinterpret_cast<int32_t*>(ws + L.tile_expert);
  int32_t* tile_row0 = reinterpret_cast<int32_t*>(ws + L.tile_row0);
  int32_t* tile_rows = reinterpret_cast<int32_t*>(ws + L.tile_rows);
  __nv_bfloat16* xp = reinterpret_cast<__nv_bfloat16*>(ws + L.xp);
  __nv_bfloat16* hbuf = reinterpret_cast<__nv_bfloat16*>(ws + L.hbuf);
  __nv_bfloat16* obuf = reinterpret_cast<__nv_bfloat16*>(ws + L.obuf);

  const bool dec = L.bm == DG_BN;    // decode tiles: <= 16 rows per expert
  CUtensorMap tm_xp, tm_wg, tm_wu, tm_h, tm_wd;
  const uint32_t act_rows = dec ? DG_BN : GM_BM, act_cols = dec ? DG_KS : 64;
  // weight boxes: decode = 16 rows x every slab of the expert; prefill = 64 rows x 2 (gate,
  // up) or 4 (down) slabs
  const uint32_t w_rows = dec ? DG_KS : 64;
  const uint32_t gu_slabs = dec ? (uint32_t)(I / 64) : 2u, d_slabs = dec ? (uint32_t)(H / 64) : 4u;
  // Prefill tiles gather their A rows from x inside GEMM-1; their A map is a placeholder.
  const bool ok_x = dec ? make_map_2d(&tm_xp, xp, H, P, act_rows, act_cols)
                        : make_map_2d(&tm_xp, x, H, T, 1, 64);
  if (!ok_x ||
      !make_map_slabs(&tm_wg, w_gate, I, H, E, w_rows, gu_slabs) ||
      !make_map_slabs(&tm_wu, w_up, I, H, E, w_rows, gu_slabs) ||
      !make_map_2d(&tm_h, hbuf, I, P, act_rows, act_cols) ||
      !make_map_slabs(&tm_wd, w_down, H, I, E, w_rows, d_slabs))
    return cuda_failed(-1);   // a tensor map could not be encoded

  Profiler prof{d, st, (flags & MOE_FLAG_PROFILE_STAGES) != 0};
  prof.mark();
  int32_t* gemm_counters = reinterpret_cast<int32_t*>(ws + L.counters);
  const int gsm = std::max(1, d->num_sms) * 8;
  // Dependent launches, except while stage events sit between the kernels.
  const Launch launch{st, !prof.on};
  {
    const RouteBufs rb{ids, wts, stats, counts, offsets, perm, inv};
    if (const moe_status_t rs = route_and_dispatch(x, w_router, router_bias, T, H, E, k, flags, rb,
                                                   ws, L, *d, st, prof, dec || use_row_copy(T, flags));
        rs != MOE_OK)
      return rs;
  }
  // 3. GEMM-1 + GEGLU, 4. GEMM-2 (down)
  TileList tl{tile_num, tile_expert, tile_row0, tile_rows, 0, perm, k,
              static_cast<const __nv_bfloat16*>(x), H, T};
  tl.a_tma = use_row_copy(T, flags) ? 1 : 0;
  float* partials = reinterpret_cast<float*>(ws + L.partials);
  float* partials2 = reinterpret_cast<float*>(ws + L.partials2);
  const int G = std::min(std::max(1, d->num_sms), kMaxGemmCtas);
  int32_t* ctr1 = gemm_counters;
  int32_t* ctr2 = gemm_counters + kStreamKCounters;
  int32_t* h_ready = gemm_counters + 2 * kStreamKCounters;
  if (dec) {
    launch(true, grouped_gemm_decode_kernel<EPI_GEGLU>, dim3(G), dim3(DG_THREADS),
           decode_smem_bytes(I, true), tm_xp, tm_wg, tm_wu, tl, H, I, (void*)hbuf, I, partials,
           ctr1);
    if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
    launch(true, grouped_gemm_decode_kernel<EPI_STORE>, dim3(G), dim3(DG_THREADS),
           decode_smem_bytes(H, false), tm_h, tm_wd, tm_wd, tl, I, H, (void*)obuf, H, partials,
           ctr2);
    if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
  } else {
    const int smem = pgemm_smem_bytes<kGemmStages, 4>();
    const PGemm g1{(I + 127) / 128, H, I, hbuf, I, partials, ctr1};
    const PGemm g2{(H + 255) / 256, I, H, obuf, H, partials2, ctr2};
    if (const int R = dy_rows(T, flags); R > 0) {
      // at most R rows per tile, whole units handed out from a shared counter; one-slab
      // weight maps for a narrow last GEMM-1 block (I % 128 == 64)
      CUtensorMap tm_hr, tm_wg1, tm_wu1, tm_xr;
      if (!make_map_2d(&tm_hr, hbuf, I, P, R, 64) ||
          !make_map_slabs(&tm_wg1, w_gate, I, H, E, 64, 1) ||
          !make_map_slabs(&tm_wu1, w_up, I, H, E, 64, 1) ||
          !make_map_2d(&tm_xr, tl.a_tma ? (const void*)xp : x, H, tl.a_tma ? P : T, R, 64))
        return cuda_failed(-1);
      int32_t* dctr = gemm_counters + L.dy_ctr;
      const DyState dys{dctr};
      auto go = [&](auto kernel, int smem, int threads) {
        launch(true, kernel, dim3(G), dim3(threads), smem, tm_wg, tm_wu, tm_wg1, tm_wu1, tm_xr,
               tm_hr, tm_wd, tl, g1, g2, h_ready, dys);
      };
      if (L.bm == PR_ROWS) {
        // CTA pairs (2-CTA clusters, an even grid): 2-slab W_down boxes, each CTA loading
        // 128 of a block's 256 columns
        CUtensorMap tm_wd2;
        if (!make_map_slabs(&tm_wd2, w_down, H, I, E, 64, 2)) return cuda_failed(-1);
        launch(true, expert_ffn_pair_kernel, dim3(std::max(2, G & ~1)), dim3(pgemm_threads(true)),
               PR_SMEM, tm_wg, tm_wu, tm_wg1, tm_wu1, tm_xr, tm_hr, tm_wd2, tl, g1, g2, h_ready,
               dys);
      } else if (R == 8) go(expert_ffn_dynamic_kernel<8>, dy_smem_bytes<8>(), dy_threads<8>());
      else if (R == 16) go(expert_ffn_dynamic_kernel<16>, dy_smem_bytes<16>(), dy_threads<16>());
      else if (R == 32) go(expert_ffn_dynamic_kernel<32>, dy_smem_bytes<32>(), dy_threads<32>());
      else if (R == 64) go(expert_ffn_dynamic_kernel<64>, dy_smem_bytes<64>(), dy_threads<64>());
      else go(expert_ffn_dynamic_kernel<128>, dy_smem_bytes<128>(), dy_threads<128>());
    } else if (flags & MOE_FLAG_UNFUSED_FFN) {
      // static stream-K schedule, GEMM-1 (+GEGLU) and GEMM-2 as two launches
      launch(true, GEMM_GEGLU, dim3(G), dim3(pgemm_threads(true)), smem, tm_xp, tm_wg, tm_wu,
             tm_xp, tm_wg, tl, g1, g1, h_ready);
      if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
      launch(true, GEMM_STORE, dim3(G), dim3(pgemm_threads(false)), smem, tm_h, tm_wd, tm_wd,
             tm_h, tm_wd, tl, g2, g2, h_ready);
    } else if (T <= PG_SMALL_ROWS) {
      // static schedule in one launch; every tile has at most T <= 8 rows: 8-row A slots (and an 8-row box over h)
      CUtensorMap tm_h8;
      if (!make_map_2d(&tm_h8, hbuf, I, P, PG_SMALL_ROWS, 64)) return cuda_failed(-1);
      launch(true, GEMM_FFN_SMALL, dim3(G), dim3(pgemm_threads(true)),
             pgemm_smem_bytes<kSmallStages, 4, true>(), tm_xp, tm_wg, tm_wu, tm_h8, tm_wd, tl, g1,
             g2, h_ready);
    } else {
      launch(true, GEMM_FFN, dim3(G), dim3(pgemm_threads(true)), smem, tm_xp, tm_wg, tm_wu, tm_h,
             tm_wd, tl, g1, g2, h_ready);
    }
    if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
  }
  prof.mark();
  // 5. combine: one warp per (token, 64-vector chunk), 8 warps per block
  const long long citems = (long long)T * ((H / 8 + kCombineChunkVec - 1) / kCombineChunkVec);
  launch(true, combine_kernel<false>, dim3((int)std::min<long long>((citems + 7) / 8, gsm)),
         dim3(256), 0, reinterpret_cast<const uint4*>(obuf), (const int32_t*)inv,
         (const float*)wts, T, k, H / 8, 0, P, y);
  if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
  prof.mark();
  prof.finish();
  return MOE_OK;
}

// ----------------------------------------------------------------------------- dense MLP
// The dense GEGLU MLP beside the MoE: the expert FFN kernel with every row in one "expert"
// (uniform tiles of 128 rows, no permutation), GEMM-2 writing y in token order.
// Workspace: h [T][I] bf16, then the unit counter and the h-ready counters (one per row
// tile, plus their total).
struct DenseLayout {
  size_t hbuf = 0, counters = 0, total = 0;
  int n_tiles = 0, n_counters = 0;
};

DenseLayout dense_layout(int T, int I) {
  DenseLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.n_tiles = (T + GM_BM - 1) / GM_BM;
  L.hbuf = take(2 * (size_t)T * I);
  L.n_counters = 1 + L.n_tiles + 1;
  L.counters = take(sizeof(int32_t) * L.n_counters);
  L.total = off;
  return L;
}

size_t moe_dense_workspace_size(int T, int H, int I) {
  if (T < 1 || T > 1048576 || H < 64 || H > 16384 || H % 64 || I < 64 || I > 8192 || I % 64)
    return 0;
  return dense_layout(T, I).total;
}

moe_status_t moe_dense_ffn(const void* x, const void* w_gate, const void* w_up,
                           const void* w_down, int T, int H, int I, void* y, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (T < 0 || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_gate || !w_up || !w_down || !y || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(y) || !aligned16(workspace))
    return MOE_ERR_INVALID_ARG;
  if (x == y) return MOE_ERR_INVALID_ARG;
  if (moe_dense_workspace_size(T, H, I) == 0) return MOE_ERR_UNSUPPORTED;
  const DenseLayout L = dense_layout(T, I);
  if (workspace_bytes < L.total) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* hbuf = reinterpret_cast<__nv_bfloat16*>(ws + L.hbuf);
  int32_t* ctr = reinterpret_cast<int32_t*>(ws + L.counters);
  MOE_TRY_CUDA(cudaMemsetAsync(ctr, 0, sizeof(int32_t) * L.n_counters, st));

  const int R = dy_rows(T, 0);
  CUtensorMap tm_wg, tm_wu, tm_wg1, tm_wu1, tm_wd, tm_hr, tm_xr;
  if (!make_map_slabs(&tm_wg, w_gate, I, H, 1, 64, 2) ||
      !make_map_slabs(&tm_wu, w_up, I, H, 1, 64, 2) ||
      !make_map_slabs(&tm_wg1, w_gate, I, H, 1, 64, 1) ||
      !make_map_slabs(&tm_wu1, w_up, I, H, 1, 64, 1) ||
      !make_map_slabs(&tm_wd, w_down, H, I, 1, 64, 4) || !make_map_2d(&tm_hr, hbuf, I, T, R, 64) ||
      !make_map_2d(&tm_xr, x, H, T, R, 64))
    return cuda_failed(-1);   // a tensor map could not be encoded
  // the rows of x are the A rows in place: TMA tiles of them
  TileList tl{nullptr, nullptr, nullptr, nullptr, T,
              nullptr, 1,       static_cast<const __nv_bfloat16*>(x), H, T};
  tl.a_tma = 1;
  const PGemm g1{(I + 127) / 128, H, I, hbuf, I, nullptr, nullptr};
  const PGemm g2{(H + 255) / 256, I, H, y, H, nullptr, nullptr};
  int32_t* h_ready = ctr + 1;
  const DyState dys{ctr};
  const int G = std::min(std::max(1, d->num_sms), kMaxGemmCtas);
  const Launch launch{st, false};
  auto go = [&](auto kernel, int smem, int threads) {
    launch(false, kernel, dim3(G), dim3(threads), smem, tm_wg, tm_wu, tm_wg1, tm_wu1, tm_xr,
           tm_hr, tm_wd, tl, g1, g2, h_ready, dys);
  };
  if (dy_rows(T, 0) == 128 && T >= kDensePairMinTokens) {
    // CTA pairs over 256-row tiles of x (the counters above cover ceil(T / 128) tiles)
    CUtensorMap tm_wd2;
    if (!make_map_slabs(&tm_wd2, w_down, H, I, 1, 64, 2)) return cuda_failed(-1);
    launch(false, expert_ffn_pair_kernel, dim3(std::max(2, G & ~1)), dim3(pgemm_threads(true)),
           PR_SMEM, tm_wg, tm_wu, tm_wg1, tm_wu1, tm_xr, tm_hr, tm_wd2, tl, g1, g2, h_ready, dys);
  } else if (R == 8) go(expert_ffn_dynamic_kernel<8>, dy_smem_bytes<8>(), dy_threads<8>());
  else if (R == 16) go(expert_ffn_dynamic_kernel<16>, dy_smem_bytes<16>(), dy_threads<16>());
  else if (R == 32) go(expert_ffn_dynamic_kernel<32>, dy_smem_bytes<32>(), dy_threads<32>());
  else if (R == 64) go(expert_ffn_dynamic_kernel<64>, dy_smem_bytes<64>(), dy_threads<64>());
  else go(expert_ffn_dynamic_kernel<128>, dy_smem_bytes<128>(), dy_threads<128>());
  return launched();
}

// ----------------------------------------------------------------------------- steps alone
// The steps of moe_forward as separate calls (dispatch, row gather, grouped expert FFN over
// row segments, combine), which an expert-parallel layer strings together around its
// exchanges.
}  // extern "C"

namespace moe {
namespace {
struct DispatchLayout {
  size_t chunk_counts = 0, chunk_base = 0, dsync = 0, tile_num = 0, tile_expert = 0;
  size_t tile_row0 = 0, tile_rows = 0, total = 0;
  int nchunks = 0, max_tiles = 0;
};
DispatchLayout dispatch_layout(int T, int E, int k) {
  DispatchLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t P = (size_t)T * k;
  L.nchunks = (int)((P + kDispatchChunk - 1) / kDispatchChunk);
  L.max_tiles = (int)(P / GM_BM) + E;
  L.chunk_counts = take(sizeof(int32_t) * (size_t)L.nchunks * E);
  L.chunk_base = take(sizeof(int32_t) * (size_t)L.nchunks * E);
  L.dsync = take(2 * sizeof(int32_t));
  L.tile_num = take(sizeof(int32_t));
  L.tile_expert = take(sizeof(int32_t) * L.max_tiles);
  L.tile_row0 = take(sizeof(int32_t) * L.max_tiles);
  L.tile_rows = take(sizeof(int32_t) * L.max_tiles);
  L.total = off;
  return L;
}
bool dispatch_shape_ok(int T, int E, int k) {
  return T >= 1 && T <= 1048576 && E >= 1 && E <= 256 && k >= 1 && k <= 8 && k <= E;
}

// Rows of a grouped FFN over contiguous row segments at which CTA pairs take over (its rows
// are loaded by TMA in place, as the dense MLP's are).
constexpr int kPairMinRows = 8 * kDensePairMinTokens;

struct FfnLayout {
  size_t tile_num = 0, tile_expert = 0, tile_row0 = 0, tile_rows = 0, hbuf = 0, counters = 0;
  size_t total = 0;
  int max_tiles = 0, n_counters = 0, bm = 0;
};
FfnLayout ffn_layout(int N, int I, int n_seg) {
  FfnLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.bm = N >= kPairMinRows ? PR_ROWS : GM_BM;
  L.max_tiles = N / L.bm + n_seg;
  L.tile_num = take(sizeof(int32_t));
  L.tile_expert = take(sizeof(int32_t) * L.max_tiles);
  L.tile_row0 = take(sizeof(int32_t) * L.max_tiles);
  L.tile_rows = take(sizeof(int32_t) * L.max_tiles);
  L.hbuf = take(2 * (size_t)N * I);
  L.n_counters = 1 + L.max_tiles + 1;   // unit counter, h-ready per tile, their total
  L.counters = take(sizeof(int32_t) * L.n_counters);
  L.total = off;
  return L;
}
bool ffn_shape_ok(int N, int H, int E, int I, int n_seg) {
  return N >= 1 && N <= 8 * 1048576 && H >= 64 && H <= 16384 && H % 64 == 0 && I >= 64 &&
         I <= 8192 && I % 64 == 0 && E >= 1 && E <= 256 && n_seg >= 1 && n_seg <= kMaxSegments;
}
}  // namespace
}  // namespace moe

extern "C" {

size_t moe_dispatch_workspace_size(int T, int E, int k) {
  if (!dispatch_shape_ok(T, E, k)) return 0;
  return dispatch_layout(T, E, k).total;
}

moe_status_t moe_dispatch(const int32_t* topk_ids, int T, int E, int k, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (T < 0 || E <= 0 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!topk_ids || !counts || !offsets || !perm || !inv || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  if (!dispatch_shape_ok(T, E, k)) return MOE_ERR_UNSUPPORTED;
  const DispatchLayout L = dispatch_layout(T, E, k);
  if (workspace_bytes < L.total) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int P = T * k;
  int32_t* chunk_counts = reinterpret_cast<int32_t*>(ws + L.chunk_counts);
  int32_t* chunk_base = reinterpret_cast<int32_t*>(ws + L.chunk_base);
  int32_t* dsync = reinterpret_cast<int32_t*>(ws + L.dsync);
  int32_t* tile_num = reinterpret_cast<int32_t*>(ws + L.tile_num);
  int32_t* tile_expert = reinterpret_cast<int32_t*>(ws + L.tile_expert);
  int32_t* tile_row0 = reinterpret_cast<int32_t*>(ws + L.tile_row0);
  int32_t* tile_rows = reinterpret_cast<int32_t*>(ws + L.tile_rows);
  const Launch launch{st, true};
  const bool fused = L.nchunks > 1 && L.nchunks <= std::min(kFusedDispatchMaxChunks, d->num_sms);
  if (L.nchunks == 1) {
    launch(false, dispatch_small_kernel, dim3(1), dim3(256), 0, topk_ids, P, E, GM_BM, counts,
           offsets, perm, inv, tile_num, tile_expert, tile_row0, tile_rows, (int32_t*)nullptr, 0);
  } else if (fused) {
    MOE_TRY_CUDA(cudaMemsetAsync(dsync, 0, 2 * sizeof(int32_t), st));
    launch(false, dispatch_fused_kernel, dim3(L.nchunks), dim3(32 * kRankWarps),
           (kRankWarps + 1) * E * sizeof(int), topk_ids, P, E, GM_BM, L.nchunks, chunk_counts,
           chunk_base, counts, offsets, perm, inv, tile_num, tile_expert, tile_row0, tile_rows,
           (int32_t*)nullptr, 0, dsync);
  } else {
    launch(false, dispatch_count_kernel, dim3(L.nchunks), dim3(256), E * sizeof(int), topk_ids,
           P, E, chunk_counts);
    launch(true, dispatch_scan_kernel, dim3(1), dim3(256), 0, (const int32_t*)chunk_counts,
           L.nchunks, E, P, GM_BM, counts, offsets, chunk_base, tile_num, tile_expert, tile_row0,
           tile_rows, (int32_t*)nullptr, 0);
    launch(true, dispatch_rank_kernel, dim3(L.nchunks), dim3(32 * kRankWarps),
           (kRankWarps + 1) * E * sizeof(int), topk_ids, P, E, (const int32_t*)chunk_base, perm,
           inv);
  }
  return launched();
}

moe_status_t moe_gather_rows(const void* x, const int32_t* perm, int n_rows, int T, int H,
                             int k, void* xp, void* stream) {
  if (n_rows < 0 || T < 0 || H <= 0 || k < 1) return MOE_ERR_INVALID_ARG;
  if (n_rows == 0) return MOE_OK;
  if (!x || !perm || !xp || !aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
  if (H % 8 || (long long)T * k > 8ll * 1048576) return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  const Launch launch{static_cast<cudaStream_t>(stream), true};
  const int gsm = std::max(1, d->num_sms) * 8;
  launch(false, gather_rows_kernel, dim3(std::min((n_rows + 7) / 8, gsm)), dim3(256), 0,
         static_cast<const uint4*>(x), perm, n_rows, k, T * k, H / 8, static_cast<uint4*>(xp));
  return launched();
}

size_t moe_expert_ffn_workspace_size(int N, int H, int E, int I, int n_seg) {
  if (!ffn_shape_ok(N, H, E, I, n_seg)) return 0;
  return ffn_layout(N, I, n_seg).total;
}

moe_status_t moe_expert_ffn(const void* xs, int N, const int32_t* seg_rows,
                            const int32_t* seg_expert, int n_seg, const void* w_gate,
                            const void* w_up, const void* w_down, int H, int E, int I, void* out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (N < 0 || n_seg < 0 || H <= 0 || E <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
  if (N == 0 || n_seg == 0) return MOE_OK;
  if (!xs || !seg_rows || !seg_expert || !w_gate || !w_up || !w_down || !out || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(xs) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(out) || !aligned16(workspace))
    return MOE_ERR_INVALID_ARG;
  if (xs == out) return MOE_ERR_INVALID_ARG;
  if (!ffn_shape_ok(N, H, E, I, n_seg)) return MOE_ERR_UNSUPPORTED;
  const FfnLayout L = ffn_layout(N, I, n_seg);
  if (workspace_bytes < L.total) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* tile_num = reinterpret_cast<int32_t*>(ws + L.tile_num);
  int32_t* tile_expert = reinterpret_cast<int32_t*>(ws + L.tile_expert);
  int32_t* tile_row0 = reinterpret_cast<int32_t*>(ws + L.tile_row0);
  int32_t* tile_rows = reinterpret_cast<int32_t*>(ws + L.tile_rows);
  __nv_bfloat16* hbuf = reinterpret_cast<__nv_bfloat16*>(ws + L.hbuf);
  int32_t* ctr = reinterpret_cast<int32_t*>(ws + L.counters);
  const int R = dy_rows(N, 0);
  CUtensorMap tm_wg, tm_wu, tm_wg1, tm_wu1, tm_wd, tm_hr, tm_xr;
  if (!make_map_slabs(&tm_wg, w_gate, I, H, E, 64, 2) ||
      !make_map_slabs(&tm_wu, w_up, I, H, E, 64, 2) ||
      !make_map_slabs(&tm_wg1, w_gate, I, H, E, 64, 1) ||
      !make_map_slabs(&tm_wu1, w_up, I, H, E, 64, 1) ||
      !make_map_slabs(&tm_wd, w_down, H, I, E, 64, L.bm == PR_ROWS ? 2 : 4) ||
      !make_map_2d(&tm_hr, hbuf, I, N, R, 64) || !make_map_2d(&tm_xr, xs, H, N, R, 64))
    return cuda_failed(-1);   // a tensor map could not be encoded
  const Launch launch{st, true};
  launch(false, segment_tiles_kernel, dim3(1), dim3(256), 0, seg_rows, seg_expert, n_seg, N, E,
         L.bm, L.max_tiles, tile_num, tile_expert, tile_row0, tile_rows, ctr, L.n_counters);
  // the rows are read in place (no permutation) by TMA: sorted row r of the A operand is xs[r]
  TileList tl{tile_num, tile_expert, tile_row0, tile_rows, 0,
              nullptr,  1,           static_cast<const __nv_bfloat16*>(xs), H, N};
  tl.a_tma = 1;
  const PGemm g1{(I + 127) / 128, H, I, hbuf, I, nullptr, nullptr};
  const PGemm g2{(H + 255) / 256, I, H, out, H, nullptr, nullptr};
  int32_t* h_ready = ctr + 1;
  const DyState dys{ctr};
  const int G = std::min(std::max(1, d->num_sms), kMaxGemmCtas);
  auto go = [&](auto kernel, int smem, int threads) {
    launch(true, kernel, dim3(G), dim3(threads), smem, tm_wg, tm_wu, tm_wg1, tm_wu1, tm_xr, tm_hr,
           tm_wd, tl, g1, g2, h_ready, dys);
  };
  if (L.bm == PR_ROWS)
    launch(true, expert_ffn_pair_kernel, dim3(std::max(2, G & ~1)), dim3(pgemm_threads(true)),
           PR_SMEM, tm_wg, tm_wu, tm_wg1, tm_wu1, tm_xr, tm_hr, tm_wd, tl, g1, g2, h_ready, dys);
  else if (R == 8) go(expert_ffn_dynamic_kernel<8>, dy_smem_bytes<8>(), dy_threads<8>());
  else if (R == 16) go(expert_ffn_dynamic_kernel<16>, dy_smem_bytes<16>(), dy_threads<16>());
  else if (R == 32) go(expert_ffn_dynamic_kernel<32>, dy_smem_bytes<32>(), dy_threads<32>());
  else if (R == 64) go(expert_ffn_dynamic_kernel<64>, dy_smem_bytes<64>(), dy_threads<64>());
  else go(expert_ffn_dynamic_kernel<128>, dy_smem_bytes<128>(), dy_threads<128>());
  return launched();
}

moe_status_t moe_combine(const void* o, const int32_t* inv, const float* topk_weights, int T,
                         int k, int H, int row_lo, int row_hi, unsigned flags, void* y,
                         void* stream) {
  if (T < 0 || k < 1 || k > 8 || H <= 0) return MOE_ERR_INVALID_ARG;
  if (flags & ~(unsigned)MOE_COMBINE_F32) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!o || !inv || !topk_weights || !y || !aligned16(o) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  if (row_lo < 0 || row_hi < row_lo || (long long)row_hi > (long long)T * k)
    return MOE_ERR_INVALID_ARG;
  if (H % 8 || (long long)T * k > 8ll * 1048576) return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  const Launch launch{static_cast<cudaStream_t>(stream), true};
  const int gsm = std::max(1, d->num_sms) * 8;
  const long long citems = (long long)T * ((H / 8 + kCombineChunkVec - 1) / kCombineChunkVec);
  const dim3 grid((int)std::min<long long>((citems + 7) / 8, gsm));
  if (flags & MOE_COMBINE_F32)
    launch(false, combine_kernel<true>, grid, dim3(256), 0, static_cast<const uint4*>(o), inv,
           topk_weights, T, k, H / 8, row_lo, row_hi, y);
  else
    launch(false, combine_kernel<false>, grid, dim3(256), 0, static_cast<const uint4*>(o), inv,
           topk_weights, T, k, H / 8, row_lo, row_hi, y);
  return launched();
}

// ----------------------------------------------------------------------------- NVFP4
size_t moe_nvfp4_quantize_workspace_size(int E) {
  return E >= 1 ? align256(sizeof(unsigned) * (size_t)E) : 0;
}

moe_status_t moe_nvfp4_quantize_weights(const void* w, int E, int K, int N, uint8_t* codes,
                                        uint8_t* scales, float* ts, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (E <= 0 || K <= 0 || N <= 0) return MOE_ERR_INVALID_ARG;
  if (!w || !codes || !scales || !ts || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  if (K % 64 || K > 16384 || N > (1 << 20) || E > 65535) return MOE_ERR_UNSUPPORTED;
  if (workspace_bytes < moe_nvfp4_quantize_workspace_size(E)) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* amax = static_cast<unsigned*>(workspace);
  MOE_TRY_CUDA(cudaMemsetAsync(amax, 0, sizeof(unsigned) * E, st));
  const long long per = (long long)K * N;
  const Launch launch{st, false};
  launch(false, nvfp4_amax_kernel, dim3((unsigned)std::min<long long>((per + 2047) / 2048, 1024), E),
         dim3(256), 0, static_cast<const __nv_bfloat16*>(w), per, amax);
  launch(false, nvfp4_weight_quant_kernel, dim3(((N + 127) / 128 * 128 + 255) / 256, K / 16, E),
         dim3(256), 0,
         static_cast<const __nv_bfloat16*>(w), K, N, (const unsigned*)amax, codes, scales, ts);
  return launched();
}

moe_status_t moe_nvfp4_quantize_rows(const void* x, int rows, int K, float ts, uint8_t* codes,
                                     uint8_t* scales, void* stream) {
  if (rows < 0 || K <= 0 || !(ts > 0.f)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  if (K % 16 || (long long)rows * K > (1ll << 34)) return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  const Launch launch{static_cast<cudaStream_t>(stream), false};
  const long long groups = (long long)rows * (K / 16);
  launch(false, nvfp4_rows_quant_kernel,
         dim3((unsigned)std::min<long long>((groups + 255) / 256, (long long)d->num_sms * 16)),
         dim3(256), 0, static_cast<const __nv_bfloat16*>(x), (long long)rows, K, ts, codes, scales);
  return launched();
}

namespace {
constexpr unsigned kFp4Flags = MOE_FLAG_NO_RENORM | MOE_FLAG_ROUTER_FP64 | MOE_FLAG_ROUTER_SCREEN |
                               MOE_FLAG_PROFILE_STAGES;
// The forward's own layout, then (256-byte aligned): sorted x codes [P][H/2], x scale lines
// [H/64][P + 16][16], h codes [P][I/2], h scale lines [I/64][P + 16][16], the FFN counters
// (unit counter, h_ready per tile).
struct Fp4Layout {
  size_t xq, xl, hq, hl, ctr, total;
  int n_ctr;
};
Fp4Layout fp4_layout(size_t at, int T, int H, int E, int I, int k) {
  Fp4Layout F;
  const size_t P = (size_t)T * k, Pp = P + 16;
  auto take = [&](size_t bytes) {
    const size_t o = at;
    at = align256(at + bytes);
    return o;
  };
  F.xq = take(P * H / 2);
  F.xl = take((size_t)(H / 64) * Pp * 16);
  F.hq = take(P * I / 2);
  F.hl = take((size_t)(I / 64) * Pp * 16);
  F.n_ctr = 1 + std::min(E, (int)P);
  F.ctr = take(sizeof(int) * F.n_ctr);
  F.total = at;
  return F;
}
bool fp4_shape_ok(int T, int H, int E, int I, int k) {
  return shape_supported(T, H, E, I, k, true) && T <= FP4_MAX_ROWS;
}
}  // namespace

size_t moe_nvfp4_workspace_size(int T, int H, int E, int I, int k, unsigned flags) {
  if ((flags & ~kFp4Flags) || !flags_ok(flags) || !fp4_shape_ok(T, H, E, I, k) ||
      !forced_path_ok(E, flags))
    return 0;
  return fp4_layout(make_layout(T, H, E, I, k, flags, true).total, T, H, E, I, k).total;
}

moe_status_t moe_forward_nvfp4(const void* x, const void* w_router, const float* router_bias,
                               const moe_nvfp4_weights_t* w, int T, int H, int E, int I, int k,
                               unsigned flags, float act_scale_x, float act_scale_h, void* y,
                               const moe_aux_t* aux, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (T < 0 || H <= 0 || E <= 0 || I <= 0 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if ((flags & ~kFp4Flags) || !flags_ok(flags)) return MOE_ERR_INVALID_ARG;
  if (!(act_scale_x > 0.f) || !(act_scale_h > 0.f)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !w || !y || !workspace || !w->gate_codes || !w->gate_scales ||
      !w->gate_ts || !w->up_codes || !w->up_scales || !w->up_ts || !w->down_codes ||
      !w->down_scales || !w->down_ts)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(y) || !aligned16(workspace) ||
      !aligned16(w->gate_codes) || !aligned16(w->up_codes) || !aligned16(w->down_codes) ||
      !aligned16(w->gate_scales) || !aligned16(w->up_scales) || !aligned16(w->down_scales))
    return MOE_ERR_INVALID_ARG;
  if (x == y) return MOE_ERR_INVALID_ARG;
  if (!fp4_shape_ok(T, H, E, I, k) || !forced_path_ok(E, flags)) return MOE_ERR_UNSUPPORTED;
  const Layout L = make_layout(T, H, E, I, k, flags, true);
  const Fp4Layout F = fp4_layout(L.total, T, H, E, I, k);
  if (workspace_bytes < F.total) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int P = T * k;
  int32_t* ids = (aux && aux->topk_ids) ? aux->topk_ids : reinterpret_cast<int32_t*>(ws + L.ids);
  float* wts = (aux && aux->topk_weights) ? aux->topk_weights : reinterpret_cast<float*>(ws + L.wts);
  int32_t* counts =
      (aux && aux->expert_counts) ? aux->expert_counts : reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = (aux && aux->expert_offsets) ? aux->expert_offsets
                                                  : reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm = (aux && aux->perm) ? aux->perm : reinterpret_cast<int32_t*>(ws + L.perm);
  unsigned* stats = (aux && aux->router_stats) ? aux->router_stats
                                               : reinterpret_cast<unsigned*>(ws + L.stats);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
  int32_t* tile_num = reinterpret_cast<int32_t*>(ws + L.tile_num);
  int32_t* tile_expert = reinterpret_cast<int32_t*>(ws + L.tile_expert);
  int32_t* tile_row0 = reinterpret_cast<int32_t*>(ws + L.tile_row0);
  int32_t* tile_rows = reinterpret_cast<int32_t*>(ws + L.tile_rows);
  __nv_bfloat16* obuf = reinterpret_cast<__nv_bfloat16*>(ws + L.obuf);

  Profiler prof{d, st, (flags & MOE_FLAG_PROFILE_STAGES) != 0};
  prof.mark();
  const RouteBufs rb{ids, wts, stats, counts, offsets, perm, inv};
  if (const moe_status_t rs = route_and_dispatch(x, w_router, router_bias, T, H, E, k, flags, rb,
                                                 ws, L, *d, st, prof, false);
      rs != MOE_OK)
    return rs;
  // 3. the routed x rows in sorted order, quantised (and the FFN's counters zeroed);
  // 4. GEMM-1 + GEGLU + h quantised, GEMM-2: one persistent tensor-core launch
  const Launch launch{st, !prof.on};
  const int Pp = P + 16;
  CUtensorMap tm_wg, tm_wu, tm_wd, tm_xq, tm_hq, tm_xl, tm_hl;
  if (!make_map_u8_3d(&tm_wg, w->gate_codes, H / 2, I, E) ||
      !make_map_u8_3d(&tm_wu, w->up_codes, H / 2, I, E) ||
      !make_map_u8_3d(&tm_wd, w->down_codes, I / 2, H, E) ||
      !make_map_u8_2d(&tm_xq, ws + F.xq, H / 2, P, F4_BN) ||
      !make_map_u8_2d(&tm_hq, ws + F.hq, I / 2, P, F4_BN) ||
      !make_map_lines(&tm_xl, ws + F.xl, Pp, H / 64) ||
      !make_map_lines(&tm_hl, ws + F.hl, Pp, I / 64))
    return cuda_failed(-1);
  int* ctr = reinterpret_cast<int*>(ws + F.ctr);
  const int items = Pp * (H / 64);
  launch(true, nvfp4_rows_sorted_kernel, dim3(std::min((items + 127) / 128, d->num_sms * 4)),
         dim3(128), 0, static_cast<const __nv_bfloat16*>(x), (const int32_t*)perm, k, T, P, H,
         act_scale_x, ws + F.xq, reinterpret_cast<uint4*>(ws + F.xl),
         reinterpret_cast<uint4*>(ws + F.hl), (I / 64) * Pp, ctr, F.n_ctr);
  Fp4Ffn fa;
  fa.sfa_g = w->gate_scales;
  fa.sfa_u = w->up_scales;
  fa.sfa_d = w->down_scales;
  fa.ts_g = w->gate_ts;
  fa.ts_u = w->up_ts;
  fa.ts_d = w->down_ts;
  fa.x_lines = ws + F.xl;
  fa.hq = ws + F.hq;
  fa.h_lines = ws + F.hl;
  fa.Pp = Pp;
  fa.O = obuf;
  fa.tile_num = tile_num;
  fa.tile_expert = tile_expert;
  fa.tile_row0 = tile_row0;
  fa.tile_rows = tile_rows;
  fa.next = ctr;
  fa.h_ready = ctr + 1;
  fa.H = H;
  fa.I = I;
  fa.E = E;
  fa.sx = act_scale_x;
  fa.sh = act_scale_h;
  launch(true, nvfp4_ffn_kernel, dim3(d->num_sms), dim3(F4_THREADS), F4_SMEM, tm_wg, tm_wu, tm_wd,
         tm_xq, tm_hq, tm_xl, tm_hl, fa);
  if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
  prof.mark();
  // 5. combine
  const int gsm = std::max(1, d->num_sms) * 8;
  const long long citems = (long long)T * ((H / 8 + kCombineChunkVec - 1) / kCombineChunkVec);
  launch(true, combine_kernel<false>, dim3((int)std::min<long long>((citems + 7) / 8, gsm)),
         dim3(256), 0, reinterpret_cast<const uint4*>(obuf), (const int32_t*)inv,
         (const float*)wts, T, k, H / 8, 0, P, y);
  if (const moe_status_t ls = launched(); ls != MOE_OK) return ls;
  prof.mark();
  prof.finish();
  return MOE_OK;
}

moe_status_t moe_route_static(const void* x, const void* w_router, const float* router_bias,
                              int T, int H, int E, int k, unsigned flags, int32_t* topk_ids,
                              float* topk_weights, void* stream) {
  if (T < 0 || H <= 0 || E <= 0 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (!flags_ok(flags) || (flags & (MOE_FLAG_ROUTER_SCREEN | MOE_FLAG_PROFILE_STAGES)))
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !topk_ids || !topk_weights) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
  if (!shape_supported(T, H, E, 64, k, false)) return MOE_ERR_UNSUPPORTED;
  const unsigned f = flags | MOE_FLAG_ROUTER_FP64;   // fp64 logits: no screen buffers
  const Layout L = make_layout(T, H, E, 64, k, f, false);
  if (L.total > kStaticScratchBytes) return MOE_ERR_NO_WORKSPACE;
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d) return MOE_ERR_CUDA;
  t_kernels = 0;
  void* scratch = nullptr;
  {
    // First call on this device: look up the array's device address (with this device
    // current).  Later calls reuse it.
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_static_scratch_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
      g_static_scratch_ptr[dev] = p;
    }
    scratch = g_static_scratch_ptr[dev];
  }
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  return launch_router(static_cast<const __nv_bfloat16*>(x),
                       static_cast<const __nv_bfloat16*>(w_router), router_bias, T, H, E, k, f,
                       topk_ids, topk_weights, reinterpret_cast<unsigned*>(ws + L.stats), ws, L,
                       *d, static_cast<cudaStream_t>(stream), true);
}

moe_status_t moe_sync_status(void* stream) {
  MOE_TRY_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  unsigned w = 0;
  MOE_TRY_CUDA(cudaMemcpyFromSymbol(&w, g_error_word, sizeof w));
  if (w) {
    const unsigned zero = 0;
    MOE_TRY_CUDA(cudaMemcpyToSymbol(g_error_word, &zero, sizeof zero));
  }
  if (w & MOE_DEVERR_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (w) return MOE_ERR_CUDA;
  return MOE_OK;
}

const char* moe_ffn_kernel_name(int T, unsigned flags) {
  if (T < 1 || !flags_ok(flags)) return "";
  if (flags & MOE_FLAG_DECODE_TILES)
    return T <= kDecodeMaxTokens ? "grouped_gemm_decode_kernel<EPI_GEGLU>+<EPI_STORE>" : "";
  if (flags & MOE_FLAG_UNFUSED_FFN)
    return "grouped_gemm_persistent_kernel<4,EPI_GEGLU,4,1,0>+<4,EPI_STORE,4,0,0>";
  if (flags & MOE_FLAG_FUSED_FFN)
    return T <= PG_SMALL_ROWS ? "grouped_gemm_persistent_kernel<6,EPI_GEGLU,4,1,1,1>"
                              : "grouped_gemm_persistent_kernel<4,EPI_GEGLU,4,1,1>";
  if (use_pair_ffn(T, flags))
    return use_row_copy(T, flags) ? "expert_ffn_pair_kernel (rows copied)" : "expert_ffn_pair_kernel";
  if (use_row_copy(T, flags)) return "expert_ffn_dynamic_kernel<128> (rows copied)";
  switch (dy_rows(T, flags)) {
    case 8: return "expert_ffn_dynamic_kernel<8>";
    case 16: return "expert_ffn_dynamic_kernel<16>";
    case 32: return "expert_ffn_dynamic_kernel<32>";
    case 64: return "expert_ffn_dynamic_kernel<64>";
    default: return "expert_ffn_dynamic_kernel<128>";
  }
}

int moe_last_cuda_error(void) { return t_last_cuda_error; }

int moe_last_kernel_count(void) { return t_kernels; }

const char* moe_cuda_error_name(int code) {
  if (code == 0) return "";
  if (code == -1) return "tensor map encoding failed";
  return cudaGetErrorName(static_cast<cudaError_t>(code));
}

int moe_last_stage_times(float* ms, int n) {
  int dev = 0;
  DeviceState* d = device_state(&dev);
  if (!d || d->n_profiled < 0) return -1;
  const int ns = d->n_profiled;
  if (cudaEventSynchronize(d->ev[ns]) != cudaSuccess) return -1;
  for (int i = 0; i < ns && i < n; ++i) {
    float t = 0.f;
    cudaEventElapsedTime(&t, d->ev[i], d->ev[i + 1]);
    ms[i] = t;
  }
  return ns;
}

const char* moe_stage_name(int i) {
  return (i >= 0 && i < kNumStages) ? kStageNames[i] : "";
}

moe_status_t moe_debug_set_wait_limit_ns(unsigned long long ns) {
  const unsigned long long v = ns ? ns : 2000000000ull;
  return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof v) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_debug_unsatisfied_wait(void* stream) {
  unsatisfied_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>();
  return launched();
}

}  // extern "C"
