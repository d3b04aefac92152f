// nvfp4.cuh -- NVFP4 quantisation (4-bit E2M1 elements, one E4M3 scale per 16 consecutive
// elements along the reduction axis, one fp32 scale per tensor):
// the checkpoint format of Gemma-4-26B-A4B-NVFP4 ("4-bit float, group_size=16" for weights
// and activations, Gemma-4-26B-A4B-NVFP4 Ascend verification report §2.3 量化配置 (NVFP4)).
//
// Value of element i of group g: e2m1(code_i) * e4m3(scale_g) * tensor_scale.
// Quantisation of a group v[16] (every step one IEEE fp32 operation, round to nearest even):
//   amax = max |v|;  s = (amax / 6) / ts;  s8 = E4M3(s) (saturating);  S = e4m3(s8) * ts;
//   code_i = E2M1(v_i / S) (saturating; sign kept), or 0 when S == 0.
//
// Weight layout (the layout of a Linear layer's weight, out x in, in contiguous): a projection
// with reduction depth K and N outputs is codes [E][N][K/2] (byte b of a row holds elements 2b
// in its low nibble and 2b+1 in its high nibble), scales in the blocked layout of
// nvfp4_scale_offset (E4M3 bytes), ts [E].
//
// This file holds the quantisers; the decode FFN on the tensor cores is nvfp4_mma.cuh.
#pragma once
#include <cuda_fp16.h>
#include "ptx.cuh"

namespace moe {

constexpr int FP4_MAX_ROWS = 16;      // rows per expert tile (batches of at most 16 tokens)

// ---------------------------------------------------------------- format conversions
__device__ __forceinline__ uint32_t e4m3_round_sat(float v) {   // -> byte
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(d) : "f"(v));
  return d & 0xffu;
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t h2;
  const uint16_t pair = static_cast<uint16_t>(b | (b << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xffffu)));
}
// Two values -> one byte: `lo` in the low nibble, `hi` in the high nibble.
__device__ __forceinline__ uint32_t e2m1x2_round_sat(float lo, float hi) {
  uint32_t d;
  asm("{.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(d)
      : "f"(hi), "f"(lo));
  return d & 0xffu;
}
// One byte of two codes -> f16x2 (low nibble in the low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t d;
  asm("{.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(d) : "r"(byte));
  return d;
}
// Quantise one group of 16 fp32 values: packed codes (8 bytes), the scale byte, and the
// group's values code * e4m3(scale) as 8 f16x2 words (exact; the tensor scale left out).
__device__ __forceinline__ void nvfp4_quantize16(const float (&v)[16], float ts, uint32_t (&codes)[2],
                                                 uint32_t& scale, uint32_t (&dq)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float s = __fdiv_rn(__fdiv_rn(amax, 6.0f), ts);
  scale = e4m3_round_sat(s);
  const float sv = e4m3_to_f32(scale);
  const float S = __fmul_rn(sv, ts);
  codes[0] = codes[1] = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t b = S == 0.f ? 0u : e2m1x2_round_sat(__fdiv_rn(v[2 * i], S), __fdiv_rn(v[2 * i + 1], S));
    codes[i >> 2] |= b << (8 * (i & 3));
    // dequantised (without ts): code values times the group scale, exact in f16
    const uint32_t cw = e2m1x2_to_f16x2(b);
    const __half2 r2 = __hmul2(*reinterpret_cast<const __half2*>(&cw), __float2half2_rn(sv));
    dq[i] = *reinterpret_cast<const uint32_t*>(&r2);
  }
}

// ---------------------------------------------------------------- weight quantiser
// amax_bits[e] = max |w| over expert e (fp32 bits; non-negative floats order like their bits).
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const __nv_bfloat16* __restrict__ w,
                                                        long long per_expert,
                                                        unsigned* __restrict__ amax_bits) {
  const int e = blockIdx.y;
  const __nv_bfloat16* we = w + (size_t)e * per_expert;
  float m = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < per_expert;
       i += (long long)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(__bfloat162float(we[i])));
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + e, __float_as_uint(m));
}

// Byte offset of the scale of (row n, group g) of expert e in the blocked scale layout: one
// 512-byte block per (expert, 128 rows, 4 groups), blocks ordered [e][n / 128][g / 4]; in a
// block, rows n % 32 are 16-byte lines holding (row n % 32 + 32 i, group 4 (g / 4) + j) at byte
// 4 i + j.  This is the tensor cores' scale-factor layout: a block is what one 64-deep MMA of
// 128 rows reads, and a plain copy moves it into tensor memory.
__host__ __device__ inline size_t nvfp4_scale_offset(int e, int n, int g, int N, int K) {
  const size_t nb = (size_t)(N + 127) / 128, kb = (size_t)K / 64;
  return (((size_t)e * nb + n / 128) * kb + g / 4) * 512 + 16 * (n % 32) + 4 * ((n % 128) / 32) +
         (g % 4);
}
__host__ __device__ inline size_t nvfp4_scale_bytes(int E, int N, int K) {
  return (size_t)E * ((N + 127) / 128) * (K / 64) * 512;
}

// Weight w [E][K][N] (N contiguous, the library's bf16 layout) -> codes [E][N][K/2], blocked
// scales (rows N .. up to the next multiple of 128 get scale 0), ts[e] = amax_e / (6 * 448).
// Thread per (n, group of 16 along K); grid.x covers the padded rows.
__global__ void __launch_bounds__(256) nvfp4_weight_quant_kernel(
    const __nv_bfloat16* __restrict__ w, int K, int N, const unsigned* __restrict__ amax_bits,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ ts_out) {
  const int e = blockIdx.z;
  const float ts = __fdiv_rn(__uint_as_float(amax_bits[e]), 2688.0f);
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;
  if (n == 0 && g == 0) ts_out[e] = ts;
  if (n >= (N + 127) / 128 * 128) return;
  if (n >= N) {
    scales[nvfp4_scale_offset(e, n, g, N, K)] = 0;
    return;
  }
  const __nv_bfloat16* we = w + (size_t)e * K * N;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __bfloat162float(we[(size_t)(16 * g + i) * N + n]);
  uint32_t c[2], s, dq[8];
  nvfp4_quantize16(v, ts, c, s, dq);
  uint2* dst = reinterpret_cast<uint2*>(codes + ((size_t)e * N + n) * (K / 2) + 8 * g);
  *dst = make_uint2(c[0], c[1]);
  scales[nvfp4_scale_offset(e, n, g, N, K)] = static_cast<uint8_t>(s);
}

// Rows of bf16 activations [rows][K] -> codes [rows][K/2], scales [rows][K/16] with a fixed
// tensor scale (the activation quantiser of the layer, as a call of its own).
__global__ void __launch_bounds__(256) nvfp4_rows_quant_kernel(
    const __nv_bfloat16* __restrict__ x, long long rows, int K, float ts,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const long long groups = rows * (K / 16);
  for (long long gi = (long long)blockIdx.x * blockDim.x + threadIdx.x; gi < groups;
       gi += (long long)gridDim.x * blockDim.x) {
    float v[16];
    const uint4* src = reinterpret_cast<const uint4*>(x + gi * 16);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 r = src[h];
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        v[8 * h + 2 * i] = f.x;
        v[8 * h + 2 * i + 1] = f.y;
      }
    }
    uint32_t c[2], s, dq[8];
    nvfp4_quantize16(v, ts, c, s, dq);
    reinterpret_cast<uint2*>(codes)[gi] = make_uint2(c[0], c[1]);
    scales[gi] = static_cast<uint8_t>(s);
  }
}

// ---------------------------------------------------------------- activations, sorted
// The expert FFN's activation operand: the routed rows in expert-sorted order (row j holds
// the token of pair perm[j]) quantised with tensor scale ts -> codes [P][K/2] and scale LINES:
// lines [K/64][Pp][16 bytes], line (kb, j) = the 4 scales of row j's groups 4 kb .. 4 kb + 3,
// then 12 zero bytes (the rows 0-15 of a tensor-core scale block, so that 16 consecutive rows
// of one K block are one 256-byte copy).  Pp = P + 16: rows P .. P + 15 are zero lines.
// Also zeroes h_lines ([I/64][Pp][16], filled in later by the FFN's GEMM-1 epilogue) and the
// FFN's counters.  One thread per (row, 64-element K block).
__global__ void __launch_bounds__(256) nvfp4_rows_sorted_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ perm, int k, int T, int P,
    int K, float ts, uint8_t* __restrict__ codes, uint4* __restrict__ lines,
    uint4* __restrict__ h_lines, int n_h_lines, int* __restrict__ counters, int n_ctr) {
  pdl_trigger();
  pdl_wait();
  const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_ctr; i += blockDim.x) counters[i] = 0;
  for (int i = tid; i < n_h_lines; i += nth) h_lines[i] = make_uint4(0, 0, 0, 0);
  const int nkb = K / 64, Pp = P + 16;
  for (int gi = tid; gi < Pp * nkb; gi += nth) {
    const int j = gi / nkb, kb = gi - j * nkb;
    uint32_t sc4 = 0;
    if (j < P) {
      const int q = perm[j];
      const bool ok = (unsigned)q < (unsigned)(T * k);
      if (!ok) raise_error(MOE_DEVERR_BAD_INDEX);
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(ok ? q / k : 0) * K + 64 * kb);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float v[16];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint4 r = ok ? __ldg(src + 2 * g + hh) : make_uint4(0, 0, 0, 0);
          const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(pr[i]);
            v[8 * hh + 2 * i] = f.x;
            v[8 * hh + 2 * i + 1] = f.y;
          }
        }
        uint32_t c[2], sc, dq[8];
        nvfp4_quantize16(v, ts, c, sc, dq);
        *reinterpret_cast<uint2*>(codes + (size_t)j * (K / 2) + 32 * kb + 8 * g) =
            make_uint2(c[0], c[1]);
        sc4 |= sc << (8 * g);
      }
    }
    lines[(size_t)kb * Pp + j] = make_uint4(sc4, 0, 0, 0);
  }
}

}  // namespace moe
