// nvfp4.cuh -- the expert FFN with NVFP4 weights and activations (4-bit E2M1 elements, one
// E4M3 scale per 16 consecutive elements along the reduction axis, one fp32 scale per tensor):
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
// in its low nibble and 2b+1 in its high nibble), scales [E][N][K/16] (E4M3 bytes), ts [E].
//
// The decode FFN (at most 16 rows per expert tile) is a weight stream: every weight element
// is used by about one row, so it runs on the CUDA cores with 16-byte coalesced loads, one
// cvt per two codes and one fp32 FMA per element and row (products of two NVFP4 values are
// exact in fp32; fma.rn.f32.f16 keeps them so).  x is quantised by each GEMM-1 CTA as it
// stages the tile's rows, h (written in fp32 by GEMM-1) by each GEMM-2 CTA as it stages them:
// the same decisions in every CTA.
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
// acc + a.lo * b.lo + a.hi * b.hi, each product exact, two fp32 roundings.
__device__ __forceinline__ float fma2_f16_f32(uint32_t a, uint32_t b, float acc) {
  float d;
  asm("{.reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %3;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "=f"(d)
      : "r"(a), "r"(b), "f"(acc));
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

// Weight w [E][K][N] (N contiguous, the library's bf16 layout) -> codes [E][N][K/2], scales
// [E][N][K/16], ts[e] = amax_e / (6 * 448).  Thread per (n, group of 16 along K).
__global__ void __launch_bounds__(256) nvfp4_weight_quant_kernel(
    const __nv_bfloat16* __restrict__ w, int K, int N, const unsigned* __restrict__ amax_bits,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ ts_out) {
  const int e = blockIdx.z;
  const float ts = __fdiv_rn(__uint_as_float(amax_bits[e]), 2688.0f);
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;
  if (n == 0 && g == 0) ts_out[e] = ts;
  if (n >= N) return;
  const __nv_bfloat16* we = w + (size_t)e * K * N;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __bfloat162float(we[(size_t)(16 * g + i) * N + n]);
  uint32_t c[2], s, dq[8];
  nvfp4_quantize16(v, ts, c, s, dq);
  uint2* dst = reinterpret_cast<uint2*>(codes + ((size_t)e * N + n) * (K / 2) + 8 * g);
  *dst = make_uint2(c[0], c[1]);
  scales[((size_t)e * N + n) * (K / 16) + g] = static_cast<uint8_t>(s);
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

// ---------------------------------------------------------------- GEMM-1 (+ GEGLU)
// Both FFN kernels stream weight rows of codes with 16-byte loads: every lane issues all its
// loads of a row block first, so a warp has the whole block in flight, and only then waits
// -- while the CTA stages its activation rows in shared memory.  Lane l takes the chunks of
// 32 elements l, l + 32, l + 64 of a row (FP4_CHUNKS per lane per block).
constexpr int FP4_CHUNKS = 3;
constexpr int FP4_G1_FEATS = 8;     // GEMM-1: one warp per feature, 8 features per CTA
constexpr int FP4_G2_PER_WARP = 8;  // GEMM-2: 8 output columns per warp, 64 per CTA

// Staged rows in shared memory: K/2 f16x2 words per row, chunk ch (32 elements) at words
// 16 ch .. 16 ch + 15 as four pieces of 8 elements; piece p sits at slot p ^ ((ch >> 1) & 3),
// so that 8 lanes reading the same piece of 8 consecutive chunks hit 32 different banks.
__device__ __forceinline__ int fp4_piece_word(int ch, int p) { return 16 * ch + 4 * (p ^ ((ch >> 1) & 3)); }

// Stage rows of activations (row_of(r, g, v) gives group g of row r as 16 fp32 values)
// quantised as NVFP4 with tensor scale ts into xs: words of code * group scale (one thread
// per group; group g is pieces 2 (g & 1) and 2 (g & 1) + 1 of chunk g / 2).
template <typename RowOf>
__device__ __forceinline__ void nvfp4_stage_rows(uint32_t* xs, int rows, int K, float ts,
                                                 RowOf row_of) {
  const int ng = K / 16;
  for (int gi = threadIdx.x; gi < rows * ng; gi += blockDim.x) {
    const int r = gi / ng, g = gi - r * ng;
    float v[16];
    row_of(r, g, v);
    uint32_t c[2], sc, dq[8];
    nvfp4_quantize16(v, ts, c, sc, dq);
    uint32_t* row = xs + (size_t)r * (K / 2);
    const int ch = g >> 1, p = 2 * (g & 1);
    *reinterpret_cast<uint4*>(row + fp4_piece_word(ch, p)) = make_uint4(dq[0], dq[1], dq[2], dq[3]);
    *reinterpret_cast<uint4*>(row + fp4_piece_word(ch, p + 1)) = make_uint4(dq[4], dq[5], dq[6], dq[7]);
  }
}

// One chunk (32 elements: two groups) of a weight row against `rows` staged rows: acc[r] +=
// scale_g * sum over the group of (code * x) for both groups, exact products.
template <int MAXR>
__device__ __forceinline__ void nvfp4_chunk(const uint4& c, uint32_t sc2, const uint32_t* xs,
                                            int K, int ch, int rows, float (&acc)[MAXR]) {
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int sub = 0; sub < 2; ++sub) {
    uint32_t w2[8];
#pragma unroll
    for (int b = 0; b < 8; ++b)
      w2[b] = e2m1x2_to_f16x2((cw[2 * sub + (b >> 2)] >> (8 * (b & 3))) & 0xffu);
    const float sf = e4m3_to_f32((sc2 >> (8 * sub)) & 0xffu);
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
      if (r < rows) {
        const uint32_t* row = xs + (size_t)r * (K / 2);
        const uint4 xa = *reinterpret_cast<const uint4*>(row + fp4_piece_word(ch, 2 * sub));
        const uint4 xb = *reinterpret_cast<const uint4*>(row + fp4_piece_word(ch, 2 * sub + 1));
        const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        float p = 0.f;
#pragma unroll
        for (int b = 0; b < 8; ++b) p = fma2_f16_f32(w2[b], xw[b], p);
        acc[r] = fmaf(sf, p, acc[r]);
      }
    }
  }
}

// Grid: (tile, group of 8 features); warp w computes feature f = 8 blockIdx.y + w of every
// row of the tile: h[row][f] = gelu_tanh(g) u (fp32; the GEMM-2 CTAs quantise it).
template <int MAXR>
__global__ void __launch_bounds__(32 * FP4_G1_FEATS) nvfp4_gemm1_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ perm, int k, int T,
    const int32_t* __restrict__ tile_num, const int32_t* __restrict__ tile_expert,
    const int32_t* __restrict__ tile_row0, const int32_t* __restrict__ tile_rows,
    const uint8_t* __restrict__ gc, const uint8_t* __restrict__ gs, const float* __restrict__ gts,
    const uint8_t* __restrict__ uc, const uint8_t* __restrict__ us, const float* __restrict__ uts,
    int H, int I, float sx, float* __restrict__ h32) {
  pdl_trigger();
  pdl_wait();
  if (*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT) return;
  const int tile = blockIdx.x;
  if (tile >= *tile_num) return;
  const int e = tile_expert[tile], row0 = tile_row0[tile];
  const int rows = min(tile_rows[tile], MAXR);
  extern __shared__ __align__(16) uint8_t fsm[];
  uint32_t* xs = reinterpret_cast<uint32_t*>(fsm);          // [rows][H/2] f16x2
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.y * FP4_G1_FEATS + warp;
  const int hw = H / 2, ng = H / 16, nch = H / 32;
  const uint4* grow = reinterpret_cast<const uint4*>(gc + ((size_t)e * I + f) * hw);
  const uint4* urow = reinterpret_cast<const uint4*>(uc + ((size_t)e * I + f) * hw);
  const uint16_t* gsr = reinterpret_cast<const uint16_t*>(gs + ((size_t)e * I + f) * ng);
  const uint16_t* usr = reinterpret_cast<const uint16_t*>(us + ((size_t)e * I + f) * ng);
  float accg[MAXR], accu[MAXR];
#pragma unroll
  for (int r = 0; r < MAXR; ++r) accg[r] = accu[r] = 0.f;
  for (int cb = 0; cb < nch; cb += 32 * FP4_CHUNKS) {
    uint4 cg[FP4_CHUNKS], cu[FP4_CHUNKS];
    uint32_t sg[FP4_CHUNKS], su[FP4_CHUNKS];
#pragma unroll
    for (int j = 0; j < FP4_CHUNKS; ++j) {     // the block's loads, all issued first
      const int ch = cb + lane + 32 * j;
      if (f < I && ch < nch) {
        cg[j] = __ldcs(grow + ch);
        cu[j] = __ldcs(urow + ch);
        sg[j] = __ldcs(gsr + ch);
        su[j] = __ldcs(usr + ch);
      }
    }
    if (cb == 0) {
      // stage the tile's x rows (through perm) while the first loads are in flight
      nvfp4_stage_rows(xs, rows, H, sx, [&](int r, int g, float (&v)[16]) {
        const int q = perm[row0 + r];
        if ((unsigned)q >= (unsigned)(T * k)) {
          raise_error(MOE_DEVERR_BAD_INDEX);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0.f;
          return;
        }
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(q / k) * H + 16 * g);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint4 rr = __ldg(src + hh);
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&rr);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 fv = __bfloat1622float2(p[i]);
            v[8 * hh + 2 * i] = fv.x;
            v[8 * hh + 2 * i + 1] = fv.y;
          }
        }
      });
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < FP4_CHUNKS; ++j) {
      const int ch = cb + lane + 32 * j;
      if (f < I && ch < nch) {
        nvfp4_chunk<MAXR>(cg[j], sg[j], xs, H, ch, rows, accg);
        nvfp4_chunk<MAXR>(cu[j], su[j], xs, H, ch, rows, accu);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < MAXR; ++r) {
    if (r < rows) {
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        accg[r] += __shfl_xor_sync(0xffffffffu, accg[r], off);
        accu[r] += __shfl_xor_sync(0xffffffffu, accu[r], off);
      }
    }
  }
  if (f < I) {
    const float cg2 = __fmul_rn(sx, gts[e]), cu2 = __fmul_rn(sx, uts[e]);
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
      if (r < rows && lane == r) {   // lane r stores row r
        const float g = accg[r] * cg2, u = accu[r] * cu2;
        const float inner = 0.7978845608028654f * fmaf(0.044715f * g, g * g, g);
        h32[(size_t)(row0 + r) * I + f] = 0.5f * g * (1.0f + tanhf(inner)) * u;
      }
    }
  }
}

// ---------------------------------------------------------------- GEMM-2
// Grid: (tile, 64 output columns).  Each warp issues the code loads of its 8 columns (rows of
// W_down's codes, [N = H][K = I/2] bytes), then the CTA quantises the tile's h rows (groups
// of 16 consecutive features, tensor scale sh) into shared memory, then every warp computes
// its columns for every row; o = acc * sh * ts_d[e], stored as bf16 rows of O (64-byte runs).
template <int MAXR>
__global__ void __launch_bounds__(256) nvfp4_gemm2_kernel(
    const float* __restrict__ h32, const int32_t* __restrict__ tile_num,
    const int32_t* __restrict__ tile_expert, const int32_t* __restrict__ tile_row0,
    const int32_t* __restrict__ tile_rows, const uint8_t* __restrict__ dc,
    const uint8_t* __restrict__ ds, const float* __restrict__ dts, int H, int I, float sh,
    __nv_bfloat16* __restrict__ O) {
  pdl_trigger();
  pdl_wait();
  if (*reinterpret_cast<volatile unsigned*>(&g_error_word) & MOE_DEVERR_TIMEOUT) return;
  const int tile = blockIdx.x;
  if (tile >= *tile_num) return;
  constexpr int COLS = 8 * FP4_G2_PER_WARP;
  const int e = tile_expert[tile], row0 = tile_row0[tile];
  const int rows = min(tile_rows[tile], MAXR);
  const int n0 = blockIdx.y * COLS;
  extern __shared__ __align__(16) uint8_t fsm[];
  uint32_t* hs = reinterpret_cast<uint32_t*>(fsm);                        // [rows][I/2] f16x2
  __nv_bfloat16* ot = reinterpret_cast<__nv_bfloat16*>(fsm + (size_t)rows * I * 2);  // [rows][64]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int iw = I / 2, ng = I / 16, nch = I / 32;
  const float c = __fmul_rn(sh, dts[e]);
  for (int cb = 0; cb < nch; cb += 32) {
    const int ch = cb + lane;
    uint4 cd[FP4_G2_PER_WARP];
    uint32_t sd[FP4_G2_PER_WARP];
#pragma unroll
    for (int j = 0; j < FP4_G2_PER_WARP; ++j) {   // the warp's columns, all loads first
      const int n = n0 + warp * FP4_G2_PER_WARP + j;
      if (n < H && ch < nch) {
        cd[j] = __ldcs(reinterpret_cast<const uint4*>(dc + ((size_t)e * H + n) * iw) + ch);
        sd[j] = __ldcs(reinterpret_cast<const uint16_t*>(ds + ((size_t)e * H + n) * ng) + ch);
      }
    }
    if (cb == 0) {
      nvfp4_stage_rows(hs, rows, I, sh, [&](int r, int g, float (&v)[16]) {
        const float4* src = reinterpret_cast<const float4*>(h32 + (size_t)(row0 + r) * I + 16 * g);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 a = src[q];
          v[4 * q] = a.x;
          v[4 * q + 1] = a.y;
          v[4 * q + 2] = a.z;
          v[4 * q + 3] = a.w;
        }
      });
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < FP4_G2_PER_WARP; ++j) {
      const int n = n0 + warp * FP4_G2_PER_WARP + j;
      float acc[MAXR];
#pragma unroll
      for (int r = 0; r < MAXR; ++r) acc[r] = 0.f;
      if (n < H && ch < nch) nvfp4_chunk<MAXR>(cd[j], sd[j], hs, I, ch, rows, acc);
#pragma unroll
      for (int r = 0; r < MAXR; ++r) {
        if (r < rows) {
#pragma unroll
          for (int off = 16; off; off >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
        }
      }
      // column partials of this chunk block, added in block order
      if (lane == 0 && n < H) {
#pragma unroll
        for (int r = 0; r < MAXR; ++r)
          if (r < rows) {
            float* slot = reinterpret_cast<float*>(fsm + (size_t)rows * I * 2 + (size_t)MAXR * COLS * 2) +
                          r * COLS + (n - n0);
            *slot = cb == 0 ? acc[r] : *slot + acc[r];
          }
      }
    }
  }
  __syncthreads();
  const float* part = reinterpret_cast<const float*>(fsm + (size_t)rows * I * 2 + (size_t)MAXR * COLS * 2);
  for (int i = threadIdx.x; i < rows * COLS; i += blockDim.x) {
    const int r = i / COLS, cc = i - r * COLS;
    ot[r * COLS + cc] = __float2bfloat16_rn(part[r * COLS + cc] * c);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows * (COLS / 8); i += blockDim.x) {
    const int r = i / (COLS / 8), v = i - r * (COLS / 8);
    if (n0 + 8 * v < H)
      *reinterpret_cast<uint4*>(O + (size_t)(row0 + r) * H + n0 + 8 * v) =
          reinterpret_cast<const uint4*>(ot + r * COLS)[v];
  }
}

}  // namespace moe
