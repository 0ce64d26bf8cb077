// attn_i8f8_common.cuh -- device helpers shared by the INT8/FP8 attention
// kernels (one CTA per work item, and the persistent variant): constants,
// the register split, TMEM fills, the row max and the exp / P~
// quantization of a 32-key chunk.  Everything is in an anonymous namespace:
// each kernel file gets its own copy.
#pragma once

#include <climits>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "exp2_poly.cuh"
#include "sage_internal.h"
#include "sage_ptx.cuh"

// Of every 8 groups of 4 scores in the exp pass, how many take 2^t from the
// FMA-pipe polynomial (exp2_poly.cuh) instead of the SFU.
#ifndef SAGE_EXP_POLY_GROUPS
#define SAGE_EXP_POLY_GROUPS 0
#endif

namespace sage {
namespace {

constexpr int kThreadsAttn = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)
constexpr uint32_t kBiasBits = 0x4B400000u;       // bit pattern of 1.5 * 2^23
constexpr float kBias = 12582912.0f;
// Register split (launch: 512 threads x 128 = 65536):
//   producer/MMA 32, two exp warpgroups keep 128, stats/fold 216
//   -> 128 x (32 + 128 + 128 + 216) = 64512 <= 65536.
constexpr uint32_t kRegsProducer = 32;
constexpr uint32_t kRegsStats = 216;

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}


// Global load the compiler keeps where it is written (a plain load of a
// value needed only in the next loop iteration may be sunk to the end of
// the current one, exposing its latency at the top of the next).
__device__ __forceinline__ float ldg_early(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Four consecutive floats (16-byte aligned), kept where written as above.
__device__ __forceinline__ float4 ldg4_early(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

// An INT8 score A as read from TMEM (the INT32 accumulator) turned into the
// float 1.5 * 2^23 + A, exactly, by one integer add to its bit pattern
// (|A| <= 127^2 * 128 < 2^22, inside the binade of 1.5 * 2^23 where floats
// are the integers): no conversion instruction, whose pipe the
// exponentials use.  FP8 Q/K scores are plain FP32 already.
template <bool QF8>
__device__ __forceinline__ float score(uint32_t a) {
  return QF8 ? __uint_as_float(a) : __uint_as_float(a + kBiasBits);
}

// Max of 32 FP32 scores (keys col0 .. col0+31).  MASKED: keys past lim
// (the causal diagonal tile, lim = the row; the last tile of a ragged
// sequence, lim = its last key) read as -inf.
template <bool MASKED>
__device__ __forceinline__ float max32_f(const uint32_t* s, int col0, int lim) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float x = __uint_as_float(s[k]), y = __uint_as_float(s[k + 8]);
    float z = __uint_as_float(s[k + 16]), w = __uint_as_float(s[k + 24]);
    if (MASKED) {
      x = (col0 + k <= lim) ? x : -INFINITY;
      y = (col0 + k + 8 <= lim) ? y : -INFINITY;
      z = (col0 + k + 16 <= lim) ? z : -INFINITY;
      w = (col0 + k + 24 <= lim) ? w : -INFINITY;
    }
    a[k] = fmax3(fmaxf(x, y), z, w);
  }
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

// Max of 32 INT32 scores, as the exact float; masking as above (masked keys
// read as the smallest integer, below every INT8 score).
template <bool MASKED>
__device__ __forceinline__ float max32_i(const uint32_t* s, int col0, int lim) {
  int a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    int x = (int)s[k], y = (int)s[k + 8], z = (int)s[k + 16], w = (int)s[k + 24];
    if (MASKED) {
      x = (col0 + k <= lim) ? x : INT_MIN;
      y = (col0 + k + 8 <= lim) ? y : INT_MIN;
      z = (col0 + k + 16 <= lim) ? z : INT_MIN;
      w = (col0 + k + 24 <= lim) ? w : INT_MIN;
    }
    a[k] = max(max(x, y), max(z, w));
  }
  const int m = max(max(max(a[0], a[1]), max(a[2], a[3])), max(max(a[4], a[5]), max(a[6], a[7])));
  return score<false>((uint32_t)m) - kBias;
}

// The scaled maximum of 64 scores of a row, keys 64 hh .. 64 hh + 63, in
// two 32-key chunks that dequantize with their own factors c0, c1 (one K
// scale per 32 keys); a chunk wholly past the mask limit takes no part.
template <bool MASKED, bool QF8>
__device__ __forceinline__ float scaled_max64(const uint32_t* s, int hh, int lim, float c0,
                                              float c1, float acc) {
  const float m0 = QF8 ? max32_f<MASKED>(s, 64 * hh, lim) : max32_i<MASKED>(s, 64 * hh, lim);
  const float m1 = QF8 ? max32_f<MASKED>(s + 32, 64 * hh + 32, lim)
                       : max32_i<MASKED>(s + 32, 64 * hh + 32, lim);
  float v0 = m0 * c0, v1 = m1 * c1;
  if (MASKED) {
    v0 = 64 * hh > lim ? -INFINITY : v0;
    v1 = 64 * hh + 32 > lim ? -INFINITY : v1;
  }
  return fmax3(acc, v0, v1);
}

// Whether group g (0..7) of 4 scores takes the FMA-pipe polynomial: the
// groups are spread evenly over the 32 scores of a chunk.
__device__ __forceinline__ constexpr bool poly_group(int g) {
  return (g * SAGE_EXP_POLY_GROUPS) % 8 < SAGE_EXP_POLY_GROUPS;
}

// 448 P~ for 32 scores of a row -> 8 words of e4m3 codes (key i in byte
// i % 4 of word i / 4) and the sum of the unquantized values.  QF8: the
// scores are plain FP32 (no bias to remove).
template <bool MASKED, bool QF8>
__device__ __forceinline__ float exp_quant32(const uint32_t (&s)[32], float c, float neg, int col0,
                                             int lim, uint32_t (&p)[8]) {
  const float2 c2 = make_float2(c, c);
  const float2 n2 = make_float2(neg, neg);
  const float2 mb = make_float2(-kBias, -kBias);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    // (1.5*2^23 + A) - 1.5*2^23 = A exactly
    float2 x01 = make_float2(score<QF8>(s[i]), score<QF8>(s[i + 1]));
    float2 x23 = make_float2(score<QF8>(s[i + 2]), score<QF8>(s[i + 3]));
    if (!QF8) {
      x01 = __fadd2_rn(x01, mb);
      x23 = __fadd2_rn(x23, mb);
    }
    const float2 t01 = __ffma2_rn(x01, c2, n2);
    const float2 t23 = __ffma2_rn(x23, c2, n2);
    float f0, f1, f2, f3;
    if (poly_group(i >> 2)) {
      const float2 e01 = exp2_poly2(t01), e23 = exp2_poly2(t23);
      f0 = e01.x, f1 = e01.y, f2 = e23.x, f3 = e23.y;
    } else {
      f0 = ex2(t01.x), f1 = ex2(t01.y), f2 = ex2(t23.x), f3 = ex2(t23.y);
    }
    if (MASKED) {
      f0 = (col0 + i + 0 <= lim) ? f0 : 0.f;
      f1 = (col0 + i + 1 <= lim) ? f1 : 0.f;
      f2 = (col0 + i + 2 <= lim) ? f2 : 0.f;
      f3 = (col0 + i + 3 <= lim) ? f3 : 0.f;
    }
    acc0 = __fadd2_rn(acc0, make_float2(f0, f1));
    acc1 = __fadd2_rn(acc1, make_float2(f2, f3));
    p[i >> 2] = cvt_e4m3x2(f0, f1) | (cvt_e4m3x2(f2, f3) << 16);
  }
  const float2 t = __fadd2_rn(acc0, acc1);
  return t.x + t.y;
}

template <typename OutT>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One 32-key chunk cc (0..3) of the exp pass: its e4m3 codes go to the 8
// TMEM columns pcol (four keys per column, the A-operand layout of the
// P~V MMA); returns the chunk's row sum.
template <bool MASKED, bool QF8>
__device__ __forceinline__ float exp_chunk(const uint32_t (&s)[32], int cc, float c, float neg,
                                           int lim, uint32_t pcol) {
  uint32_t p[8];
  const float sum = exp_quant32<MASKED, QF8>(s, c, neg, 32 * cc, lim, p);
  tmem_st8(pcol, p);
  return sum;
}

}  // namespace
}  // namespace sage
