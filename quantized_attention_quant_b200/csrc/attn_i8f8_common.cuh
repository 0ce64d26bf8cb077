// attn_i8f8_common.cuh -- device helpers shared by the INT8/FP8 attention
// kernels (one CTA per work item, and the persistent variant): constants,
// the register split, TMEM fills, the row max and the exp / P~
// quantization of a 32-key chunk.  Everything is in an anonymous namespace:
// each kernel file gets its own copy.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

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


// 32 columns of the same 32-bit value.
__device__ __forceinline__ void tmem_fill32(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
      "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

// Global load the compiler keeps where it is written (a plain load of a
// value needed only in the next loop iteration may be sunk to the end of
// the current one, exposing its latency at the top of the next).
__device__ __forceinline__ float ldg_early(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// A score as read from TMEM: the float 1.5 * 2^23 + A (exact).
__device__ __forceinline__ float biased(uint32_t a) { return __uint_as_float(a); }

// Max of 64 scores and a running value.  MASKED: columns col0 + i > lim are
// ignored (the causal diagonal tile, lim = the row; the last tile of a
// ragged sequence, lim = its last key): they read as 0, below every biased
// INT8 score, or -inf for the plain FP32 scores of the FP8 Q K^T.
template <bool MASKED, bool QF8>
__device__ __forceinline__ float max64(const uint32_t* s, int col0, int lim, float acc) {
  constexpr float kLow = QF8 ? -INFINITY : 0.f;
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float x = biased(s[k]), y = biased(s[k + 8]);
    if (MASKED) {
      x = (col0 + k <= lim) ? x : kLow;
      y = (col0 + k + 8 <= lim) ? y : kLow;
    }
    a[k] = fmaxf(x, y);
  }
#pragma unroll
  for (int i = 16; i < 64; i += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float x = biased(s[i + k]), y = biased(s[i + 8 + k]);
      if (MASKED) {
        x = (col0 + i + k <= lim) ? x : kLow;
        y = (col0 + i + 8 + k <= lim) ? y : kLow;
      }
      a[k] = fmax3(a[k], x, y);
    }
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmax3(a[6], a[7], acc));
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
    float2 x01 = make_float2(biased(s[i]), biased(s[i + 1]));
    float2 x23 = make_float2(biased(s[i + 2]), biased(s[i + 3]));
    if (!QF8) {
      x01 = __fadd2_rn(x01, mb);
      x23 = __fadd2_rn(x23, mb);
    }
    const float2 t01 = __ffma2_rn(x01, c2, n2);
    const float2 t23 = __ffma2_rn(x23, c2, n2);
    float f0 = ex2(t01.x), f1 = ex2(t01.y), f2 = ex2(t23.x), f3 = ex2(t23.y);
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
