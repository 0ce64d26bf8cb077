// quant.cu -- the quantization pre-pass: K channel statistics, INT8 / FP8
// and FP4 encodings of Q, K and V.
//
// Every step that decides a code is taken in the precision the oracle
// states: FP64 sums for the K mean (per 128-token chunk in token order,
// then chunks in order), IEEE FP32 subtraction and division, round to
// nearest even with saturation in every cast.  The codes and scales are
// therefore bit-identical to the CPU restatement.
//
// Method: SageAttention abstract (K smoothing, INT8 Q/K), SageAttention2
// abstract (FP8 V), SageAttention3 abstract (FP4 with one FP8 scale per 16
// elements), all on the dblp author page on taxoreview.com.
//
// Launch structure (one 256-thread CTA per 128-token tile and role):
//   kernel A  roles that need no head-wide statistic: Q codes, FP4 V codes,
//             and the per-chunk K sums / V maxima;
//   finalize  per (b, h): fold the chunk partials in chunk order into the
//             K mean and the per-channel V scale;
//   kernel B  roles that need them: smoothed K codes, FP8 V codes.
// sage_attn_fwd runs all roles of Q, K and V in these three launches.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {
namespace {

constexpr int kThreads = 256;

enum Role : int {
  kQuantQ8 = 0,   // INT8 Q codes + block scales
  kQuantK8 = 1,   // INT8 smoothed-K codes + block scales (needs the K mean)
  kQuantV8 = 2,   // FP8 V^T codes (needs the V scales)
  kQuantQ4 = 3,   // FP4 Q codes, block-16 scales, tile scale
  kQuantK4 = 4,   // FP4 smoothed-K codes (needs the K mean)
  kQuantV4 = 5,   // FP4 V^T codes (tile-local scales)
  kStatsK = 6,    // K chunk sums
  kStatsKV = 7,   // K chunk sums and V chunk maxima
  kStatsV = 8,    // V chunk maxima
};

struct Roles {
  int n;
  int r[4];
};

// Pointers of every role (unused ones may be null).
struct PrepassPtrs {
  const void* q;
  const void* k;
  const void* v;
  int N;
  void* q_codes;
  float* q_scales;
  uint8_t* q_sf;
  void* k_codes;
  float* k_scales;
  uint8_t* k_sf;
  float* k_mean;
  void* v_codes;
  float* v_scales;
  uint8_t* v_sf;
  double* ksum;  // [B*H, N/128, d] FP64 chunk sums of K
  float* vmax;   // [B*H, N/128, d] chunk maxima of |V|
};

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 t = __half22float2(h);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
}

template <typename T>
__device__ __forceinline__ float load1(const T* p) {
  return static_cast<float>(*p);
}

// Division-free quotient for code decisions.  With rs = fp32(1/s) (correctly
// rounded), q = fp32(x * rs) lies within 3 * 2^-24 |x/s| of fp32(x / s), so
// the interval [q (1 - 2^-20), q (1 + 2^-20)] (each end rounded to fp32)
// contains fp32(x / s).  Rounding to a code is monotonic, so when both ends
// give the same code, fp32(x / s) gives it too and q may stand in for the
// quotient; otherwise (q within ~2^-20 of a rounding boundary, or rs not
// finite) the IEEE division is taken.  The result is bit-identical to
// deciding on fp32(x / s).
constexpr float kBracketLo = 1.0f - 0x1p-20f;
constexpr float kBracketHi = 1.0f + 0x1p-20f;

// INT8 code clamp(rne(fp32(x / s)), +-127), s != 0.  Rounding to an integer
// is an FP32 add of 1.5 * 2^23 (exact round-half-even for |v| < 2^22; here
// |x / s| < 128), read back from the bits, so no conversion instruction is
// needed; the bracket test compares the two rounded ends bit for bit.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;

__device__ __forceinline__ int int8_code(float x, float s, float rs) {
  const float q = x * rs;
  const float2 ends = __fadd2_rn(__fmul2_rn(make_float2(q, q), make_float2(kBracketLo, kBracketHi)),
                                 make_float2(kRoundMagic, kRoundMagic));
  const float rounded = (rs != 0.f && __float_as_uint(ends.x) == __float_as_uint(ends.y))
                            ? ends.y
                            : __fdiv_rn(x, s) + kRoundMagic;
  const int c = __float_as_int(rounded) - kRoundMagicBits;
  return max(-127, min(127, c));
}

__device__ __forceinline__ float quot_e4m3(float x, float s, float rs) {
  const float q = x * rs;
  const uint32_t pk = cvt_e4m3x2(q * kBracketLo, q * kBracketHi);
  if (rs != 0.f && (pk & 0xFFu) == (pk >> 8)) return q;
  return __fdiv_rn(x, s);
}

__device__ __forceinline__ float quot_e2m1(float x, float s, float rs) {
  const float q = x * rs;
  uint32_t two;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
      "cvt.u32.u8 %0, b;\n\t}"
      : "=r"(two)
      : "f"(q * kBracketHi), "f"(q * kBracketLo));
  if (rs != 0.f && (two & 0xFu) == (two >> 4)) return q;
  return __fdiv_rn(x, s);
}

// 1/s for the fast path, or 0 when it must not be used (s == 0 or 1/s
// overflows); quot_* are then only called with the exact fallback.
__device__ __forceinline__ float recip_or_zero(float s) {
  if (s == 0.f) return 0.f;
  const float r = __frcp_rn(s);
  return isfinite(r) ? r : 0.f;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

// ------------------------------------------------------------------ stats
// One CTA per (128-token chunk, b*h).  Thread c < D walks K's channel c over
// the chunk's tokens in order with an FP64 sum; thread D + c keeps the max
// of |V| of channel c.  Consecutive threads read consecutive channels.
template <typename T, int D>
__device__ __forceinline__ void role_stats(const PrepassPtrs& p, int64_t bh, int chunk,
                                           bool do_k, bool do_v) {
  const int nchunks = p.N / 128;
  const int t = threadIdx.x;
  const int64_t row0 = bh * p.N + (int64_t)chunk * 128;
  const int64_t out = (bh * nchunks + chunk) * D;
  if (t < D) {
    if (!do_k) return;
    const T* src = reinterpret_cast<const T*>(p.k) + row0 * D + t;
    double s = 0.0;
#pragma unroll 16
    for (int i = 0; i < 128; ++i) s += (double)load1(src + (int64_t)i * D);
    p.ksum[out + t] = s;
  } else if (t < 2 * D) {
    if (!do_v) return;
    const int c = t - D;
    const T* src = reinterpret_cast<const T*>(p.v) + row0 * D + c;
    float m = 0.f;
#pragma unroll 16
    for (int i = 0; i < 128; ++i) m = fmaxf(m, fabsf(load1(src + (int64_t)i * D)));
    p.vmax[out + c] = m;
  }
}

// ------------------------------------------------------------- INT8 Q / K
// Load, (smooth), block amax, s = amax / 127, codes = clamp(rne(x / s)).
// Two passes over the 128-token tile: the amax pass keeps nothing, the code
// pass reads the tile again (from L1/L2), so the role needs few registers and
// many CTAs fit on an SM.  A thread's vectors all cover the same 8 channels.
template <typename T, int D>
__device__ __forceinline__ void role_quant_int8(const T* __restrict__ src, const float* mean,
                                                int8_t* __restrict__ dst, float* scale_out,
                                                float* red) {
  constexpr int VPT = 128 * D / 8 / kThreads;  // 16-byte vectors per thread
  const int c0 = (threadIdx.x % (D / 8)) * 8;
  float mu[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (mean) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(mean + c0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(mean + c0 + 4));
    mu[0] = a.x; mu[1] = a.y; mu[2] = a.z; mu[3] = a.w;
    mu[4] = b.x; mu[5] = b.y; mu[6] = b.z; mu[7] = b.w;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    float x[8];
    load8(src + (threadIdx.x + i * kThreads) * 8, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float v = mean ? __fsub_rn(x[e], mu[e]) : x[e];
      amax = fmaxf(amax, fabsf(v));
    }
  }
  amax = block_max(amax, red);
  const float s = __fdiv_rn(amax, 127.f);
  const float rs = recip_or_zero(s);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    uint32_t w[2] = {0u, 0u};
    if (s != 0.f) {
      float x[8];
      load8(src + vec * 8, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = mean ? __fsub_rn(x[e], mu[e]) : x[e];
        const int c = int8_code(v, s, rs);
        w[e >> 2] |= (uint32_t)(c & 0xFF) << (8 * (e & 3));
      }
    }
    *reinterpret_cast<uint2*>(dst + vec * 8) = make_uint2(w[0], w[1]);
  }
  if (threadIdx.x == 0) *scale_out = s;
}

// ---------------------------------------------------------------- FP8 V
// codes = e4m3(V / s_V[c]) written transposed into V^T.  A thread owns a
// channel pair and 32 consecutive tokens: it reads the pair at each token
// (consecutive threads -> consecutive pairs, so a warp reads 128 contiguous
// bytes per token) and writes each channel's 32 codes as a whole 32-byte
// sector (two 16-byte stores).
template <typename T, int D>
__device__ __forceinline__ void role_quant_v_fp8(const T* __restrict__ src,
                                                 const float* __restrict__ vs,
                                                 uint8_t* __restrict__ dst, int N) {
  constexpr int UNITS = (D / 2) * 8;  // channel pairs x 16-token groups
  for (int u = threadIdx.x; u < UNITS; u += kThreads) {
    const int cp = u % (D / 2), grp = u / (D / 2);
    const float s0 = __ldg(vs + 2 * cp), s1 = __ldg(vs + 2 * cp + 1);
    const float r0 = recip_or_zero(s0), r1 = recip_or_zero(s1);
    const uint32_t* p = reinterpret_cast<const uint32_t*>(src + (int64_t)(grp * 16) * D + 2 * cp);
    uint32_t w0[4] = {0u, 0u, 0u, 0u}, w1[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const uint32_t pair = __ldg(p + t * (D / 2));
      float x0, x1;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        x0 = __uint_as_float(pair << 16);
        x1 = __uint_as_float(pair & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&pair));
        x0 = f.x;
        x1 = f.y;
      }
      const float a = s0 != 0.f ? quot_e4m3(x0, s0, r0) : 0.f;
      const float b = s1 != 0.f ? quot_e4m3(x1, s1, r1) : 0.f;
      const uint32_t pk = cvt_e4m3x2(a, b);  // a in bits 0..7, b in 8..15
      w0[t >> 2] |= (pk & 0xFFu) << (8 * (t & 3));
      w1[t >> 2] |= (pk >> 8) << (8 * (t & 3));
    }
    // dst points at V^T[c = 0][tile start]
    *reinterpret_cast<uint4*>(dst + (int64_t)(2 * cp) * N + grp * 16) =
        make_uint4(w0[0], w0[1], w0[2], w0[3]);
    *reinterpret_cast<uint4*>(dst + (int64_t)(2 * cp + 1) * N + grp * 16) =
        make_uint4(w1[0], w1[1], w1[2], w1[3]);
  }
}

// -------------------------------------------------------------------- FP4
__device__ __forceinline__ float ue4m3_roundtrip(float r, uint32_t* code) {
  // r >= 0: encode as e4m3 (rne, satfinite), decode back exactly
  const uint32_t pk = cvt_e4m3x2(r, 0.f) & 0xFF;
  *code = pk;
  return e4m3_to_f32(pk);
}

// Scale-factor byte offset in the tensor-core layout: 512-byte block per
// (b*h, tile, 64-wide chunk); row r, 16-group s inside the chunk.
__device__ __forceinline__ int64_t sf_offset(int64_t bh, int ntiles, int tile, int nchunk, int chunk,
                                             int r, int s) {
  return (((bh * ntiles + tile) * nchunk + chunk) * 512) + (r & 31) * 16 + (r >> 5) * 4 + s;
}

// Q or smoothed K of one tile: g = amax/2688, per 16 channels
// s16 = ue4m3(amax16 / (6 g)), code = e2m1(x / (s16 g)).
template <typename T, int D>
__device__ __forceinline__ void role_quant_fp4_tokens(const T* __restrict__ src, const float* mean,
                                                      uint8_t* __restrict__ codes, float* g_out,
                                                      uint8_t* __restrict__ sf, int64_t bh,
                                                      int ntiles, int tile, float* red) {
  constexpr int G = D / 16;                // groups per row
  constexpr int GPT = 128 * G / kThreads;  // groups per thread
  float x[GPT][16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < GPT; ++i) {
    const int grp = threadIdx.x + i * kThreads;
    const int r = grp / G, gc = grp % G;
    float a[8], b[8];
    load8(src + r * D + gc * 16, a);
    load8(src + r * D + gc * 16 + 8, b);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[i][e] = a[e];
      x[i][8 + e] = b[e];
    }
    if (mean) {
      const float* mu = mean + gc * 16;
#pragma unroll
      for (int e = 0; e < 16; ++e) x[i][e] = __fsub_rn(x[i][e], __ldg(mu + e));
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[i][e]));
  }
  amax = block_max(amax, red);
  const float g = __fdiv_rn(amax, 2688.f);
  const float six_g = __fmul_rn(6.f, g);
#pragma unroll
  for (int i = 0; i < GPT; ++i) {
    const int grp = threadIdx.x + i * kThreads;
    const int r = grp / G, gc = grp % G;
    float a16 = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) a16 = fmaxf(a16, fabsf(x[i][e]));
    uint32_t scode = 0;
    float den = 0.f;
    if (six_g != 0.f) {
      const float sdec = ue4m3_roundtrip(__fdiv_rn(a16, six_g), &scode);
      den = __fmul_rn(sdec, g);
    }
    const float rden = recip_or_zero(den);
    float t[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) t[e] = den != 0.f ? quot_e2m1(x[i][e], den, rden) : 0.f;
    const uint2 packed =
        make_uint2(den != 0.f ? cvt_e2m1x8(t) : 0u, den != 0.f ? cvt_e2m1x8(t + 8) : 0u);
    *reinterpret_cast<uint2*>(codes + r * (D / 2) + gc * 8) = packed;
    sf[sf_offset(bh, ntiles, tile, D / 64, gc >> 2, r, gc & 3)] = (uint8_t)scode;
  }
  if (threadIdx.x == 0) *g_out = g;
}

// V of one tile for FP4: staged in shared memory in its input type; each
// thread handles (channel, 16-token group) pairs.
template <typename T, int D>
__device__ __forceinline__ void role_quant_fp4_v(const T* __restrict__ src, int N,
                                                 uint8_t* __restrict__ vt_codes, float* g_out,
                                                 uint8_t* __restrict__ v_sf, int64_t bh,
                                                 int ntiles, int tile, T (*xs)[D + 2],
                                                 float* red) {
  constexpr int VPT = 128 * D / 8 / kThreads;
  constexpr int PAIRS = D * 8;  // channels x 16-token groups
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    const int t = vec / (D / 8), c0 = (vec % (D / 8)) * 8;
    float x[8];
    load8(src + vec * 8, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      xs[t][c0 + e] = src[vec * 8 + e];
      amax = fmaxf(amax, fabsf(x[e]));
    }
  }
  amax = block_max(amax, red);  // contains __syncthreads
  const float g = __fdiv_rn(amax, 2688.f);
  const float six_g = __fmul_rn(6.f, g);
  for (int pr = threadIdx.x; pr < PAIRS; pr += kThreads) {
    const int c = pr % D, grp = pr / D;  // consecutive threads -> consecutive channels
    float x[16];
    float a16 = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      x[e] = static_cast<float>(xs[grp * 16 + e][c]);
      a16 = fmaxf(a16, fabsf(x[e]));
    }
    uint32_t scode = 0;
    float den = 0.f;
    if (six_g != 0.f) {
      const float sdec = ue4m3_roundtrip(__fdiv_rn(a16, six_g), &scode);
      den = __fmul_rn(sdec, g);
    }
    const float rden = recip_or_zero(den);
    float t[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) t[e] = den != 0.f ? quot_e2m1(x[e], den, rden) : 0.f;
    const uint2 packed =
        make_uint2(den != 0.f ? cvt_e2m1x8(t) : 0u, den != 0.f ? cvt_e2m1x8(t + 8) : 0u);
    *reinterpret_cast<uint2*>(vt_codes + (bh * D + c) * (int64_t)(N / 2) + tile * 64 + grp * 8) =
        packed;
    v_sf[sf_offset(bh, ntiles, tile, 2, grp >> 2, c, grp & 3)] = (uint8_t)scode;
  }
  // rows D..127 of the scale blocks stay zero (tensor-core rows beyond d)
  if (D < 128) {
    for (int idx = threadIdx.x; idx < (128 - D) * 8; idx += kThreads) {
      const int r = D + idx / 8, grp = idx % 8;
      v_sf[sf_offset(bh, ntiles, tile, 2, grp >> 2, r, grp & 3)] = 0;
    }
  }
  if (threadIdx.x == 0) *g_out = g;
}

// ------------------------------------------------------------- the kernels
// grid (tile, b*h, role index); roles.r[blockIdx.z] selects the work.  MASK
// (a bit per Role) lists the roles a launch may run: only their code is
// compiled in, so each launch gets the register and shared-memory footprint
// of its own roles (and the occupancy that goes with it).
#define SAGE_ROLE(r) if constexpr (((MASK >> (r)) & 1) != 0)
template <typename T, int D, int MASK>
__global__ void __launch_bounds__(kThreads) prepass_kernel(PrepassPtrs p, Roles roles) {
  constexpr int V4_BYTES = ((MASK >> kQuantV4) & 1) ? 128 * (D + 2) * (int)sizeof(T) : 16;
  __shared__ __align__(16) uint8_t smem_raw[V4_BYTES];
  __shared__ float red[kThreads / 32];
  const int role = roles.r[blockIdx.z];
  const int64_t bh = blockIdx.y;
  const int tile = blockIdx.x;
  const int ntiles = p.N / 128;
  const int64_t row0 = bh * p.N + (int64_t)tile * 128;
  switch (role) {
    case kQuantQ8:
      SAGE_ROLE(kQuantQ8)
      role_quant_int8<T, D>(reinterpret_cast<const T*>(p.q) + row0 * D, nullptr,
                            reinterpret_cast<int8_t*>(p.q_codes) + row0 * D,
                            p.q_scales + bh * ntiles + tile, red);
      break;
    case kQuantK8:
      SAGE_ROLE(kQuantK8)
      role_quant_int8<T, D>(reinterpret_cast<const T*>(p.k) + row0 * D, p.k_mean + bh * D,
                            reinterpret_cast<int8_t*>(p.k_codes) + row0 * D,
                            p.k_scales + bh * ntiles + tile, red);
      break;
    case kQuantV8:
      SAGE_ROLE(kQuantV8)
      role_quant_v_fp8<T, D>(reinterpret_cast<const T*>(p.v) + row0 * D, p.v_scales + bh * D,
                             reinterpret_cast<uint8_t*>(p.v_codes) + bh * D * (int64_t)p.N +
                                 (int64_t)tile * 128,
                             p.N);
      break;
    case kQuantQ4:
      SAGE_ROLE(kQuantQ4)
      role_quant_fp4_tokens<T, D>(reinterpret_cast<const T*>(p.q) + row0 * D, nullptr,
                                  reinterpret_cast<uint8_t*>(p.q_codes) + row0 * (D / 2),
                                  p.q_scales + bh * ntiles + tile, p.q_sf, bh, ntiles, tile, red);
      break;
    case kQuantK4:
      SAGE_ROLE(kQuantK4)
      role_quant_fp4_tokens<T, D>(reinterpret_cast<const T*>(p.k) + row0 * D, p.k_mean + bh * D,
                                  reinterpret_cast<uint8_t*>(p.k_codes) + row0 * (D / 2),
                                  p.k_scales + bh * ntiles + tile, p.k_sf, bh, ntiles, tile, red);
      break;
    case kQuantV4:
      SAGE_ROLE(kQuantV4)
      role_quant_fp4_v<T, D>(reinterpret_cast<const T*>(p.v) + row0 * D, p.N,
                             reinterpret_cast<uint8_t*>(p.v_codes), p.v_scales + bh * ntiles + tile,
                             p.v_sf, bh, ntiles, tile, reinterpret_cast<T(*)[D + 2]>(smem_raw), red);
      break;
    case kStatsK:
      SAGE_ROLE(kStatsK) role_stats<T, D>(p, bh, tile, true, false);
      break;
    case kStatsKV:
      SAGE_ROLE(kStatsKV) role_stats<T, D>(p, bh, tile, true, true);
      break;
    case kStatsV:
      SAGE_ROLE(kStatsV) role_stats<T, D>(p, bh, tile, false, true);
      break;
    default:
      break;
  }
}
#undef SAGE_ROLE

constexpr int bit(int r) { return 1 << r; }

// Fold the chunk partials in chunk order: mean = fp32(sum / N); and, for
// FP8 V, s_V = fp32(amax / 448).
__global__ void finalize_kernel(const double* __restrict__ ksum, const float* __restrict__ vmax,
                                int D, int N, int nchunks, float* __restrict__ k_mean,
                                float* __restrict__ v_scales) {
  const int64_t bh = blockIdx.x;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    if (ksum) {
      double s = 0.0;
      for (int i = 0; i < nchunks; ++i) s += ksum[(bh * nchunks + i) * D + c];
      k_mean[bh * D + c] = __double2float_rn(__ddiv_rn(s, (double)N));
    }
    if (vmax) {
      float m = 0.f;
      for (int i = 0; i < nchunks; ++i) m = fmaxf(m, vmax[(bh * nchunks + i) * D + c]);
      v_scales[bh * D + c] = __fdiv_rn(m, 448.f);
    }
  }
}

// kernel A (roles a), finalize (K mean and/or V scales), kernel B (roles b)
template <typename T, int D, int MA, int MB>
cudaError_t run_plan(const PrepassPtrs& p, int64_t BH, Roles a, bool fin_k, bool fin_v, Roles b,
                     cudaStream_t st) {
  const int ntiles = p.N / 128;
  if (a.n) prepass_kernel<T, D, MA><<<dim3(ntiles, (unsigned)BH, a.n), kThreads, 0, st>>>(p, a);
  if (fin_k || fin_v)
    finalize_kernel<<<(unsigned)BH, 128, 0, st>>>(fin_k ? p.ksum : nullptr, fin_v ? p.vmax : nullptr,
                                                  D, p.N, ntiles, p.k_mean, p.v_scales);
  if (b.n) prepass_kernel<T, D, MB><<<dim3(ntiles, (unsigned)BH, b.n), kThreads, 0, st>>>(p, b);
  return cudaGetLastError();
}

// MA / MB: the role masks of kernels A and B (they must cover a.r / b.r).
template <int MA, int MB>
cudaError_t dispatch(const PrepassPtrs& p, int dtype, int64_t d, int64_t BH, Roles a, bool fin_k,
                     bool fin_v, Roles b, cudaStream_t st) {
  if (dtype == 1)
    return d == 128 ? run_plan<__nv_bfloat16, 128, MA, MB>(p, BH, a, fin_k, fin_v, b, st)
                    : run_plan<__nv_bfloat16, 64, MA, MB>(p, BH, a, fin_k, fin_v, b, st);
  return d == 128 ? run_plan<__half, 128, MA, MB>(p, BH, a, fin_k, fin_v, b, st)
                  : run_plan<__half, 64, MA, MB>(p, BH, a, fin_k, fin_v, b, st);
}

PrepassPtrs ptrs_qk(const QuantQKArgs& a) {
  PrepassPtrs p{};
  p.q = a.q;
  p.k = a.k;
  p.N = (int)a.N;
  p.q_codes = a.q_codes;
  p.q_scales = a.q_scales;
  p.q_sf = static_cast<uint8_t*>(a.q_sf);
  p.k_codes = a.k_codes;
  p.k_scales = a.k_scales;
  p.k_sf = static_cast<uint8_t*>(a.k_sf);
  p.k_mean = a.k_mean;
  p.ksum = a.ws_ksum;
  return p;
}

void add_v(PrepassPtrs& p, const QuantVArgs& a) {
  p.v = a.v;
  p.N = (int)a.N;
  p.v_codes = a.v_codes;
  p.v_scales = a.v_scales;
  p.v_sf = static_cast<uint8_t*>(a.v_sf);
  p.vmax = a.ws_vmax;
}

}  // namespace

cudaError_t launch_quant_qk(const QuantQKArgs& a, cudaStream_t st) {
  const PrepassPtrs p = ptrs_qk(a);
  if (a.mode == 0)
    return dispatch<bit(kQuantQ8) | bit(kStatsK), bit(kQuantK8)>(
        p, a.dtype, a.d, a.B * a.H, Roles{2, {kQuantQ8, kStatsK}}, true, false,
        Roles{1, {kQuantK8}}, st);
  return dispatch<bit(kQuantQ4) | bit(kStatsK), bit(kQuantK4)>(
      p, a.dtype, a.d, a.B * a.H, Roles{2, {kQuantQ4, kStatsK}}, true, false,
      Roles{1, {kQuantK4}}, st);
}

cudaError_t launch_quant_v(const QuantVArgs& a, cudaStream_t st) {
  PrepassPtrs p{};
  add_v(p, a);
  if (a.mode == 0)
    return dispatch<bit(kStatsV), bit(kQuantV8)>(p, a.dtype, a.d, a.B * a.H, Roles{1, {kStatsV}},
                                                 false, true, Roles{1, {kQuantV8}}, st);
  return dispatch<bit(kQuantV4), 0>(p, a.dtype, a.d, a.B * a.H, Roles{1, {kQuantV4}}, false,
                                    false, Roles{0, {}}, st);
}

cudaError_t launch_prepass(const QuantQKArgs& qa, const QuantVArgs& va, cudaStream_t st) {
  PrepassPtrs p = ptrs_qk(qa);
  add_v(p, va);
  if (qa.mode == 0)
    return dispatch<bit(kQuantQ8) | bit(kStatsKV), bit(kQuantK8) | bit(kQuantV8)>(
        p, qa.dtype, qa.d, qa.B * qa.H, Roles{2, {kQuantQ8, kStatsKV}}, true, true,
        Roles{2, {kQuantK8, kQuantV8}}, st);
  return dispatch<bit(kQuantQ4) | bit(kQuantV4) | bit(kStatsK), bit(kQuantK4)>(
      p, qa.dtype, qa.d, qa.B * qa.H, Roles{3, {kQuantQ4, kQuantV4, kStatsK}}, true, false,
      Roles{1, {kQuantK4}}, st);
}

}  // namespace sage
