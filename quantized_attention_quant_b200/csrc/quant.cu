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

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {
namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (sizeof(T) == 2 && std::is_same<T, __nv_bfloat16>::value) {
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
// One thread owns 8 channels of one 128-token chunk and walks its tokens in
// order, keeping 8 FP64 sums of K (and 8 FP32 maxima of |V| when v != null).
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) stats_kernel(const T* __restrict__ k,
                                                         const T* __restrict__ v, int N,
                                                         int nchunks, int64_t total_chunks,
                                                         double* __restrict__ ksum,
                                                         float* __restrict__ vmax) {
  constexpr int TPC = D / 8;  // threads per chunk
  constexpr int CPB = kThreads / TPC;
  const int64_t chunk = (int64_t)blockIdx.x * CPB + threadIdx.x / TPC;
  if (chunk >= total_chunks) return;
  const int c0 = (threadIdx.x % TPC) * 8;
  const int64_t bh = chunk / nchunks;
  const int ci = (int)(chunk % nchunks);
  const int t0 = ci * 128;
  const int t1 = min(t0 + 128, N);
  double s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float mx[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const T* kp = k + ((bh * N + t0) * D + c0);
  const T* vp = v ? v + ((bh * N + t0) * D + c0) : nullptr;
  for (int t = t0; t < t1; ++t) {
    float f[8];
    load8(kp, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] += (double)f[i];
    kp += D;
    if (vp) {
      load8(vp, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], fabsf(f[i]));
      vp += D;
    }
  }
  double* ko = ksum + chunk * D + c0;
#pragma unroll
  for (int i = 0; i < 8; ++i) ko[i] = s[i];
  if (vp) {
    float* vo = vmax + chunk * D + c0;
#pragma unroll
    for (int i = 0; i < 8; ++i) vo[i] = mx[i];
  }
}

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

// ------------------------------------------------------------- INT8 Q / K
// One CTA per (128-token block, b*h, tensor): load, (smooth), block amax,
// s = amax/127, codes.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) quant_int8_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ k_mean, int N,
    int8_t* __restrict__ q_codes, float* __restrict__ q_scales, int8_t* __restrict__ k_codes,
    float* __restrict__ k_scales, int first_tensor) {
  constexpr int VPT = 128 * D / 8 / kThreads;  // 16-byte vectors per thread
  __shared__ float red[kThreads / 32];
  const int tensor = first_tensor + blockIdx.z;  // 0 = Q, 1 = K
  const int64_t bh = blockIdx.y;
  const int ntiles = N / 128;
  const int tile = blockIdx.x;
  const T* src = (tensor == 0 ? q : k) + (bh * N + (int64_t)tile * 128) * D;
  float x[VPT][8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    load8(src + vec * 8, x[i]);
    if (tensor == 1) {
      const int c0 = (vec % (D / 8)) * 8;
      const float* mu = k_mean + bh * D + c0;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[i][e] = __fsub_rn(x[i][e], __ldg(mu + e));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[i][e]));
  }
  amax = block_max(amax, red);
  const float s = __fdiv_rn(amax, 127.f);
  int8_t* dst = (tensor == 0 ? q_codes : k_codes) + (bh * N + (int64_t)tile * 128) * D;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    uint32_t w[2] = {0u, 0u};
    if (s != 0.f) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int c = __float2int_rn(__fdiv_rn(x[i][e], s));
        c = max(-127, min(127, c));
        w[e >> 2] |= (uint32_t)(c & 0xFF) << (8 * (e & 3));
      }
    }
    *reinterpret_cast<uint2*>(dst + vec * 8) = make_uint2(w[0], w[1]);
  }
  if (threadIdx.x == 0) (tensor == 0 ? q_scales : k_scales)[bh * ntiles + tile] = s;
}

// ---------------------------------------------------------------- FP8 V
// One CTA per (128-token block, b*h): codes = e4m3(V / s_V[c]), transposed
// through shared memory into V^T [d, N].
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) quant_v_fp8_kernel(const T* __restrict__ v,
                                                               const float* __restrict__ v_scales,
                                                               int N, uint8_t* __restrict__ vt) {
  constexpr int VPT = 128 * D / 8 / kThreads;
  __shared__ __align__(16) uint8_t tile_s[D][128 + 16];
  const int64_t bh = blockIdx.y;
  const int tile = blockIdx.x;
  const T* src = v + (bh * N + (int64_t)tile * 128) * D;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    const int t = vec / (D / 8);
    const int c0 = (vec % (D / 8)) * 8;
    float x[8];
    load8(src + vec * 8, x);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float s0 = __ldg(v_scales + bh * D + c0 + e);
      const float s1 = __ldg(v_scales + bh * D + c0 + e + 1);
      const float a = s0 != 0.f ? __fdiv_rn(x[e], s0) : 0.f;
      const float b = s1 != 0.f ? __fdiv_rn(x[e + 1], s1) : 0.f;
      const uint32_t p = cvt_e4m3x2(a, b);
      tile_s[c0 + e][t] = (uint8_t)(p & 0xFF);
      tile_s[c0 + e + 1][t] = (uint8_t)(p >> 8);
    }
  }
  __syncthreads();
  // D rows x 128 bytes = D*8 16-byte chunks
  for (int ch = threadIdx.x; ch < D * 8; ch += kThreads) {
    const int c = ch >> 3, part = ch & 7;
    const uint4 val = *reinterpret_cast<const uint4*>(&tile_s[c][part * 16]);
    *reinterpret_cast<uint4*>(vt + ((bh * D + c) * (int64_t)N + (int64_t)tile * 128 + part * 16)) =
        val;
  }
}

// -------------------------------------------------------------------- FP4
__device__ __forceinline__ float ue4m3_roundtrip(float r, uint32_t* code) {
  // r >= 0: encode as e4m3 (rne, satfinite), decode back exactly
  const uint32_t p = cvt_e4m3x2(r, 0.f) & 0xFF;
  *code = p;
  return e4m3_to_f32(p);
}

// Scale-factor byte offset in the tensor-core layout: 512-byte block per
// (b*h, tile, 64-wide chunk); row r, 16-group s inside the chunk.
__device__ __forceinline__ int64_t sf_offset(int64_t bh, int ntiles, int tile, int nchunk, int chunk,
                                             int r, int s) {
  return (((bh * ntiles + tile) * nchunk + chunk) * 512) + (r & 31) * 16 + (r >> 5) * 4 + s;
}

// Q or smoothed K, one CTA per (tile, b*h, tensor).  Thread handles whole
// 16-channel groups: 128 rows x D/16 groups per tile.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) quant_fp4_qk_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ k_mean, int N,
    uint8_t* __restrict__ q_codes, float* __restrict__ q_g, uint8_t* __restrict__ q_sf,
    uint8_t* __restrict__ k_codes, float* __restrict__ k_g, uint8_t* __restrict__ k_sf,
    int first_tensor) {
  constexpr int G = D / 16;                  // groups per row
  constexpr int GPT = 128 * G / kThreads;    // groups per thread
  __shared__ float red[kThreads / 32];
  const int tensor = first_tensor + blockIdx.z;
  const int64_t bh = blockIdx.y;
  const int ntiles = N / 128;
  const int tile = blockIdx.x;
  const T* src = (tensor == 0 ? q : k) + (bh * N + (int64_t)tile * 128) * D;
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
    if (tensor == 1) {
      const float* mu = k_mean + bh * D + gc * 16;
#pragma unroll
      for (int e = 0; e < 16; ++e) x[i][e] = __fsub_rn(x[i][e], __ldg(mu + e));
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[i][e]));
  }
  amax = block_max(amax, red);
  const float g = __fdiv_rn(amax, 2688.f);
  const float six_g = __fmul_rn(6.f, g);
  uint8_t* codes = (tensor == 0 ? q_codes : k_codes) + (bh * N + (int64_t)tile * 128) * (D / 2);
  uint8_t* sf = tensor == 0 ? q_sf : k_sf;
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
    float t[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) t[e] = den != 0.f ? __fdiv_rn(x[i][e], den) : 0.f;
    uint2 packed = make_uint2(den != 0.f ? cvt_e2m1x8(t) : 0u, den != 0.f ? cvt_e2m1x8(t + 8) : 0u);
    *reinterpret_cast<uint2*>(codes + r * (D / 2) + gc * 8) = packed;
    sf[sf_offset(bh, ntiles, tile, D / 64, gc >> 2, r, gc & 3)] = (uint8_t)scode;
  }
  if (threadIdx.x == 0) (tensor == 0 ? q_g : k_g)[bh * ntiles + tile] = g;
}

// V for FP4: one CTA per (tile, b*h).  The tile (128 tokens x D) is staged
// in shared memory as float; thread handles (channel, 16-token group) pairs.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) quant_fp4_v_kernel(const T* __restrict__ v, int N,
                                                               uint8_t* __restrict__ vt_codes,
                                                               float* __restrict__ v_g,
                                                               uint8_t* __restrict__ v_sf) {
  constexpr int VPT = 128 * D / 8 / kThreads;
  constexpr int PAIRS = D * 8;  // channels x 16-token groups
  __shared__ T xs[128][D + 2];  // the tile in its input type (exact)
  __shared__ float red[kThreads / 32];
  const int64_t bh = blockIdx.y;
  const int ntiles = N / 128;
  const int tile = blockIdx.x;
  const T* src = v + (bh * N + (int64_t)tile * 128) * D;
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
    float t[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) t[e] = den != 0.f ? __fdiv_rn(x[e], den) : 0.f;
    uint2 packed = make_uint2(den != 0.f ? cvt_e2m1x8(t) : 0u, den != 0.f ? cvt_e2m1x8(t + 8) : 0u);
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
  if (threadIdx.x == 0) v_g[bh * ntiles + tile] = g;
}

template <typename T, int D>
cudaError_t launch_qk(const QuantQKArgs& a, cudaStream_t st) {
  const int64_t BH = a.B * a.H;
  const int nchunks = (int)(a.N / 128);
  const int64_t total = BH * nchunks;
  constexpr int CPB = kThreads / (D / 8);
  stats_kernel<T, D><<<(unsigned)((total + CPB - 1) / CPB), kThreads, 0, st>>>(
      (const T*)a.k, nullptr, (int)a.N, nchunks, total, a.ws_ksum, nullptr);
  finalize_kernel<<<(unsigned)BH, 128, 0, st>>>(a.ws_ksum, nullptr, D, (int)a.N, nchunks, a.k_mean,
                                                nullptr);
  dim3 grid((unsigned)nchunks, (unsigned)BH, 2);
  if (a.mode == 0) {
    quant_int8_kernel<T, D><<<grid, kThreads, 0, st>>>(
        (const T*)a.q, (const T*)a.k, a.k_mean, (int)a.N, (int8_t*)a.q_codes, a.q_scales,
        (int8_t*)a.k_codes, a.k_scales, 0);
  } else {
    quant_fp4_qk_kernel<T, D><<<grid, kThreads, 0, st>>>(
        (const T*)a.q, (const T*)a.k, a.k_mean, (int)a.N, (uint8_t*)a.q_codes, a.q_scales,
        (uint8_t*)a.q_sf, (uint8_t*)a.k_codes, a.k_scales, (uint8_t*)a.k_sf, 0);
  }
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_v(const QuantVArgs& a, cudaStream_t st) {
  const int64_t BH = a.B * a.H;
  const int nchunks = (int)(a.N / 128);
  const int64_t total = BH * nchunks;
  constexpr int CPB = kThreads / (D / 8);
  dim3 grid((unsigned)nchunks, (unsigned)BH, 1);
  if (a.mode == 0) {
    // |V| maxima per chunk (the K sums are not needed: pass K = V and
    // discard them into the same workspace)
    stats_kernel<T, D><<<(unsigned)((total + CPB - 1) / CPB), kThreads, 0, st>>>(
        (const T*)a.v, (const T*)a.v, (int)a.N, nchunks, total, a.ws_ksum, a.ws_vmax);
    finalize_kernel<<<(unsigned)BH, 128, 0, st>>>(nullptr, a.ws_vmax, D, (int)a.N, nchunks,
                                                  nullptr, a.v_scales);
    quant_v_fp8_kernel<T, D><<<grid, kThreads, 0, st>>>((const T*)a.v, a.v_scales, (int)a.N,
                                                        (uint8_t*)a.v_codes);
  } else {
    quant_fp4_v_kernel<T, D><<<grid, kThreads, 0, st>>>((const T*)a.v, (int)a.N,
                                                        (uint8_t*)a.v_codes, a.v_scales,
                                                        (uint8_t*)a.v_sf);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_qk(const QuantQKArgs& a, cudaStream_t st) {
  if (a.dtype == 1) {
    return a.d == 128 ? launch_qk<__nv_bfloat16, 128>(a, st) : launch_qk<__nv_bfloat16, 64>(a, st);
  }
  return a.d == 128 ? launch_qk<__half, 128>(a, st) : launch_qk<__half, 64>(a, st);
}

cudaError_t launch_quant_v(const QuantVArgs& a, cudaStream_t st) {
  if (a.dtype == 1) {
    return a.d == 128 ? launch_v<__nv_bfloat16, 128>(a, st) : launch_v<__nv_bfloat16, 64>(a, st);
  }
  return a.d == 128 ? launch_v<__half, 128>(a, st) : launch_v<__half, 64>(a, st);
}

}  // namespace sage
