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
// Launch structure of the chains (one 256-thread CTA per 128-token tile and
// role):
//   kernel A  roles that need no head-wide statistic: Q codes, FP4 V codes,
//             and the per-chunk K sums / V maxima.  The last statistics CTA
//             of each (b, h) (a per-head counter tells it) folds the chunk
//             partials in chunk order into the K mean and the per-channel V
//             scale, then resets the counter;
//   kernel B  roles that need them: smoothed K codes, FP8 V codes.
// The Q/K pre-pass is one A -> B chain, the V pre-pass another (in FP4 mode
// a single launch); sage_quant_qkv and sage_attn_fwd run the two chains on
// two streams, or, for short heads in the 8-bit modes, the one launch of the
// cluster-fused kernel at the end of this file.

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
  kQuantQF8 = 9,  // FP8 (e4m3) Q codes + block scales
  kQuantKF8 = 10, // FP8 (e4m3) smoothed-K codes + block scales (needs the K mean)
  kQuantQ8S = 11,  // INT8 codes of the smoothed Q (tile mean out) + scales + the mean
  kQuantQF8S = 12, // FP8 codes of the smoothed Q + scales + the mean
  kQuantQ4S = 13,  // FP4 codes of the smoothed Q + scales + the mean
};

struct Roles {
  int n;
  int r[4];
  // walk the grid backwards: the second launch of a chain then re-reads
  // first the tiles its first launch read last (the ones most likely still
  // in L2)
  int reverse = 0;
};

// Pointers of every role (unused ones may be null).
struct PrepassPtrs {
  const void* q;
  const void* k;
  const void* v;
  int N;   // tokens per head
  int Np;  // N rounded up to whole 128-token tiles: the token stride of every code buffer
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
  uint32_t* cnt;  // [2][kMaxHeads] statistics CTAs done per head (K, V); 0 between passes
  float* q_mean;  // [B*H, Np/128, d] per-tile Q means (Q smoothing)
  int64_t bh_q;   // Q heads (B * H)
  int64_t bh_kv;  // K/V heads (B * Hkv; fewer than bh_q under grouped-query attention)
};

constexpr int kMaxHeads = kMaxStatHeads;

// Eight elements as FP32 from global memory (read-only path) or, SHARED,
// from shared memory.
template <typename T, bool SHARED = false>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]) {
  uint4 u = SHARED ? *reinterpret_cast<const uint4*>(p) : __ldg(reinterpret_cast<const uint4*>(p));
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

// INT8 rounding to an integer is an FP32 add of 1.5 * 2^23 (exact
// round-half-even for |v| < 2^22; here |x / s| < 128), read back from the
// bits, so no conversion instruction is needed.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

// Eight INT8 codes clamp(rne(fp32(v / s)), +-127) for one block scale
// s != 0, packed little-endian (code of v[i] in byte i).  The bracket test
// runs on the whole vector without a branch: for each value the
// two ends are rounded to integers by one FFMA2 each (q * bound + 1.5 * 2^23,
// a single rounding of the exact product, as monotonic as the quotient),
// and their bit patterns are XOR-accumulated; only when some end pair
// differs (or 1/s is unusable) is the vector redone on IEEE quotients.  The
// low byte of the float 1.5*2^23 + c is c mod 256, so the codes are packed
// straight from the rounded bits (|c| <= 127 here since |v| <= 127 s).
__device__ __forceinline__ uint2 int8_codes8(const float (&v)[8], float s, float rs) {
  const float2 rs2 = make_float2(rs, rs);
  const float2 lo2 = make_float2(kBracketLo, kBracketLo);
  const float2 hi2 = make_float2(kBracketHi, kBracketHi);
  const float2 m2 = make_float2(kRoundMagic, kRoundMagic);
  uint32_t hb[8];
  uint32_t diff = rs == 0.f ? 1u : 0u;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 q = __fmul2_rn(make_float2(v[e], v[e + 1]), rs2);
    const float2 a = __ffma2_rn(q, lo2, m2);
    const float2 b = __ffma2_rn(q, hi2, m2);
    diff |= (__float_as_uint(a.x) ^ __float_as_uint(b.x)) |
            (__float_as_uint(a.y) ^ __float_as_uint(b.y));
    hb[e] = __float_as_uint(b.x);
    hb[e + 1] = __float_as_uint(b.y);
  }
  if (diff != 0u) {
#pragma unroll
    for (int e = 0; e < 8; ++e) hb[e] = __float_as_uint(__fdiv_rn(v[e], s) + kRoundMagic);
  }
  const uint32_t w0 = __byte_perm(__byte_perm(hb[0], hb[1], 0x0040), __byte_perm(hb[2], hb[3], 0x0040), 0x5410);
  const uint32_t w1 = __byte_perm(__byte_perm(hb[4], hb[5], 0x0040), __byte_perm(hb[6], hb[7], 0x0040), 0x5410);
  return make_uint2(w0, w1);
}

// Eight e4m3 codes e4m3(fp32(v / s)) for one block scale s != 0, packed
// little-endian.  The same bracket test: both ends of each pair of
// quotients go through one e4m3x2 conversion each (rounding to e4m3 is
// monotonic, saturation included); any mismatch (or an unusable 1/s) redoes
// the vector on IEEE quotients.
__device__ __forceinline__ uint2 fp8_codes8(const float (&v)[8], float s, float rs) {
  const float2 rs2 = make_float2(rs, rs);
  const float2 lo2 = make_float2(kBracketLo, kBracketLo);
  const float2 hi2 = make_float2(kBracketHi, kBracketHi);
  uint32_t c[4];
  uint32_t diff = rs == 0.f ? 1u : 0u;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 q = __fmul2_rn(make_float2(v[e], v[e + 1]), rs2);
    const float2 a = __fmul2_rn(q, lo2);
    const float2 b = __fmul2_rn(q, hi2);
    const uint32_t ca = cvt_e4m3x2(a.x, a.y), cb = cvt_e4m3x2(b.x, b.y);
    diff |= ca ^ cb;
    c[e / 2] = cb;
  }
  if (diff != 0u) {
#pragma unroll
    for (int e = 0; e < 8; e += 2) c[e / 2] = cvt_e4m3x2(__fdiv_rn(v[e], s), __fdiv_rn(v[e + 1], s));
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
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

// Index of a 16-byte vector of a [128][D] tile, with padding tokens (nv and
// up) moved onto the last real token: loads stay unconditional, so they can
// all be in flight at once; the caller zeroes what it read for padding.
template <int D, bool RAGGED>
__device__ __forceinline__ int clamp_vec(int vec, int nv) {
  if (!RAGGED) return vec;
  const int t = vec / (D / 8);
  return t < nv ? vec : (nv - 1) * (D / 8) + vec % (D / 8);
}

// Copies one 128-token tile [128][D] of T into shared memory with 16-byte
// loads (consecutive threads, consecutive vectors).  Tokens nv..127 (past
// the end of a ragged sequence) are not read and stage as zeros.
template <typename T, int D, bool RAGGED>
__device__ __forceinline__ void stage_tile(const T* __restrict__ src, T* tile, int nv) {
  constexpr int VPT = 128 * D / 8 / kThreads;
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(tile);
  uint4 v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    // every load issued (a padding token re-reads a real one), then zeroed
    const int vec = threadIdx.x + i * kThreads;
    const bool pad = RAGGED && vec / (D / 8) >= nv;
    v[i] = __ldg(s + clamp_vec<D, RAGGED>(vec, nv));
    if (pad) v[i] = make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < VPT; ++i) d[threadIdx.x + i * kThreads] = v[i];
}

// ------------------------------------------------------------------ stats
// One CTA per (128-token chunk, b*h).  K: the tile is staged in shared
// memory, then thread c < D walks channel c over the chunk's tokens in
// order with an FP64 sum.  V: each thread keeps the max of |V| over its
// vectors (8 channels each) and merges it into a shared per-channel max
// (non-negative floats order like their bit patterns).
template <typename T, int D, bool RAGGED>
__device__ __forceinline__ void role_stats(const PrepassPtrs& p, int64_t bh, int chunk, int nv,
                                           bool do_k, bool do_v, T* tile, uint32_t* vmax_s) {
  constexpr int VPT = 128 * D / 8 / kThreads;
  const int nchunks = (RAGGED ? p.Np : p.N) / 128;
  const int t = threadIdx.x;
  const int64_t row0 = bh * p.N + (int64_t)chunk * 128;
  const int64_t out = (bh * nchunks + chunk) * D;
  if (do_v && t < D) vmax_s[t] = 0u;
  if (do_k) stage_tile<T, D, RAGGED>(reinterpret_cast<const T*>(p.k) + row0 * D, tile, nv);
  __syncthreads();
  if (do_v) {
    const T* src = reinterpret_cast<const T*>(p.v) + row0 * D;
    const int c0 = (t % (D / 8)) * 8;
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vec = t + i * kThreads;
      float x[8];
      load8(src + clamp_vec<D, RAGGED>(vec, nv) * 8, x);  // a re-read real token changes no max
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(x[e]));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicMax(vmax_s + c0 + e, __float_as_uint(m[e]));
  }
  __syncthreads();
  if (t < D) {
    if (do_k) {
      // the chunk's tokens in order (its first nv tokens)
      double acc = 0.0;
#pragma unroll 16
      for (int i = 0; i < nv; ++i) acc += (double)static_cast<float>(tile[i * D + t]);
      p.ksum[out + t] = acc;
    }
    if (do_v) p.vmax[out + t] = __uint_as_float(vmax_s[t]);
  }
  // The last chunk of this head to finish folds all partials (threadfence
  // reduction: each CTA publishes its partials before taking a ticket, the
  // CTA with the last ticket sees every partial).
  __shared__ int last[2];
  __threadfence();
  __syncthreads();
  if (t == 0) {
    last[0] = do_k && atomicAdd(p.cnt + bh, 1u) == (uint32_t)(nchunks - 1);
    last[1] = do_v && atomicAdd(p.cnt + kMaxHeads + bh, 1u) == (uint32_t)(nchunks - 1);
  }
  __syncthreads();
  if (!last[0] && !last[1]) return;
  __threadfence();
  if (t < D) {
    const int64_t base = bh * nchunks * D + t;
    if (last[0]) {
      // sum of the chunk partials in chunk order; mean = fp32(sum / N)
      double acc = 0.0;
      for (int i = 0; i < nchunks; ++i) acc += __ldcg(p.ksum + base + (int64_t)i * D);
      p.k_mean[bh * D + t] = __double2float_rn(__ddiv_rn(acc, (double)p.N));
    }
    if (last[1]) {
      // s_V = fp32(amax / 448)
      float m = 0.f;
      for (int i = 0; i < nchunks; ++i) m = fmaxf(m, __ldcg(p.vmax + base + (int64_t)i * D));
      p.v_scales[bh * D + t] = __fdiv_rn(m, 448.f);
    }
  }
  if (t == 0) {
    if (last[0]) p.cnt[bh] = 0u;
    if (last[1]) p.cnt[kMaxHeads + bh] = 0u;
  }
}

// ------------------------------------------------------- INT8 / FP8 Q / K
// Load, (smooth), block amax, s = amax / 127, codes = clamp(rne(x / s))
// (FP8: s = amax / 448, codes = e4m3(x / s)).  Blocks of GROUP tokens:
// GROUP = 1 (Q: one scale per query row) or 32 (K: one scale per 32 keys).
// Two passes over the 128-token tile: the amax pass keeps one maximum per
// vector, the code pass reads the tile again (from L1/L2), so the role needs
// few registers and many CTAs fit on an SM.  A thread's vectors all cover
// the same 8 channels: vector i of thread t holds token t / (D/8) + TPI i.
// SHARED: the tile and the mean are in shared memory (the cluster-fused
// pre-pass), else in global memory.  scale_out: the tile's first scale
// (128 per tile for GROUP = 1, 4 for GROUP = 32); red: 4 * kThreads / 32
// floats of shared memory.
template <typename T, int D, bool FP8, bool RAGGED, int GROUP, bool SHARED = false>
__device__ __forceinline__ void role_quant_8bit(const T* __restrict__ src, const float* mean,
                                                uint8_t* __restrict__ dst, float* scale_out,
                                                float* red, int nv) {
  static_assert(GROUP == 1 || GROUP == 32, "Q scales per token, K scales per 32 tokens");
  constexpr int VPT = 128 * D / 8 / kThreads;  // 16-byte vectors per thread
  constexpr int VPTOK = D / 8;                 // vectors per token
  constexpr int TPI = kThreads / VPTOK;        // tokens between a thread's vectors
  constexpr int VPB = 32 / TPI;                // a thread's vectors per 32-token block
  static_assert(VPB * TPI == 32 && VPT / VPB == 4, "four 32-token blocks per tile");
  const int tok0 = threadIdx.x / VPTOK;
  const int c0 = (threadIdx.x % VPTOK) * 8;
  // x - mu as x + (-mu): the same single rounding
  float nmu[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (mean) {
    const float4 a = SHARED ? *reinterpret_cast<const float4*>(mean + c0)
                            : __ldg(reinterpret_cast<const float4*>(mean + c0));
    const float4 b = SHARED ? *reinterpret_cast<const float4*>(mean + c0 + 4)
                            : __ldg(reinterpret_cast<const float4*>(mean + c0 + 4));
    nmu[0] = -a.x; nmu[1] = -a.y; nmu[2] = -a.z; nmu[3] = -a.w;
    nmu[4] = -b.x; nmu[5] = -b.y; nmu[6] = -b.z; nmu[7] = -b.w;
  }
  auto smooth = [&](float (&x)[8]) {
    if (mean) {
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float2 t = __fadd2_rn(make_float2(x[e], x[e + 1]), make_float2(nmu[e], nmu[e + 1]));
        x[e] = t.x;
        x[e + 1] = t.y;
      }
    }
  };
  // tokens nv..127 (padding of a ragged sequence) re-read the last real
  // token, so no maximum of a block holding real tokens changes; they get
  // code 0, and a block of padding only gets scale 0
  float amax[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    float x[8];
    load8<T, SHARED>(src + clamp_vec<D, RAGGED>(vec, nv) * 8, x);
    smooth(x);
    float a = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[e]));
    amax[i] = a;
  }
  float s[GROUP == 1 ? VPT : 4];
  if constexpr (GROUP == 1) {
    // one token's vectors sit in VPTOK consecutive lanes
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      float a = amax[i];
#pragma unroll
      for (int o = VPTOK / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      const int tok = tok0 + TPI * i;
      s[i] = (RAGGED && tok >= nv) ? 0.f : __fdiv_rn(a, FP8 ? 448.f : 127.f);
      if (threadIdx.x % VPTOK == 0) scale_out[tok] = s[i];
    }
  } else {
    // the four block maxima over the whole CTA
    float bm[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float a = amax[VPB * b];
#pragma unroll
      for (int v = 1; v < VPB; ++v) a = fmaxf(a, amax[VPB * b + v]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      bm[b] = a;
    }
    const int w = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
      for (int b = 0; b < 4; ++b) red[4 * w + b] = bm[b];
    }
    __syncthreads();
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float a = red[b];
#pragma unroll
      for (int i = 1; i < kThreads / 32; ++i) a = fmaxf(a, red[4 * i + b]);
      s[b] = (RAGGED && 32 * b >= nv) ? 0.f : __fdiv_rn(a, FP8 ? 448.f : 127.f);
    }
    if (threadIdx.x < 4) scale_out[threadIdx.x] = s[threadIdx.x];
  }
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    const float si = s[GROUP == 1 ? i : i / VPB];
    uint2 w = make_uint2(0u, 0u);
    if (si != 0.f) {
      const float rs = recip_or_zero(si);
      float x[8];
      load8<T, SHARED>(src + clamp_vec<D, RAGGED>(vec, nv) * 8, x);
      smooth(x);
      w = FP8 ? fp8_codes8(x, si, rs) : int8_codes8(x, si, rs);
    }
    if (RAGGED && vec / VPTOK >= nv) w = make_uint2(0u, 0u);
    *reinterpret_cast<uint2*>(dst + vec * 8) = w;
  }
}

// ------------------------------------------------------- smoothed Q
// Q smoothing (SageAttention2 abstract: "we propose a method to smooth Q"):
// the tile is staged in shared memory, thread c < D takes the FP64 sum of
// channel c over the tile's real tokens in token order, qbar = fp32(sum /
// count) goes to global memory and to shared memory, and the tile is
// encoded as Q - qbar (one FP32 subtraction) with the 8-bit encoder.
template <typename T, int D, bool RAGGED>
__device__ __forceinline__ void stage_tile_mean(const T* __restrict__ src, float* q_mean_out,
                                                T* tile, float* mean_s, int nv) {
  stage_tile<T, D, RAGGED>(src, tile, nv);
  __syncthreads();
  const int t = threadIdx.x;
  if (t < D) {
    double acc = 0.0;
#pragma unroll 16
    for (int i = 0; i < nv; ++i) acc += (double)static_cast<float>(tile[i * D + t]);
    const float m = __double2float_rn(__ddiv_rn(acc, (double)nv));
    mean_s[t] = m;
    q_mean_out[t] = m;
  }
  __syncthreads();
}

template <typename T, int D, bool FP8, bool RAGGED>
__device__ __forceinline__ void role_quant_q_smooth(const T* __restrict__ src, float* q_mean_out,
                                                    uint8_t* __restrict__ dst, float* scale_out,
                                                    T* tile, float* mean_s, float* red, int nv) {
  stage_tile_mean<T, D, RAGGED>(src, q_mean_out, tile, mean_s, nv);
  role_quant_8bit<T, D, FP8, RAGGED, 1, true>(tile, mean_s, dst, scale_out, red, nv);
}

// ---------------------------------------------------------------- FP8 V
// codes = e4m3(V / s_V[c]) written transposed into V^T.  The tile is staged
// in shared memory; a thread then owns a channel pair and 32 consecutive
// tokens (reads conflict-free: consecutive threads, consecutive pairs) and
// writes each channel's 32 codes as one 32-byte sector (two 16-byte stores).  The bracket
// test of the INT8 path runs per pair of tokens: both ends of two tokens go
// through one e4m3x2 conversion each, and the two 16-bit results must match
// (else the unit is redone on IEEE quotients); the matching result is the
// two codes, already packed.
// The encoding of one staged tile (shared memory, padding tokens zero); vs:
// the head's s_V (global or shared memory).
template <typename T, int D>
__device__ __forceinline__ void encode_v_fp8_tile(const T* tile, const float* vs,
                                                  uint8_t* __restrict__ dst, int N) {
  constexpr int UNITS = (D / 2) * 4;  // channel pairs x 32-token groups
  const float2 lo2 = make_float2(kBracketLo, kBracketLo);
  const float2 hi2 = make_float2(kBracketHi, kBracketHi);
  for (int u = threadIdx.x; u < UNITS; u += kThreads) {
    const int cp = u % (D / 2), grp = u / (D / 2);
    const float s0 = vs[2 * cp], s1 = vs[2 * cp + 1];
    const float r0 = recip_or_zero(s0), r1 = recip_or_zero(s1);
    const uint32_t* col = reinterpret_cast<const uint32_t*>(tile) + (grp * 32) * (D / 2) + cp;
    auto pair_of = [&](int tok, float& x0, float& x1) {
      const uint32_t w = col[tok * (D / 2)];
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        x0 = __uint_as_float(w << 16);
        x1 = __uint_as_float(w & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
        x0 = f.x;
        x1 = f.y;
      }
    };
    // 1/s unusable for a nonzero scale: decide on quotients throughout
    const uint32_t bad = ((s0 != 0.f && r0 == 0.f) || (s1 != 0.f && r1 == 0.f)) ? 1u : 0u;
    // dst points at V^T[c = 0][tile start]
    uint8_t* d0 = dst + (int64_t)(2 * cp) * N + grp * 32;
    uint8_t* d1 = dst + (int64_t)(2 * cp + 1) * N + grp * 32;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t diff = bad;
      uint32_t w0[4], w1[4];
#pragma unroll
      for (int k = 0; k < 16; k += 4) {
        float a[4], b[4];  // channel 2cp / 2cp+1 at 4 consecutive tokens
#pragma unroll
        for (int i = 0; i < 4; ++i) pair_of(16 * half + k + i, a[i], b[i]);
        uint32_t ca[2], cb[2];
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
          const float2 qa = __fmul2_rn(make_float2(a[i], a[i + 1]), make_float2(r0, r0));
          const float2 qb = __fmul2_rn(make_float2(b[i], b[i + 1]), make_float2(r1, r1));
          const float2 qal = __fmul2_rn(qa, lo2), qah = __fmul2_rn(qa, hi2);
          const float2 qbl = __fmul2_rn(qb, lo2), qbh = __fmul2_rn(qb, hi2);
          const uint32_t al = cvt_e4m3x2(qal.x, qal.y), ah = cvt_e4m3x2(qah.x, qah.y);
          const uint32_t bl = cvt_e4m3x2(qbl.x, qbl.y), bhh = cvt_e4m3x2(qbh.x, qbh.y);
          diff |= (al ^ ah) | (bl ^ bhh);
          ca[i >> 1] = ah;
          cb[i >> 1] = bhh;
        }
        w0[k >> 2] = ca[0] | (ca[1] << 16);
        w1[k >> 2] = cb[0] | (cb[1] << 16);
      }
      if (diff != 0u) {
#pragma unroll 1
        for (int k = 0; k < 16; k += 4) {
          float a[4], b[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) pair_of(16 * half + k + i, a[i], b[i]);
          w0[k >> 2] = cvt_e4m3x2(__fdiv_rn(a[0], s0), __fdiv_rn(a[1], s0)) |
                       (cvt_e4m3x2(__fdiv_rn(a[2], s0), __fdiv_rn(a[3], s0)) << 16);
          w1[k >> 2] = cvt_e4m3x2(__fdiv_rn(b[0], s1), __fdiv_rn(b[1], s1)) |
                       (cvt_e4m3x2(__fdiv_rn(b[2], s1), __fdiv_rn(b[3], s1)) << 16);
        }
      }
      // a zero scale (an all-zero channel) gives +0 codes
      const uint4 v0 = s0 != 0.f ? make_uint4(w0[0], w0[1], w0[2], w0[3]) : make_uint4(0, 0, 0, 0);
      const uint4 v1 = s1 != 0.f ? make_uint4(w1[0], w1[1], w1[2], w1[3]) : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(d0 + 16 * half) = v0;
      *reinterpret_cast<uint4*>(d1 + 16 * half) = v1;
    }
  }
}

template <typename T, int D, bool RAGGED>
__device__ __forceinline__ void role_quant_v_fp8(const T* __restrict__ src,
                                                 const float* __restrict__ vs,
                                                 uint8_t* __restrict__ dst, int N, T* tile,
                                                 int nv) {
  // padding tokens stage as zeros and so get code 0; N is the row length of
  // V^T (the padded token count)
  stage_tile<T, D, RAGGED>(src, tile, nv);
  __syncthreads();
  encode_v_fp8_tile<T, D>(tile, vs, dst, N);
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
// SHARED: the tile and the mean are in shared memory (the smoothed Q role).
template <typename T, int D, bool RAGGED, bool SHARED = false>
__device__ __forceinline__ void role_quant_fp4_tokens(const T* __restrict__ src, const float* mean,
                                                      uint8_t* __restrict__ codes, float* g_out,
                                                      uint8_t* __restrict__ sf, int64_t bh,
                                                      int ntiles, int tile, float* red, int nv) {
  constexpr int G = D / 16;                // groups per row
  constexpr int GPT = 128 * G / kThreads;  // groups per thread
  float x[GPT][16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < GPT; ++i) {
    const int grp = threadIdx.x + i * kThreads;
    const int r = grp / G, gc = grp % G;
    // a padding row re-reads the last real row (loads stay unconditional)
    // and is zeroed below: code 0, scale 0
    const int rr = (!RAGGED || r < nv) ? r : nv - 1;
    float a[8], b[8];
    load8<T, SHARED>(src + rr * D + gc * 16, a);
    load8<T, SHARED>(src + rr * D + gc * 16 + 8, b);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[i][e] = a[e];
      x[i][8 + e] = b[e];
    }
    if (mean) {
      const float* mu = mean + gc * 16;
#pragma unroll
      for (int e = 0; e < 16; ++e) x[i][e] = __fsub_rn(x[i][e], SHARED ? mu[e] : __ldg(mu + e));
    }
    if (RAGGED && r >= nv) {
#pragma unroll
      for (int e = 0; e < 16; ++e) x[i][e] = 0.f;
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
template <typename T, int D, bool RAGGED>
__device__ __forceinline__ void role_quant_fp4_v(const T* __restrict__ src, int N,
                                                 uint8_t* __restrict__ vt_codes, float* g_out,
                                                 uint8_t* __restrict__ v_sf, int64_t bh,
                                                 int ntiles, int tile, T (*xs)[D + 2],
                                                 float* red, int nv) {
  constexpr int VPT = 128 * D / 8 / kThreads;
  constexpr int PAIRS = D * 8;  // channels x 16-token groups
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vec = threadIdx.x + i * kThreads;
    const int t = vec / (D / 8), c0 = (vec % (D / 8)) * 8;
    // a padding token re-reads a real one (no change to the max) and
    // stages as zeros
    const bool pad = RAGGED && t >= nv;
    const int cv = clamp_vec<D, RAGGED>(vec, nv);
    float x[8];
    load8(src + cv * 8, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      xs[t][c0 + e] = pad ? static_cast<T>(0.f) : src[cv * 8 + e];
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
// RAGGED: N is not a multiple of 128, so the last tile is partial (without
// it every guard on padding tokens compiles away).
template <typename T, int D, int MASK, bool RAGGED>
__global__ void __launch_bounds__(kThreads) prepass_kernel(PrepassPtrs p, Roles roles) {
  // one staging buffer, sized for the largest role of the mask (a CTA runs
  // one role)
  constexpr bool kV4 = ((MASK >> kQuantV4) & 1) != 0;
  constexpr bool kTile = ((MASK >> kQuantV8) & 1) || ((MASK >> kStatsK) & 1) ||
                         ((MASK >> kStatsKV) & 1) || ((MASK >> kQuantQ8S) & 1) ||
                         ((MASK >> kQuantQF8S) & 1) || ((MASK >> kQuantQ4S) & 1);
  constexpr int V4_BYTES = kV4 ? 128 * (D + 2) * (int)sizeof(T) : 16;
  constexpr int TILE_BYTES = kTile ? 128 * D * (int)sizeof(T) : 16;
  constexpr int SMEM_BYTES = V4_BYTES > TILE_BYTES ? V4_BYTES : TILE_BYTES;
  __shared__ __align__(16) uint8_t smem_raw[SMEM_BYTES];
  __shared__ uint32_t vmax_s[D];
  __shared__ float red[4 * (kThreads / 32)];
  __shared__ __align__(16) float qmean_s[D];
  const int role = roles.r[blockIdx.z];
  const int64_t bh = roles.reverse ? (int64_t)(gridDim.y - 1 - blockIdx.y) : (int64_t)blockIdx.y;
  const int tile = roles.reverse ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  // the grid spans the larger head count: Q roles cover bh_q heads, K/V
  // roles bh_kv (a CTA leaves as a whole, before any barrier)
  const bool q_role = role == kQuantQ8 || role == kQuantQ4 || role == kQuantQF8 ||
                      role == kQuantQ8S || role == kQuantQF8S || role == kQuantQ4S;
  if (bh >= (q_role ? p.bh_q : p.bh_kv)) return;
  // (without RAGGED, Np == N: the same offsets as before padding existed)
  const int ntiles = (RAGGED ? p.Np : p.N) / 128;
  const int nv = RAGGED ? min(128, p.N - tile * 128) : 128;  // real tokens of this tile
  const int64_t row0 = bh * p.N + (int64_t)tile * 128;       // input rows
  const int64_t crow0 = RAGGED ? bh * p.Np + (int64_t)tile * 128 : row0;  // code rows
  const int Np = RAGGED ? p.Np : p.N;
  switch (role) {
    case kQuantQ8:
      SAGE_ROLE(kQuantQ8)
      role_quant_8bit<T, D, false, RAGGED, 1>(reinterpret_cast<const T*>(p.q) + row0 * D, nullptr,
                                   reinterpret_cast<uint8_t*>(p.q_codes) + crow0 * D,
                                   p.q_scales + crow0, red, nv);
      break;
    case kQuantK8:
      SAGE_ROLE(kQuantK8)
      role_quant_8bit<T, D, false, RAGGED, 32>(reinterpret_cast<const T*>(p.k) + row0 * D,
                                   p.k_mean + bh * D,
                                   reinterpret_cast<uint8_t*>(p.k_codes) + crow0 * D,
                                   p.k_scales + crow0 / 32, red, nv);
      break;
    case kQuantQF8:
      SAGE_ROLE(kQuantQF8)
      role_quant_8bit<T, D, true, RAGGED, 1>(reinterpret_cast<const T*>(p.q) + row0 * D, nullptr,
                                  reinterpret_cast<uint8_t*>(p.q_codes) + crow0 * D,
                                  p.q_scales + crow0, red, nv);
      break;
    case kQuantKF8:
      SAGE_ROLE(kQuantKF8)
      role_quant_8bit<T, D, true, RAGGED, 32>(reinterpret_cast<const T*>(p.k) + row0 * D,
                                  p.k_mean + bh * D,
                                  reinterpret_cast<uint8_t*>(p.k_codes) + crow0 * D,
                                  p.k_scales + crow0 / 32, red, nv);
      break;
    case kQuantQ8S:
      SAGE_ROLE(kQuantQ8S)
      role_quant_q_smooth<T, D, false, RAGGED>(
          reinterpret_cast<const T*>(p.q) + row0 * D, p.q_mean + (bh * ntiles + tile) * D,
          reinterpret_cast<uint8_t*>(p.q_codes) + crow0 * D, p.q_scales + crow0,
          reinterpret_cast<T*>(smem_raw), qmean_s, red, nv);
      break;
    case kQuantQF8S:
      SAGE_ROLE(kQuantQF8S)
      role_quant_q_smooth<T, D, true, RAGGED>(
          reinterpret_cast<const T*>(p.q) + row0 * D, p.q_mean + (bh * ntiles + tile) * D,
          reinterpret_cast<uint8_t*>(p.q_codes) + crow0 * D, p.q_scales + crow0,
          reinterpret_cast<T*>(smem_raw), qmean_s, red, nv);
      break;
    case kQuantV8:
      SAGE_ROLE(kQuantV8)
      role_quant_v_fp8<T, D, RAGGED>(reinterpret_cast<const T*>(p.v) + row0 * D, p.v_scales + bh * D,
                             reinterpret_cast<uint8_t*>(p.v_codes) + bh * D * (int64_t)Np +
                                 (int64_t)tile * 128,
                             Np, reinterpret_cast<T*>(smem_raw), nv);
      break;
    case kQuantQ4:
      SAGE_ROLE(kQuantQ4)
      role_quant_fp4_tokens<T, D, RAGGED>(reinterpret_cast<const T*>(p.q) + row0 * D, nullptr,
                                  reinterpret_cast<uint8_t*>(p.q_codes) + crow0 * (D / 2),
                                  p.q_scales + bh * ntiles + tile, p.q_sf, bh, ntiles, tile, red,
                                  nv);
      break;
    case kQuantQ4S:
      SAGE_ROLE(kQuantQ4S) {
        stage_tile_mean<T, D, RAGGED>(reinterpret_cast<const T*>(p.q) + row0 * D,
                                      p.q_mean + (bh * ntiles + tile) * D,
                                      reinterpret_cast<T*>(smem_raw), qmean_s, nv);
        role_quant_fp4_tokens<T, D, RAGGED, true>(
            reinterpret_cast<const T*>(smem_raw), qmean_s,
            reinterpret_cast<uint8_t*>(p.q_codes) + crow0 * (D / 2),
            p.q_scales + bh * ntiles + tile, p.q_sf, bh, ntiles, tile, red, nv);
      }
      break;
    case kQuantK4:
      SAGE_ROLE(kQuantK4)
      role_quant_fp4_tokens<T, D, RAGGED>(reinterpret_cast<const T*>(p.k) + row0 * D, p.k_mean + bh * D,
                                  reinterpret_cast<uint8_t*>(p.k_codes) + crow0 * (D / 2),
                                  p.k_scales + bh * ntiles + tile, p.k_sf, bh, ntiles, tile, red,
                                  nv);
      break;
    case kQuantV4:
      SAGE_ROLE(kQuantV4)
      role_quant_fp4_v<T, D, RAGGED>(reinterpret_cast<const T*>(p.v) + row0 * D, Np,
                             reinterpret_cast<uint8_t*>(p.v_codes), p.v_scales + bh * ntiles + tile,
                             p.v_sf, bh, ntiles, tile, reinterpret_cast<T(*)[D + 2]>(smem_raw), red,
                             nv);
      break;
    case kStatsK:
      SAGE_ROLE(kStatsK)
      role_stats<T, D, RAGGED>(p, bh, tile, nv, true, false, reinterpret_cast<T*>(smem_raw), vmax_s);
      break;
    case kStatsKV:
      SAGE_ROLE(kStatsKV)
      role_stats<T, D, RAGGED>(p, bh, tile, nv, true, true, reinterpret_cast<T*>(smem_raw), vmax_s);
      break;
    case kStatsV:
      SAGE_ROLE(kStatsV)
      role_stats<T, D, RAGGED>(p, bh, tile, nv, false, true, reinterpret_cast<T*>(smem_raw), vmax_s);
      break;
    default:
      break;
  }
}
#undef SAGE_ROLE

// ------------------------------------------------ the cluster-fused pre-pass
// For the 8-bit modes, heads of at most 8 tiles (1024 tokens) and at most
// 16 of them, where the two-launch chains are bound by launch latency: one
// launch encodes Q, K and V.  A cluster of 8 CTAs per (b*h, tensor) holds the head's tiles in shared
// memory, one tile per CTA (one bulk copy each), and reduces the head
// statistics through distributed shared memory in the order the two-launch
// path uses (FP64 K sums per tile in token order, then tiles in order; the
// |V| maximum), so the codes are the same bits; each input is read once.
// grid (8, max(B*Hq, B*Hkv), 3): z = 0 Q codes, 1 K mean + K codes, 2 V scales
// + V codes; a cluster spans x only, so all its CTAs share (b*h, tensor).
constexpr int kFusedCluster = 8;

template <typename T, int D, bool FP8, bool RAGGED>
__global__ void __cluster_dims__(kFusedCluster, 1, 1) __launch_bounds__(kThreads)
    prepass_fused_kernel(PrepassPtrs p, uint32_t* status) {
  __shared__ __align__(128) T tile[128 * D];
  __shared__ uint64_t bar;
  __shared__ double ksum_s[D];
  __shared__ uint32_t vmax_s[D];
  __shared__ __align__(16) float stat_s[D];  // the head's K mean or s_V
  __shared__ float red[4 * (kThreads / 32)];
  __shared__ int abort_flag;
  const int role = blockIdx.z;
  const int64_t bh = blockIdx.y;
  // whole clusters leave here (before any cluster barrier)
  if (bh >= (role == 0 ? p.bh_q : p.bh_kv)) return;
  const int t = threadIdx.x;
  const int g = (int)cluster_ctarank();  // this CTA's tile
  const int Np = RAGGED ? p.Np : p.N;
  const int ntiles = Np / 128;
  const bool has = g < ntiles;
  const int nv = RAGGED ? min(128, p.N - g * 128) : 128;  // its real tokens (when has)
  const T* src = reinterpret_cast<const T*>(role == 0 ? p.q : role == 1 ? p.k : p.v) +
                 (bh * p.N + (int64_t)g * 128) * D;

  if (t == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (t < D) vmax_s[t] = 0u;
  __syncthreads();
  if (t == 0 && has) {
    const uint32_t bytes = (uint32_t)(nv * D * (int)sizeof(T));
    mbar_arrive_expect_tx(&bar, bytes);
    bulk_load(tile, src, bytes, &bar);
  }
  // padding tokens of a partial last tile stage as zeros (V codes read them)
  if (RAGGED && has && nv < 128) {
    uint4* pad = reinterpret_cast<uint4*>(tile + nv * D);
    for (int i = t; i < (128 - nv) * D / 8; i += kThreads) pad[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  // every thread observes the copy's completion before it reads the tile
  if (has) mbar_wait(&bar, 0, &abort_flag, status, kDevTimeoutTma);

  if (role == 0) {
    if (has)
      role_quant_8bit<T, D, FP8, RAGGED, 1, true>(
          tile, nullptr, reinterpret_cast<uint8_t*>(p.q_codes) + (bh * Np + g * 128) * D,
          p.q_scales + bh * Np + g * 128, red, nv);
  } else if (role == 1) {
    // FP64 sum of the tile's tokens in order, channel t
    if (has && t < D) {
      double acc = 0.0;
#pragma unroll 16
      for (int k = 0; k < nv; ++k) acc += (double)static_cast<float>(tile[k * D + t]);
      ksum_s[t] = acc;
    }
    cluster_sync();
    if (t < D) {
      // every CTA folds the tiles of the head in tile order: the same mean
      double part[kFusedCluster];
#pragma unroll
      for (int r = 0; r < kFusedCluster; ++r)
        part[r] = r < ntiles ? ld_dsmem_f64(dsmem_addr(&ksum_s[t], (uint32_t)r)) : 0.0;
      double acc = 0.0;
#pragma unroll
      for (int r = 0; r < kFusedCluster; ++r)
        if (r < ntiles) acc += part[r];
      const float mean = __double2float_rn(__ddiv_rn(acc, (double)p.N));
      stat_s[t] = mean;
      if (g == 0) p.k_mean[bh * D + t] = mean;
    }
    // no CTA leaves while others read its partials
    cluster_sync();
    if (has)
      role_quant_8bit<T, D, FP8, RAGGED, 32, true>(
          tile, stat_s, reinterpret_cast<uint8_t*>(p.k_codes) + (bh * Np + g * 128) * D,
          p.k_scales + (bh * Np + g * 128) / 32, red, nv);
  } else {
    if (has) {
      // |V| maximum per channel (a thread keeps 8 channels; a padding token
      // re-reads a real one, so no maximum changes)
      constexpr int VPT = 128 * D / 8 / kThreads;
      const int c0 = (t % (D / 8)) * 8;
      float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        float x[8];
        load8<T, true>(tile + clamp_vec<D, RAGGED>(t + j * kThreads, nv) * 8, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(x[e]));
      }
      // non-negative floats order like their bit patterns
#pragma unroll
      for (int e = 0; e < 8; ++e) atomicMax(vmax_s + c0 + e, __float_as_uint(m[e]));
    }
    cluster_sync();
    if (t < D) {
      uint32_t mb[kFusedCluster];
#pragma unroll
      for (int r = 0; r < kFusedCluster; ++r) mb[r] = ld_dsmem_u32(dsmem_addr(&vmax_s[t], (uint32_t)r));
      float mx = 0.f;
#pragma unroll
      for (int r = 0; r < kFusedCluster; ++r) mx = fmaxf(mx, __uint_as_float(mb[r]));
      const float sv = __fdiv_rn(mx, 448.f);  // s_V = fp32(amax / 448)
      stat_s[t] = sv;
      if (g == 0) p.v_scales[bh * D + t] = sv;
    }
    cluster_sync();
    if (has)
      encode_v_fp8_tile<T, D>(tile, stat_s,
                              reinterpret_cast<uint8_t*>(p.v_codes) + bh * D * (int64_t)Np +
                                  (int64_t)g * 128,
                              Np);
  }
  // after an expired wait, let the copy land before the CTA leaves
  __syncthreads();
  if (t == 0 && has && abort_flag) {
    volatile int no_abort = 0;
    mbar_wait(&bar, 0, &no_abort, status, kDevTimeoutTma);
  }
}

constexpr int bit(int r) { return 1 << r; }

// kernel A (roles a; its statistics CTAs also fold the head statistics),
// then kernel B (roles b); the grids span the larger of the Q and K/V head
// counts
// The reversed second launch pays off while the re-read K (or V) fits in
// half of the 126 MB L2 (llm, 32 MB: the chains 2 us faster); on larger
// tensors nothing is left to hit and the forward order is slightly faster.
constexpr int64_t kReverseMaxBytes = int64_t(64) << 20;

template <typename T, int D, int MA, int MB>
cudaError_t run_plan(const PrepassPtrs& p, Roles a, Roles b, cudaStream_t st) {
  b.reverse = p.bh_kv * (int64_t)p.N * D * (int64_t)sizeof(T) <= kReverseMaxBytes;
  const int ntiles = p.Np / 128;
  const int64_t BH = p.bh_q > p.bh_kv ? p.bh_q : p.bh_kv;
  const dim3 grid_a(ntiles, (unsigned)BH, a.n), grid_b(ntiles, (unsigned)BH, b.n);
  if (p.N % 128 != 0) {
    if (a.n) prepass_kernel<T, D, MA, true><<<grid_a, kThreads, 0, st>>>(p, a);
    if (b.n) prepass_kernel<T, D, MB, true><<<grid_b, kThreads, 0, st>>>(p, b);
  } else {
    if (a.n) prepass_kernel<T, D, MA, false><<<grid_a, kThreads, 0, st>>>(p, a);
    if (b.n) prepass_kernel<T, D, MB, false><<<grid_b, kThreads, 0, st>>>(p, b);
  }
  return cudaGetLastError();
}

// MA / MB: the role masks of kernels A and B (they must cover a.r / b.r).
template <int MA, int MB>
cudaError_t dispatch(const PrepassPtrs& p, int dtype, int64_t d, Roles a, Roles b,
                     cudaStream_t st) {
  if (dtype == 1)
    return d == 128 ? run_plan<__nv_bfloat16, 128, MA, MB>(p, a, b, st)
                    : run_plan<__nv_bfloat16, 64, MA, MB>(p, a, b, st);
  return d == 128 ? run_plan<__half, 128, MA, MB>(p, a, b, st)
                  : run_plan<__half, 64, MA, MB>(p, a, b, st);
}

// ------------------------------------------------- smoothing bias dS
// dS[bh, blk, j] = fp32(sum_c qbar[bh, blk, c] * k'[j, c]), k' = fp32(K) -
// mean_K of the key/value head, the sum in FP64 in channel order (products
// of FP32 values are exact in FP64, so FMA and multiply-then-add agree):
// the oracle's arithmetic, bit for bit.  The work is B H N^2 d / 128 FP64
// FMAs, so the kernel is built to keep the FP64 pipe busy: a CTA takes 256
// keys and 32 query blocks of one query head, a thread two keys (tx and
// tx + 128) against all 32 blocks (64 FP64 accumulators).  A thread reads
// its keys' rows itself, 8 channels per 16-byte load issued one step ahead;
// the block means sit in shared memory as [channel][block] doubles, and
// every warp reads the same 16 bytes at once (a broadcast), so shared
// memory serves one load per four FMAs of a warp.  Keys past N get 0.
constexpr int kBiasThreads = 128;
constexpr int kBiasKeys = 2 * kBiasThreads;
constexpr int kBiasBlocks = 32;

template <int D>
constexpr int bias_smem_bytes() {
  return D * kBiasBlocks * 8 + D * 4;
}

// 8 channels of a K row (one 16-byte load, u) as FP32 values minus the mean
template <typename T>
__device__ __forceinline__ void k_smoothed8(const uint4 u, const float* mu, float (&kv)[8]) {
  T v[8];
  memcpy(v, &u, 16);
#pragma unroll
  for (int e = 0; e < 8; ++e) kv[e] = __fsub_rn(static_cast<float>(v[e]), mu[e]);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBiasThreads)
    smoothing_bias_kernel(const T* __restrict__ k, const float* __restrict__ k_mean,
                          const float* __restrict__ q_mean, float* __restrict__ ds, int N, int Np,
                          int nblk, int H, int G) {
  extern __shared__ __align__(16) double bias_smem[];
  double* qs = bias_smem;                                          // [D][32] qbar
  float* mu = reinterpret_cast<float*>(bias_smem + D * kBiasBlocks);  // [D] K mean
  const int bh = (int)blockIdx.z;
  const int bhk = kv_head(bh, H, G);
  const int j0 = (int)blockIdx.x * kBiasKeys;
  const int b0 = (int)blockIdx.y * kBiasBlocks;
  const int nb = min(kBiasBlocks, nblk - b0);
  const int t = threadIdx.x;
  // block-fastest order: a warp's 32 stores fill one channel's row of 32
  // doubles (no bank conflicts)
  for (int i = t; i < kBiasBlocks * D; i += kBiasThreads) {
    const int blk = i % kBiasBlocks, c = i / kBiasBlocks;
    qs[c * kBiasBlocks + blk] =
        blk < nb ? (double)q_mean[((int64_t)bh * nblk + b0 + blk) * D + c] : 0.0;
  }
  for (int c = t; c < D; c += kBiasThreads) mu[c] = k_mean[(int64_t)bhk * D + c];
  __syncthreads();
  // this thread's keys; rows past N read row N - 1 (their sums are not stored)
  const int ja = j0 + t, jb = j0 + kBiasThreads + t;
  const T* ra = k + ((int64_t)bhk * N + min(ja, N - 1)) * D;
  const T* rb = k + ((int64_t)bhk * N + min(jb, N - 1)) * D;
  double acc[2][kBiasBlocks];
#pragma unroll
  for (int i = 0; i < kBiasBlocks; ++i) acc[0][i] = acc[1][i] = 0.0;
  // the next 8 channels of both rows are loaded while these are summed
  uint4 ua = __ldg(reinterpret_cast<const uint4*>(ra));
  uint4 ub = __ldg(reinterpret_cast<const uint4*>(rb));
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 8) {
    float ka[8], kb[8];
    k_smoothed8<T>(ua, mu + c0, ka);
    k_smoothed8<T>(ub, mu + c0, kb);
    if (c0 + 8 < D) {
      ua = __ldg(reinterpret_cast<const uint4*>(ra + c0 + 8));
      ub = __ldg(reinterpret_cast<const uint4*>(rb + c0 + 8));
    }
    // channels c0 .. c0 + 7 in order: the channel order of every sum
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double da = (double)ka[e], db = (double)kb[e];
      const double2* q2 = reinterpret_cast<const double2*>(qs + (c0 + e) * kBiasBlocks);
#pragma unroll
      for (int i = 0; i < kBiasBlocks / 2; ++i) {
        const double2 q = q2[i];
        acc[0][2 * i] = __fma_rn(q.x, da, acc[0][2 * i]);
        acc[0][2 * i + 1] = __fma_rn(q.y, da, acc[0][2 * i + 1]);
        acc[1][2 * i] = __fma_rn(q.x, db, acc[1][2 * i]);
        acc[1][2 * i + 1] = __fma_rn(q.y, db, acc[1][2 * i + 1]);
      }
    }
  }
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int j = kk ? jb : ja;
    if (j >= Np) continue;
#pragma unroll
    for (int i = 0; i < kBiasBlocks; ++i)
      if (i < nb)
        ds[((int64_t)bh * nblk + b0 + i) * Np + j] = j < N ? __double2float_rn(acc[kk][i]) : 0.f;
  }
}

template <typename T, int D>
cudaError_t run_bias(const QuantQKArgs& a, cudaStream_t st) {
  auto kern = smoothing_bias_kernel<T, D>;
  const cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bias_smem_bytes<D>());
  if (e != cudaSuccess) return e;
  const int Np = (int)((a.N + 127) / 128 * 128);
  const int nblk = Np / 128;
  const dim3 grid((unsigned)((Np + kBiasKeys - 1) / kBiasKeys),
                  (unsigned)((nblk + kBiasBlocks - 1) / kBiasBlocks), (unsigned)(a.B * a.H));
  kern<<<grid, kBiasThreads, bias_smem_bytes<D>(), st>>>(
      static_cast<const T*>(a.k), a.k_mean, a.q_mean, a.ds, (int)a.N, Np, nblk, (int)a.H,
      (int)(a.H / a.Hkv));
  return cudaGetLastError();
}

cudaError_t launch_smoothing_bias(const QuantQKArgs& a, cudaStream_t st) {
  if (a.dtype == 1)
    return a.d == 128 ? run_bias<__nv_bfloat16, 128>(a, st) : run_bias<__nv_bfloat16, 64>(a, st);
  return a.d == 128 ? run_bias<__half, 128>(a, st) : run_bias<__half, 64>(a, st);
}

PrepassPtrs ptrs_qk(const QuantQKArgs& a) {
  PrepassPtrs p{};
  p.q = a.q;
  p.k = a.k;
  p.N = (int)a.N;
  p.Np = (int)((a.N + 127) / 128 * 128);
  p.q_codes = a.q_codes;
  p.q_scales = a.q_scales;
  p.q_sf = static_cast<uint8_t*>(a.q_sf);
  p.k_codes = a.k_codes;
  p.k_scales = a.k_scales;
  p.k_sf = static_cast<uint8_t*>(a.k_sf);
  p.k_mean = a.k_mean;
  p.ksum = a.ws_ksum;
  p.cnt = a.ws_cnt;
  p.q_mean = a.q_mean;
  p.bh_q = a.B * a.H;
  p.bh_kv = a.B * a.Hkv;
  return p;
}

void add_v(PrepassPtrs& p, const QuantVArgs& a) {
  p.v = a.v;
  p.N = (int)a.N;
  p.Np = (int)((a.N + 127) / 128 * 128);
  p.v_codes = a.v_codes;
  p.v_scales = a.v_scales;
  p.v_sf = static_cast<uint8_t*>(a.v_sf);
  p.vmax = a.ws_vmax;
  p.cnt = a.ws_cnt;
  p.bh_kv = a.B * a.H;  // QuantVArgs counts K/V heads in H
}

template <typename T, int D, bool FP8>
cudaError_t run_fused(const PrepassPtrs& p, uint32_t* status, cudaStream_t st) {
  const int64_t BH = p.bh_q > p.bh_kv ? p.bh_q : p.bh_kv;
  const dim3 grid(kFusedCluster, (unsigned)BH, 3);
  if (p.N % 128 != 0)
    prepass_fused_kernel<T, D, FP8, true><<<grid, kThreads, 0, st>>>(p, status);
  else
    prepass_fused_kernel<T, D, FP8, false><<<grid, kThreads, 0, st>>>(p, status);
  return cudaGetLastError();
}

}  // namespace

// The fused kernel runs at two CTAs per SM (its registers): it beats the
// chains while the whole pre-pass is about one wave of it (launch latency
// bound), and loses to them on many heads, where they overlap loads better
// (256 heads of 1024 tokens: 0.153 ms against 0.103).
constexpr int64_t kFusedMaxHeads = 16;

bool fused_prepass_fits(const QuantQKArgs& a) {
  const int64_t ntiles = (a.N + 127) / 128;
  const int64_t BH = a.B * a.H;
  return a.mode != kModeFp4 && a.status != nullptr && a.q_mean == nullptr && ntiles > 0 &&
         ntiles <= kFusedCluster && BH <= kFusedMaxHeads && (a.d == 64 || a.d == 128);
}

cudaError_t launch_prepass_fused(const QuantQKArgs& qa, const QuantVArgs& va, cudaStream_t st) {
  PrepassPtrs p = ptrs_qk(qa);
  add_v(p, va);
  const bool fp8 = qa.mode == kModeFp8;
  if (qa.dtype == 1) {
    if (qa.d == 128)
      return fp8 ? run_fused<__nv_bfloat16, 128, true>(p, qa.status, st)
                 : run_fused<__nv_bfloat16, 128, false>(p, qa.status, st);
    return fp8 ? run_fused<__nv_bfloat16, 64, true>(p, qa.status, st)
               : run_fused<__nv_bfloat16, 64, false>(p, qa.status, st);
  }
  if (qa.d == 128)
    return fp8 ? run_fused<__half, 128, true>(p, qa.status, st)
               : run_fused<__half, 128, false>(p, qa.status, st);
  return fp8 ? run_fused<__half, 64, true>(p, qa.status, st)
             : run_fused<__half, 64, false>(p, qa.status, st);
}

cudaError_t launch_quant_qk(const QuantQKArgs& a, cudaStream_t st) {
  const PrepassPtrs p = ptrs_qk(a);
  if (a.q_mean) {
    // Q smoothing: smoothed Q codes and the means beside the K
    // statistics, then the K codes, then the bias (it needs both means)
    cudaError_t e;
    if (a.mode == kModeInt8Fp8)
      e = dispatch<bit(kQuantQ8S) | bit(kStatsK), bit(kQuantK8)>(
          p, a.dtype, a.d, Roles{2, {kQuantQ8S, kStatsK}}, Roles{1, {kQuantK8}}, st);
    else if (a.mode == kModeFp8)
      e = dispatch<bit(kQuantQF8S) | bit(kStatsK), bit(kQuantKF8)>(
          p, a.dtype, a.d, Roles{2, {kQuantQF8S, kStatsK}}, Roles{1, {kQuantKF8}}, st);
    else
      e = dispatch<bit(kQuantQ4S) | bit(kStatsK), bit(kQuantK4)>(
          p, a.dtype, a.d, Roles{2, {kQuantQ4S, kStatsK}}, Roles{1, {kQuantK4}}, st);
    if (e != cudaSuccess) return e;
    return launch_smoothing_bias(a, st);
  }
  if (a.mode == kModeInt8Fp8)
    return dispatch<bit(kQuantQ8) | bit(kStatsK), bit(kQuantK8)>(
        p, a.dtype, a.d, Roles{2, {kQuantQ8, kStatsK}}, Roles{1, {kQuantK8}}, st);
  if (a.mode == kModeFp8)
    return dispatch<bit(kQuantQF8) | bit(kStatsK), bit(kQuantKF8)>(
        p, a.dtype, a.d, Roles{2, {kQuantQF8, kStatsK}}, Roles{1, {kQuantKF8}}, st);
  return dispatch<bit(kQuantQ4) | bit(kStatsK), bit(kQuantK4)>(
      p, a.dtype, a.d, Roles{2, {kQuantQ4, kStatsK}}, Roles{1, {kQuantK4}}, st);
}

cudaError_t launch_quant_v(const QuantVArgs& a, cudaStream_t st) {
  PrepassPtrs p{};
  add_v(p, a);
  if (a.mode != kModeFp4)
    return dispatch<bit(kStatsV), bit(kQuantV8)>(p, a.dtype, a.d, Roles{1, {kStatsV}},
                                                 Roles{1, {kQuantV8}}, st);
  return dispatch<bit(kQuantV4), 0>(p, a.dtype, a.d, Roles{1, {kQuantV4}},
                                    Roles{0, {}}, st);
}


}  // namespace sage
