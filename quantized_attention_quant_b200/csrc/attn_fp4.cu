// attn_fp4.cu -- fused FP4 (E2M1 with UE4M3 scales per 16 elements and an
// FP32 scale per 128-token tile) attention forward for sm_100a.
//
// What it computes (SageAttention3 abstract, dblp author page on
// taxoreview.com: attention on the FP4 tensor cores of Blackwell GPUs; the
// two-level P~V accumulation of the SageAttention2 abstract; the online
// softmax of "Flash Attention vs Sage Attention: Kernel Comparison", section
// "How FlashAttention reduces memory traffic"):
//
//   per query row, over 128-key tiles j (causal: j <= query tile):
//     A      = sum_c (q_code s16_Q)(k_code s16_K)   (kind::mxf4nvf4, block16)
//     t      = A * (g_Q g_Kj sm_scale log2 e)        (log2 domain)
//     m_j    = max(m_{j-1}, rowmax t); alpha_j = 2^(m_{j-1} - m_j)
//     P~     = 2^(t - m_j)
//     per 16 keys: s16 = ue4m3(448 amax16), p = e2m1(2688 P~ / s16)
//     l      = alpha_j l + sum P~                    (unquantized P~)
//     part_j = sum_t (p s16)(v_code s16_V)           (block-scaled, fresh FP32)
//     O      = alpha_j O + part_j g_Vj / 2688        (FP32, registers)
//   O_out = O / l
//
// The structure follows the INT8/FP8 kernel (one CTA per 128-row query tile
// of one (b, h); TMA producer warp, single-thread MMA issuer, two exp
// warpgroups splitting the key columns, one stats/fold warpgroup), with
// these differences:
//   - every operand is packed E2M1 (64 bytes per 128-element row, stored
//     with the 64-byte swizzle), and its UE4M3 scale factors travel beside
//     it: the pre-pass writes them in the tensor-core layout, the producer
//     copies them to shared memory with a plain bulk copy, and the MMA
//     thread moves them into TMEM with tcgen05.cp (32x128b, replicated to
//     the four lane quadrants) just before the MMA that reads them;
//   - the exp warpgroups also write the P~ scale factors of their rows;
//   - S is a plain FP32 accumulator (no bias trick), single-buffered: the
//     exp warpgroups release it as soon as they hold their 64 scores, and
//     the MMA thread issues the next Q K^T ahead of the previous tile's
//     P~V, so the scores the stats warpgroup needs next never queue behind
//     a partial that is folded two tiles later;
//   - Q smoothing (SMOOTH): the exp warpgroups take the row maximum of the
//     biased scores themselves and exchange the halves (exp_loop_smooth), as
//     in the 8-bit kernel.
// TMEM columns: S 0..127, PV[0] 128..255, PV[1] 256..383, scale factors
// SFA_Q 384, SFB_K 392, SFA_P 400, SFB_V 408 (8 columns each: two 64-wide
// K blocks of 4 columns).  Every barrier wait is bounded; an expired wait
// sets the device status word and makes every role leave its loop.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "exp2_poly.cuh"
#include "sage_internal.h"
#include "sage_ptx.cuh"

// Of every 8 groups of 4 scores in the exp pass, how many take 2^t from the
// FMA-pipe polynomial (exp2_poly.cuh) instead of the SFU.
#ifndef SAGE_FP4_EXP_POLY_GROUPS
#define SAGE_FP4_EXP_POLY_GROUPS 2
#endif

namespace sage {
namespace {

constexpr int kThreads = 512;
constexpr int D = 128;  // FP4 mode supports d == 128 only
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kPScale = 448.f;       // amax16 -> UE4M3 scale of P~ (P~ <= 1)
constexpr float kPInvG = 2688.f;       // 1 / g of P~ (g = 1/2688 = 1/(448*6))
constexpr float kPG = 1.f / 2688.f;
// Register split (launch: 512 threads x 128 = 65536):
//   producer/MMA 32, two exp warpgroups keep 128, stats/fold 216.
constexpr uint32_t kRegsProducer = 32;
constexpr uint32_t kRegsStats = 216;

// TMEM column offsets.
constexpr uint32_t kColPV = 128;  // PV[b] at 128 + 128 b
constexpr uint32_t kColSfaQ = 384;
constexpr uint32_t kColSfbK = 392;
constexpr uint32_t kColSfaP = 400;
constexpr uint32_t kColSfbV = 408;

struct Layout {
  static constexpr int KS = 4;            // K ring depth
  static constexpr int VS = 4;            // V ring depth
  static constexpr int TILE = 128 * 64;   // one FP4 operand tile: 128 rows x 64 bytes
  static constexpr int SF = 1024;         // scale factors of one tile (two 512-byte blocks)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + KS * TILE;
  static constexpr int OFF_P = OFF_V + VS * TILE;
  static constexpr int OFF_SFQ = OFF_P + 2 * TILE;
  static constexpr int OFF_SFK = OFF_SFQ + SF;
  static constexpr int OFF_SFV = OFF_SFK + KS * SF;
  static constexpr int OFF_SFP = OFF_SFV + VS * SF;
  static constexpr int OFF_MISC = OFF_SFP + 2 * SF;
  static constexpr int OFF_BAR = OFF_MISC;           // barriers (<= 64 x 8 B)
  static constexpr int OFF_TMEM = OFF_MISC + 512;
  static constexpr int OFF_ABORT = OFF_MISC + 528;
  static constexpr int OFF_M = OFF_MISC + 1024;      // [2 slots][m, alpha][128]
  static constexpr int OFF_L = OFF_M + 4 * 128 * 4;  // [2 halves][128] row sums
  static constexpr int OFF_C = OFF_L + 2 * 128 * 4;  // [2 slots] dequant factor of the tile
  // Q smoothing: the score bias of key tile j (log2 units) in slot j % 4;
  // the two exp warpgroups' partial maxima of tile j in slot j % 2; alpha_j
  // for the fold in slot j % 4
  static constexpr int OFF_BIAS = OFF_C + 16;
  static constexpr int OFF_PM = OFF_BIAS + 4 * 128 * 4;
  static constexpr int OFF_A4 = OFF_PM + 2 * 2 * 128 * 4;
  static constexpr int END = OFF_A4 + 4 * 128 * 4;
  // at least 120 KB so that one CTA (holding all 512 TMEM columns) runs per SM
  static constexpr int SMEM = (END + 1024 > 120 * 1024 ? END + 1024 : 120 * 1024);
  static constexpr uint32_t SBO = 8 * 64;  // 8 rows of 64 bytes (64-byte swizzle atom)
};
static_assert(Layout::OFF_SFQ % 1024 == 0, "scale-factor blocks 1 KB aligned");

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* s_full;    // [1] MMA -> stats: S holds Q K_j^T
  uint64_t* m_full;    // [2] stats -> exp: m_j, alpha_j of tile j (slot j % 2)
  uint64_t* s_ready;   // [1] exp -> MMA: S read (both halves)
  uint64_t* p_full;    // [2] exp -> MMA: P~ tile b and its scales written
  uint64_t* p_empty;   // [2] MMA -> exp: P~ tile b read by the P~V MMA
  uint64_t* pv_full;   // [2] MMA -> stats: PV[b] holds a tile's partial
  uint64_t* pv_empty;  // [2] stats -> MMA: PV[b] read
  uint64_t* l_ready;   // [1] exp -> stats: final row sums
  uint64_t* drain;     // MMA drain on abort
  uint64_t* bias_full; // [2] stats -> exp: a tile's bias is in shared memory (Q smoothing)
  uint64_t* pm_full;   // [2] exp <-> exp: both partial maxima of a tile written (Q smoothing)
  uint64_t* a_full;    // [4] exp -> stats: alpha of a tile written (Q smoothing)
};

__device__ __forceinline__ Bars carve_bars(uint8_t* smem) {
  using L = Layout;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  Bars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = r.k_full + L::KS;
  r.v_full = r.k_empty + L::KS;
  r.v_empty = r.v_full + L::VS;
  r.s_full = r.v_empty + L::VS;
  r.m_full = r.s_full + 1;
  r.s_ready = r.m_full + 2;
  r.p_full = r.s_ready + 1;
  r.p_empty = r.p_full + 2;
  r.pv_full = r.p_empty + 2;
  r.pv_empty = r.pv_full + 2;
  r.l_ready = r.pv_empty + 2;
  r.drain = r.l_ready + 1;
  r.bias_full = r.drain + 1;
  r.pm_full = r.bias_full + 2;
  r.a_full = r.pm_full + 2;
  return r;
}

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

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Global load the compiler keeps where it is written (a plain load of a
// value needed only in the next loop iteration may be sunk to the end of
// the current one, exposing its latency at the top of the next).
__device__ __forceinline__ float ldg_early(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Descriptor of a 512-byte scale-factor block for tcgen05.cp 32x128b: 32
// rows of 16 bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(const uint8_t* p) {
  return make_sdesc(smem_u32(p), 128, 128, Swz::none);
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

// Max of 64 scores and a running value.  MASKED: columns col0 + i > lim
// are ignored (the causal diagonal tile, lim = the row; the last tile of a
// ragged sequence, lim = its last key).
template <bool MASKED>
__device__ __forceinline__ float max64(const uint32_t* s, int col0, int lim, float acc) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float x = __uint_as_float(s[k]), y = __uint_as_float(s[k + 8]);
    if (MASKED) {
      x = (col0 + k <= lim) ? x : -INFINITY;
      y = (col0 + k + 8 <= lim) ? y : -INFINITY;
    }
    a[k] = fmaxf(x, y);
  }
#pragma unroll
  for (int i = 16; i < 64; i += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float x = __uint_as_float(s[i + k]), y = __uint_as_float(s[i + 8 + k]);
      if (MASKED) {
        x = (col0 + i + k <= lim) ? x : -INFINITY;
        y = (col0 + i + 8 + k <= lim) ? y : -INFINITY;
      }
      a[k] = fmax3(a[k], x, y);
    }
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmax3(a[6], a[7], acc));
}

// Q smoothing: 32 scores of a row turned in place into biased log2-domain
// scores t = A c + bias[i] (key col0 + i); returns their maximum (masking
// as in max64).
template <bool MASKED>
__device__ __forceinline__ float biased32(uint32_t (&s)[32], float c, const float* bias, int col0,
                                          int lim) {
  const float2 c2 = make_float2(c, c);
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const float4 bv = *reinterpret_cast<const float4*>(bias + i);
    const float2 t01 = __ffma2_rn(make_float2(__uint_as_float(s[i]), __uint_as_float(s[i + 1])),
                                  c2, make_float2(bv.x, bv.y));
    const float2 t23 = __ffma2_rn(make_float2(__uint_as_float(s[i + 2]), __uint_as_float(s[i + 3])),
                                  c2, make_float2(bv.z, bv.w));
    s[i] = __float_as_uint(t01.x);
    s[i + 1] = __float_as_uint(t01.y);
    s[i + 2] = __float_as_uint(t23.x);
    s[i + 3] = __float_as_uint(t23.y);
    float v0 = t01.x, v1 = t01.y, v2 = t23.x, v3 = t23.y;
    if (MASKED) {
      v0 = (col0 + i + 0 <= lim) ? v0 : -INFINITY;
      v1 = (col0 + i + 1 <= lim) ? v1 : -INFINITY;
      v2 = (col0 + i + 2 <= lim) ? v2 : -INFINITY;
      v3 = (col0 + i + 3 <= lim) ? v3 : -INFINITY;
    }
    m0 = fmax3(m0, v0, v1);
    m1 = fmax3(m1, v2, v3);
  }
  return fmaxf(m0, m1);
}

// P~ for 32 scores of a row -> 16 bytes of e2m1 codes (key i in nibble i),
// the two UE4M3 scales of its 16-key groups (bytes 0 and 1 of *sf2), and
// the sum of the unquantized values.
//   s16 = ue4m3(448 amax16); code = e2m1(P~ * 2688 / s16) (0 when s16 = 0).
template <bool MASKED>
__device__ __forceinline__ float exp_quant32(const uint32_t (&s)[32], float c, float neg, int col0,
                                             int lim, uint32_t (&p)[4], uint32_t* sf2) {
  const float2 c2 = make_float2(c, c);
  const float2 n2 = make_float2(neg, neg);
  float x[32];
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const float2 t01 =
        __ffma2_rn(make_float2(__uint_as_float(s[i]), __uint_as_float(s[i + 1])), c2, n2);
    const float2 t23 =
        __ffma2_rn(make_float2(__uint_as_float(s[i + 2]), __uint_as_float(s[i + 3])), c2, n2);
    float f0, f1, f2, f3;
    if (((i >> 2) * SAGE_FP4_EXP_POLY_GROUPS) % 8 < SAGE_FP4_EXP_POLY_GROUPS) {
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
    x[i] = f0;
    x[i + 1] = f1;
    x[i + 2] = f2;
    x[i + 3] = f3;
  }
  uint32_t sf = 0;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const float* xg = x + 16 * g;
    float a = fmax3(fmax3(xg[0], xg[1], xg[2]), fmax3(xg[3], xg[4], xg[5]),
                    fmax3(xg[6], xg[7], xg[8]));
    a = fmax3(a, fmax3(xg[9], xg[10], xg[11]), fmax3(xg[12], xg[13], xg[14]));
    a = fmaxf(a, xg[15]);
    const uint32_t code = cvt_e4m3x2(a * kPScale, 0.f) & 0xFFu;
    const float sdec = e4m3_to_f32(code);
    const float k = sdec > 0.f ? kPInvG * rcp_approx(sdec) : 0.f;
    const float2 k2 = make_float2(k, k);
#pragma unroll
    for (int hw = 0; hw < 2; ++hw) {
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float2 v = __fmul2_rn(make_float2(xg[8 * hw + e], xg[8 * hw + e + 1]), k2);
        y[e] = v.x;
        y[e + 1] = v.y;
      }
      p[2 * g + hw] = cvt_e2m1x8(y);
    }
    sf |= code << (8 * g);
  }
  *sf2 = sf;
  const float2 t = __fadd2_rn(acc0, acc1);
  return t.x + t.y;
}

// One 32-key chunk q (0..3) of row r: e2m1 codes into the 64-byte-swizzled
// P~ tile (16-byte chunk q of row r lands at q ^ ((r >> 1) & 3)); returns
// the chunk's row sum and its two scale bytes.
template <bool MASKED>
__device__ __forceinline__ float exp_chunk(const uint32_t (&s)[32], int q, float c, float neg,
                                           int r, int lim, uint32_t prow, uint32_t* sf2) {
  uint32_t p[4];
  const float sum = exp_quant32<MASKED>(s, c, neg, 32 * q, lim, p, sf2);
  st_shared_v4(prow + (((uint32_t)q ^ (uint32_t)((r >> 1) & 3)) << 4), p[0], p[1], p[2], p[3]);
  return sum;
}

// Exp warpgroup h (0 or 1): key columns 64h .. 64h+63 of every tile.
// RAGGED (non-causal launches of a sequence whose last tile is partial): the
// last key tile masks keys n_tail .. 127.
template <bool CAUSAL, bool RAGGED>
__device__ __forceinline__ void exp_loop(const int h, const int qt, const int nkv, const int n_tail,
                                         const uint32_t tmem, const Bars& bar, uint8_t* smem,
                                         volatile int* abort_flag, uint32_t* status) {
  using L = Layout;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  const float* m_s = reinterpret_cast<const float*>(smem + L::OFF_M);
  const float* c_s = reinterpret_cast<const float*>(smem + L::OFF_C);
  float* l_s = reinterpret_cast<float*>(smem + L::OFF_L);

  float l = 0.f;
  for (int j = 0; j < nkv; ++j) {
    const int b = j & 1;
    const uint32_t ph = (j >> 1) & 1;
    // m_full(j) is published by the stats warpgroup after it waited for
    // s_full(j) and read S: it orders this warpgroup after the Q K^T too
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&bar.m_full[b], ph, abort_flag, status, kDevTimeoutEpi)))
      return;
    tc_fence_after();
    const float c = c_s[b];
    const float m_j = m_s[(2 * b) * 128 + r];
    const float alpha = m_s[(2 * b + 1) * 128 + r];
    const float neg = -m_j;
    // masked tiles: the causal diagonal and the last tile of a ragged sequence
    const bool diag = CAUSAL && (j == qt);
    const bool masked = diag || (RAGGED && j == nkv - 1);
    const int lim = diag ? r : n_tail - 1;
    const uint32_t S = tmem + lanes + 64u * h;
    uint32_t sa[32], sb[32];
    tmem_ld32(S, sa);
    tmem_ld32(S + 32, sb);
    tmem_wait_ld_regs(sa);
    reg_fence(sb);
    // S is in registers (and the stats warpgroup took its max before
    // publishing m_j): free for Q K_{j+1}^T
    tc_fence_before();
    mbar_arrive(bar.s_ready);
    // P~ tile b is free once the P~V MMA of tile j - 2 has read it
    if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.p_empty[b], ph ^ 1, abort_flag, status,
                                                     kDevTimeoutMma)))
      return;
    const uint32_t prow = smem_u32(smem + L::OFF_P + b * L::TILE + r * 64);
    uint32_t sf_lo, sf_hi;
    float sum = masked ? exp_chunk<true>(sa, 2 * h, c, neg, r, lim, prow, &sf_lo)
                       : exp_chunk<false>(sa, 2 * h, c, neg, r, lim, prow, &sf_lo);
    sum += masked ? exp_chunk<true>(sb, 2 * h + 1, c, neg, r, lim, prow, &sf_hi)
                  : exp_chunk<false>(sb, 2 * h + 1, c, neg, r, lim, prow, &sf_hi);
    // the row's four group scales of this 64-key block, in the tensor-core
    // layout: byte 16 (r % 32) + 4 (r / 32) + s of the block's 512 bytes
    st_shared_u32(smem_u32(smem + L::OFF_SFP + b * L::SF + h * 512 + 16 * (r & 31) + 4 * (r >> 5)),
                  sf_lo | (sf_hi << 16));
    l = fmaf(alpha, l, sum);
    fence_proxy_async_smem();  // P~ stores visible to the tensor core
    mbar_arrive(&bar.p_full[b]);
  }
  l_s[h * 128 + r] = l;
  mbar_arrive(bar.l_ready);
}

// Q smoothing: the exp warpgroups take the row maximum themselves, as in the
// 8-bit kernel.  Each turns its 64 scores of tile j into biased log2-domain
// scores t = A c + bias in place, takes their maximum, and exchanges it with
// the other warpgroup through shared memory (pm_full); both form the same
// m_j and alpha_j, warpgroup 0 publishes alpha_j for the fold (a_full), and
// P~ = 2^(t - m_j).  The stats warpgroup only stages the biases and folds.
// Slots: the partial maxima of tile j in j % 2 (a warpgroup writes tile
// j + 2's only after passing tile j + 1's exchange, which the other enters
// only after reading tile j's); alpha in j % 4 (written for tile j + 4 only
// after the bias of tile j + 4 is staged, which the stats warpgroup does
// only after reading alpha_j).
template <bool CAUSAL, bool RAGGED>
__device__ __forceinline__ void exp_loop_smooth(const int h, const int qt, const int nkv,
                                                const int n_tail, const int bh, const int H,
                                                const int G, const int ntiles,
                                                const float* __restrict__ q_scales,
                                                const float* __restrict__ k_scales,
                                                const float scale_log2, const uint32_t tmem,
                                                const Bars& bar, uint8_t* smem,
                                                volatile int* abort_flag, uint32_t* status) {
  using L = Layout;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  const float* bias_s = reinterpret_cast<const float*>(smem + L::OFF_BIAS);
  float* pm_s = reinterpret_cast<float*>(smem + L::OFF_PM);
  float* a_s = reinterpret_cast<float*>(smem + L::OFF_A4);
  float* l_s = reinterpret_cast<float*>(smem + L::OFF_L);
  // the tile scales g_Q (this query tile) and g_K (one per key tile)
  const float qs = __ldg(q_scales + (int64_t)bh * ntiles + qt);
  const float* ksp = k_scales + (int64_t)kv_head(bh, H, G) * ntiles;

  float l = 0.f, m = -INFINITY;
  float ks = ldg_early(ksp);
  for (int j = 0; j < nkv; ++j) {
    const int b = j & 1;
    const uint32_t ph = (j >> 1) & 1;
    const float c = qs * ks * scale_log2;
    const float ks_nxt = j + 1 < nkv ? ldg_early(ksp + j + 1) : 0.f;
    if (!__all_sync(0xffffffffu,
                    mbar_wait(bar.s_full, j & 1, abort_flag, status, kDevTimeoutMma)))
      return;
    tc_fence_after();
    const bool diag = CAUSAL && (j == qt);
    const bool masked = diag || (RAGGED && j == nkv - 1);
    const int lim = diag ? r : n_tail - 1;
    const uint32_t S = tmem + lanes + 64u * h;
    uint32_t sa[32], sb[32];
    tmem_ld32(S, sa);
    tmem_ld32(S + 32, sb);
    tmem_wait_ld_regs(sa);
    reg_fence(sb);
    // S is in registers: free for Q K_{j+1}^T
    tc_fence_before();
    mbar_arrive(bar.s_ready);
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&bar.bias_full[b], ph, abort_flag, status, kDevTimeoutSoftmax)))
      return;
    const float* bias = bias_s + (j & 3) * 128 + 64 * h;
    const float p = masked ? fmaxf(biased32<true>(sa, c, bias, 64 * h, lim),
                                   biased32<true>(sb, c, bias + 32, 64 * h + 32, lim))
                           : fmaxf(biased32<false>(sa, c, bias, 64 * h, lim),
                                   biased32<false>(sb, c, bias + 32, 64 * h + 32, lim));
    pm_s[(2 * b + h) * 128 + r] = p;
    mbar_arrive(&bar.pm_full[b]);
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&bar.pm_full[b], ph, abort_flag, status, kDevTimeoutSoftmax)))
      return;
    const float m_j = fmax3(m, p, pm_s[(2 * b + (h ^ 1)) * 128 + r]);
    const float alpha = ex2(m - m_j);
    m = m_j;
    if (h == 0) {
      a_s[(j & 3) * 128 + r] = alpha;
      mbar_arrive(&bar.a_full[j & 3]);
    }
    // P~ tile b is free once the P~V MMA of tile j - 2 has read it
    if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.p_empty[b], ph ^ 1, abort_flag, status,
                                                     kDevTimeoutMma)))
      return;
    const uint32_t prow = smem_u32(smem + L::OFF_P + b * L::TILE + r * 64);
    uint32_t sf_lo, sf_hi;
    // the biased scores are plain FP32 now: t - m_j by one FMA
    float sum = masked ? exp_chunk<true>(sa, 2 * h, 1.f, -m_j, r, lim, prow, &sf_lo)
                       : exp_chunk<false>(sa, 2 * h, 1.f, -m_j, r, lim, prow, &sf_lo);
    sum += masked ? exp_chunk<true>(sb, 2 * h + 1, 1.f, -m_j, r, lim, prow, &sf_hi)
                  : exp_chunk<false>(sb, 2 * h + 1, 1.f, -m_j, r, lim, prow, &sf_hi);
    st_shared_u32(smem_u32(smem + L::OFF_SFP + b * L::SF + h * 512 + 16 * (r & 31) + 4 * (r >> 5)),
                  sf_lo | (sf_hi << 16));
    l = fmaf(alpha, l, sum);
    fence_proxy_async_smem();  // P~ stores visible to the tensor core
    mbar_arrive(&bar.p_full[b]);
    ks = ks_nxt;
  }
  l_s[h * 128 + r] = l;
  mbar_arrive(bar.l_ready);
}

// Stats warpgroup: row max / running max per key tile, level-2 fold (one
// tile behind), epilogue.
template <bool CAUSAL, typename OutT, bool RAGGED, bool SMOOTH>
__device__ __forceinline__ void stats_loop(const int qt, const int nkv, const int n_tail,
                                           const int bh,
                                           const int H, const int G, const int N,
                                           const int ntiles, const uint32_t tmem, const Bars& bar,
                                           uint8_t* smem, volatile int* abort_flag,
                                           uint32_t* status, const float* __restrict__ q_scales,
                                           const float* __restrict__ k_scales,
                                           const float* __restrict__ v_scales,
                                           const float* __restrict__ ds,
                                           OutT* __restrict__ out, const float scale_log2) {
  using L = Layout;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  float* m_s = reinterpret_cast<float*>(smem + L::OFF_M);
  const float* l_s = reinterpret_cast<const float*>(smem + L::OFF_L);
  const float qs = __ldg(q_scales + (int64_t)bh * ntiles + qt);
  const float* ksp = k_scales + (int64_t)kv_head(bh, H, G) * ntiles;
  const float* vgp = v_scales + (int64_t)kv_head(bh, H, G) * ntiles;

  float2 o2[D / 2];
#pragma unroll
  for (int c = 0; c < D / 2; ++c) o2[c] = make_float2(0.f, 0.f);
  float m = -INFINITY;
  // O = alpha_i O + part_i * g_V,i / 2688
  auto fold = [&](int i, float alpha) -> bool {
    const int pb = i & 1;
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&bar.pv_full[pb], (i >> 1) & 1, abort_flag, status, kDevTimeoutMma)))
      return false;
    tc_fence_after();
    const uint32_t PV = tmem + lanes + kColPV + 128u * (uint32_t)pb;
    const float2 a2 = make_float2(alpha, alpha);
    const float cv = ldg_early(vgp + i) * kPG;
    const float2 cv2 = make_float2(cv, cv);
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t pv[32];
      tmem_ld32(PV + 32 * cc, pv);
      tmem_wait_ld_regs(pv);
#pragma unroll
      for (int k = 0; k < 16; ++k)
        o2[cc * 16 + k] = __ffma2_rn(
            a2, o2[cc * 16 + k],
            __fmul2_rn(make_float2(__uint_as_float(pv[2 * k]), __uint_as_float(pv[2 * k + 1])),
                       cv2));
    }
    tc_fence_before();
    mbar_arrive(&bar.pv_empty[pb]);
    return true;
  };

  float alpha_hist[2] = {0.f, 0.f};
  float* c_s = reinterpret_cast<float*>(smem + L::OFF_C);
  float ks_cur = ldg_early(ksp);
  // Q smoothing: this query block's score bias, exchanged through slot j % 4
  // of a shared buffer one tile ahead (as in the 8-bit kernel): thread r
  // writes key 128 j + r after reading alpha_{j-1} and arrives on
  // bias_full[j % 2]; a slot is rewritten for tile j + 4 after alpha_{j+3}
  // is published, which both exp warpgroups do only past their reads of
  // tile j's bias.
  const float* dsr = SMOOTH ? ds + ((int64_t)bh * ntiles + qt) * (int64_t)(ntiles * 128) : nullptr;
  float* bias_s = reinterpret_cast<float*>(smem + L::OFF_BIAS);
  float d_nxt = 0.f;
  if (SMOOTH) {
    bias_s[r] = ldg_early(dsr + r) * scale_log2;
    mbar_arrive(&bar.bias_full[0]);
    if (nkv > 1) d_nxt = ldg_early(dsr + 128 + r);
  }
  for (int j = 0; SMOOTH && j < nkv; ++j) {
    // Q smoothing: the exp warpgroups take the maximum; this warpgroup
    // stages the next tile's bias and folds with the published alpha_j
    const int b = j & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.a_full[j & 3], (j >> 2) & 1, abort_flag, status,
                                           kDevTimeoutSoftmax)))
      return;
    const float alpha = reinterpret_cast<const float*>(smem + L::OFF_A4)[(j & 3) * 128 + r];
    if (j + 1 < nkv) {
      bias_s[((j + 1) & 3) * 128 + r] = d_nxt * scale_log2;
      mbar_arrive(&bar.bias_full[(j + 1) & 1]);
      if (j + 2 < nkv) d_nxt = ldg_early(dsr + 128 * (j + 2) + r);
    }
    if (j > 1 && !fold(j - 2, alpha_hist[b])) return;
    alpha_hist[b] = alpha;
  }
  for (int j = 0; !SMOOTH && j < nkv; ++j) {
    const int b = j & 1;
    const float c = qs * ks_cur * scale_log2;
    const float ks_nxt = j + 1 < nkv ? ldg_early(ksp + j + 1) : 0.f;
    if (!__all_sync(0xffffffffu,
                    mbar_wait(bar.s_full, j & 1, abort_flag, status, kDevTimeoutMma)))
      return;
    tc_fence_after();
    const bool diag = CAUSAL && (j == qt);
    const bool masked = diag || (RAGGED && j == nkv - 1);
    const int lim = diag ? r : n_tail - 1;
    const uint32_t S = tmem + lanes;
    float mx = -INFINITY;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t s[2][32];
      tmem_ld32(S + 64 * hh, s[0]);
      tmem_ld32(S + 64 * hh + 32, s[1]);
      tmem_wait_ld_regs(s[0]);
      reg_fence(s[1]);
      mx = masked ? max64<true>(&s[0][0], 64 * hh, lim, mx)
                  : max64<false>(&s[0][0], 64 * hh, lim, mx);
    }
    const float m_j = fmaxf(m, mx * c);
    const float alpha = ex2(m - m_j);
    m = m_j;
    m_s[(2 * b) * 128 + r] = m_j;
    m_s[(2 * b + 1) * 128 + r] = alpha;
    if (r == 0) c_s[b] = c;
    tc_fence_before();
    mbar_arrive(&bar.m_full[b]);
    // the fold runs two tiles behind the max
    if (j > 1 && !fold(j - 2, alpha_hist[b])) return;
    alpha_hist[b] = alpha;
    ks_cur = ks_nxt;
  }
  for (int i = nkv > 2 ? nkv - 2 : 0; i < nkv; ++i)
    if (!fold(i, alpha_hist[i & 1])) return;
  if (!__all_sync(0xffffffffu,
                  mbar_wait(bar.l_ready, 0, abort_flag, status, kDevTimeoutSoftmax)))
    return;
  const float inv_l = 1.f / (l_s[r] + l_s[128 + r]);
  // rows past the end of a ragged sequence are padding: not stored
  if (qt * 128 + r >= N) return;
  OutT* dst = out + ((int64_t)bh * N + (int64_t)qt * 128 + r) * D;
#pragma unroll
  for (int cv = 0; cv < D; cv += 8) {
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v = o2[cv / 2 + e];
      w4[e] = pack2<OutT>(v.x * inv_l, v.y * inv_l);
    }
    *reinterpret_cast<uint4*>(dst + cv) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

template <bool CAUSAL, typename OutT, bool RAGGED, bool SMOOTH>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fp4_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scales,
                    const float* __restrict__ k_scales, const float* __restrict__ v_scales,
                    const uint8_t* __restrict__ q_sf, const uint8_t* __restrict__ k_sf,
                    const uint8_t* __restrict__ v_sf, const float* __restrict__ ds,
                    OutT* __restrict__ out, int N, int H, int G, float scale_log2,
                    int head_major, uint32_t* status) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // N tokens in ntiles 128-token tiles (codes padded to Np = 128 ntiles);
  // the last tile holds n_tail of them
  const int ntiles = (N + 127) / 128;
  const int Np = ntiles * 128;
  const int n_tail = N - (ntiles - 1) * 128;
  // grid order: see head_major_grid
  const int bh = head_major ? (int)blockIdx.x : (int)blockIdx.y;
  const int tile_rank = head_major ? (int)blockIdx.y : (int)blockIdx.x;
  // K/V head of this query head (grouped-query attention: G query heads per
  // K/V head; G = 1 is plain multi-head attention)
  const int bhk = kv_head(bh, H, G);
  const int qt = CAUSAL ? (ntiles - 1 - tile_rank) : tile_rank;  // heavy first
  const int nkv = CAUSAL ? qt + 1 : ntiles;

  Bars bar = carve_bars(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);

  if (threadIdx.x == 0) {
    mbar_init(bar.q_full, 1);
    for (int i = 0; i < L::KS; ++i) {
      mbar_init(&bar.k_full[i], 1);
      mbar_init(&bar.k_empty[i], 1);
    }
    for (int i = 0; i < L::VS; ++i) {
      mbar_init(&bar.v_full[i], 1);
      mbar_init(&bar.v_empty[i], 1);
    }
    mbar_init(bar.s_full, 1);
    mbar_init(bar.s_ready, 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.m_full[i], 128);
      mbar_init(&bar.p_full[i], 256);
      mbar_init(&bar.p_empty[i], 1);
      mbar_init(&bar.pv_full[i], 1);
      mbar_init(&bar.pv_empty[i], 128);
    }
    mbar_init(bar.l_ready, 256);
    mbar_init(bar.drain, 1);
    mbar_init(&bar.bias_full[0], 128);
    mbar_init(&bar.bias_full[1], 128);
    mbar_init(&bar.pm_full[0], 256);
    mbar_init(&bar.pm_full[1], 256);
    for (int i = 0; i < 4; ++i) mbar_init(&bar.a_full[i], 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  uint8_t* sSFQ = smem + L::OFF_SFQ;
  uint8_t* sSFK = smem + L::OFF_SFK;
  uint8_t* sSFV = smem + L::OFF_SFV;
  uint8_t* sSFP = smem + L::OFF_SFP;

  const int wg = warp >> 2;
  if (wg == 0) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (elect_one()) {
        const int64_t tile0 = (int64_t)bhk * ntiles;
        mbar_arrive_expect_tx(bar.q_full, L::TILE + L::SF);
        tma_load_2d(sQ, &tm_q, 0, bh * Np + qt * 128, bar.q_full);
        bulk_load(sSFQ, q_sf + ((int64_t)bh * ntiles + qt) * L::SF, L::SF, bar.q_full);
        for (int j = 0; j < nkv; ++j) {
          const int sk = j % L::KS;
          if (!mbar_wait<true>(&bar.k_empty[sk], ((j / L::KS) & 1) ^ 1, abort_flag, status,
                               kDevTimeoutMma))
            break;
          mbar_arrive_expect_tx(&bar.k_full[sk], L::TILE + L::SF);
          tma_load_2d(sK + sk * L::TILE, &tm_k, 0, bhk * Np + j * 128, &bar.k_full[sk]);
          bulk_load(sSFK + sk * L::SF, k_sf + (tile0 + j) * L::SF, L::SF, &bar.k_full[sk]);
          const int sv = j % L::VS;
          if (!mbar_wait<true>(&bar.v_empty[sv], ((j / L::VS) & 1) ^ 1, abort_flag, status,
                               kDevTimeoutMma))
            break;
          mbar_arrive_expect_tx(&bar.v_full[sv], L::TILE + L::SF);
          tma_load_2d(sV + sv * L::TILE, &tm_v, j * 64, bhk * D, &bar.v_full[sv]);
          bulk_load(sSFV + sv * L::SF, v_sf + (tile0 + j) * L::SF, L::SF, &bar.v_full[sv]);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------------------------------------------- tcgen05 issuer
      if (elect_one()) {
        constexpr uint32_t idesc = make_idesc_nvf4(128, 128);  // Q K^T and P~V: M = N = 128
        const uint64_t qdesc = make_sdesc(smem_u32(sQ), L::SBO, 16, Swz::k64);
        bool ok = mbar_wait(bar.q_full, 0, abort_flag, status, kDevTimeoutTma);
        if (ok) {
          tc_fence_after();
          tmem_cp_32x128b_x4(tmem + kColSfaQ, sf_desc(sSFQ));
          tmem_cp_32x128b_x4(tmem + kColSfaQ + 4, sf_desc(sSFQ + 512));
        }
        // S = Q K_j^T, two K blocks of 64 channels (S free: for j >= 1 the
        // caller waited for s_ready of tile j - 1)
        auto qk = [&](int j) -> bool {
          const int sk = j % L::KS;
          if (!mbar_wait(&bar.k_full[sk], (j / L::KS) & 1, abort_flag, status, kDevTimeoutTma))
            return false;
          tc_fence_after();
          tmem_cp_32x128b_x4(tmem + kColSfbK, sf_desc(sSFK + sk * L::SF));
          tmem_cp_32x128b_x4(tmem + kColSfbK + 4, sf_desc(sSFK + sk * L::SF + 512));
          const uint64_t kdesc = make_sdesc(smem_u32(sK + sk * L::TILE), L::SBO, 16, Swz::k64);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_nvf4_ss(tmem, qdesc + 2 * kk, kdesc + 2 * kk, idesc, tmem + kColSfaQ + 4 * kk,
                        tmem + kColSfbK + 4 * kk, kk > 0);
          mma_commit(bar.s_full);
          mma_commit(&bar.k_empty[sk]);
          return true;
        };
        // P~_i V_i into PV[i % 2] (level 1)
        auto pv = [&](int i) -> bool {
          const int b = i & 1;
          const int sv = i % L::VS;
          if (!mbar_wait(&bar.p_full[b], (i >> 1) & 1, abort_flag, status, kDevTimeoutSoftmax) ||
              !mbar_wait(&bar.v_full[sv], (i / L::VS) & 1, abort_flag, status, kDevTimeoutTma) ||
              !mbar_wait(&bar.pv_empty[b], ((i >> 1) & 1) ^ 1, abort_flag, status,
                         kDevTimeoutEpi))
            return false;
          tc_fence_after();
          tmem_cp_32x128b_x4(tmem + kColSfaP, sf_desc(sSFP + b * L::SF));
          tmem_cp_32x128b_x4(tmem + kColSfaP + 4, sf_desc(sSFP + b * L::SF + 512));
          tmem_cp_32x128b_x4(tmem + kColSfbV, sf_desc(sSFV + sv * L::SF));
          tmem_cp_32x128b_x4(tmem + kColSfbV + 4, sf_desc(sSFV + sv * L::SF + 512));
          const uint64_t pdesc = make_sdesc(smem_u32(sP + b * L::TILE), L::SBO, 16, Swz::k64);
          const uint64_t vdesc = make_sdesc(smem_u32(sV + sv * L::TILE), L::SBO, 16, Swz::k64);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_nvf4_ss(tmem + kColPV + 128u * (uint32_t)b, pdesc + 2 * kk, vdesc + 2 * kk, idesc,
                        tmem + kColSfaP + 4 * kk, tmem + kColSfbV + 4 * kk, kk > 0);
          mma_commit(&bar.pv_full[b]);
          mma_commit(&bar.p_empty[b]);
          mma_commit(&bar.v_empty[sv]);
          return true;
        };
        if (ok) ok = qk(0);
        // The exp warpgroups release S early in their pass over tile i: the
        // Q K^T of tile i + 1 goes first (the scores the stats warpgroup
        // needs next), the P~V of tile i - 1 (folded two tiles behind)
        // second, so the scores never queue behind it.
        for (int i = 0; ok && i < nkv; ++i) {
          if (i + 1 < nkv) {
            if (!mbar_wait(bar.s_ready, i & 1, abort_flag, status, kDevTimeoutSoftmax)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (!qk(i + 1)) {
              ok = false;
              break;
            }
          }
          if (i >= 1 && !pv(i - 1)) {
            ok = false;
            break;
          }
        }
        if (ok && nkv > 0) ok = pv(nkv - 1);
        if (!ok) {
          // let every MMA already issued finish before TMEM is released
          mma_commit(bar.drain);
          volatile int no_abort = 0;
          mbar_wait(bar.drain, 0, &no_abort, status, kDevTimeoutMma);
        }
      }
      __syncwarp();
    }
  } else if (wg < 3 && SMOOTH) {
    exp_loop_smooth<CAUSAL, RAGGED>(wg - 1, qt, nkv, n_tail, bh, H, G, ntiles, q_scales, k_scales,
                                    scale_log2, tmem, bar, smem, abort_flag, status);
  } else if (wg < 3) {
    // the exp warpgroups keep the 128 registers they were launched with
    exp_loop<CAUSAL, RAGGED>(wg - 1, qt, nkv, n_tail, tmem, bar, smem, abort_flag, status);
  } else {
    setmaxnreg_inc<kRegsStats>();
    stats_loop<CAUSAL, OutT, RAGGED, SMOOTH>(qt, nkv, n_tail, bh, H, G, N, ntiles, tmem, bar, smem,
                                             abort_flag, status, q_scales, k_scales, v_scales, ds,
                                             out, scale_log2);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool CAUSAL, typename OutT, bool RAGGED = false>
cudaError_t launch_typed(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, cudaStream_t st) {
  using L = Layout;
  auto kern = a.ds ? attn_fp4_kernel<CAUSAL, OutT, RAGGED, true>
                   : attn_fp4_kernel<CAUSAL, OutT, RAGGED, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)((a.N + 127) / 128);
  const int hm = head_major_grid(a);
  const dim3 grid = hm ? dim3((unsigned)(a.B * a.H), (unsigned)ntiles)
                       : dim3((unsigned)ntiles, (unsigned)(a.B * a.H));
  kern<<<grid, kThreads, L::SMEM, st>>>(
      tq, tk, tv, a.q_scales, a.k_scales, a.v_scales, static_cast<const uint8_t*>(a.q_sf),
      static_cast<const uint8_t*>(a.k_sf), static_cast<const uint8_t*>(a.v_sf), a.ds,
      reinterpret_cast<OutT*>(a.o), (int)a.N, (int)a.H, (int)(a.H / a.Hkv), a.sm_scale * kLog2e,
      hm, a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fp4(const AttnArgs& a, cudaStream_t st, const char** detail) {
  if (a.d != D) {
    if (detail) *detail = "FP4 attention supports d == 128 only";
    return cudaErrorInvalidValue;
  }
  const uint64_t BH = (uint64_t)(a.B * a.H);
  const uint64_t BHK = (uint64_t)(a.B * a.Hkv);
  const uint64_t N = (uint64_t)((a.N + 127) / 128 * 128);  // codes padded to whole tiles
  CUtensorMap tq, tk, tv;
  // Q, K: [B*H*N rows, 64 bytes]; V^T: [B*H*128 rows (channels), N/2 bytes]
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q_codes, 64, BH * N, 64, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_64B, detail) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.k_codes, 64, BHK * N, 64, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_64B, detail) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.v_codes, N / 2, BHK * D, N / 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_64B, detail))
    return cudaErrorInvalidValue;
  if (a.causal)
    return a.dtype == 1 ? launch_typed<true, __nv_bfloat16>(a, tq, tk, tv, st)
                        : launch_typed<true, __half>(a, tq, tk, tv, st);
  // causal launches mask the partial last tile through the diagonal already
  if (a.N % 128 != 0)
    return a.dtype == 1 ? launch_typed<false, __nv_bfloat16, true>(a, tq, tk, tv, st)
                        : launch_typed<false, __half, true>(a, tq, tk, tv, st);
  return a.dtype == 1 ? launch_typed<false, __nv_bfloat16>(a, tq, tk, tv, st)
                      : launch_typed<false, __half>(a, tq, tk, tv, st);
}

}  // namespace sage
