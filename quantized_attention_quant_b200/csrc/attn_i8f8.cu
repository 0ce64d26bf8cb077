// attn_i8f8.cu -- fused quantized attention forward, INT8 (or FP8) Q K^T +
// FP8 P~V, for sm_100a (tcgen05 tensor cores, TMEM accumulators, TMA).
//
// What it computes (SageAttention abstract: INT8 Q K^T; SageAttention2
// abstract: FP8 P~ and V with two-level accumulation of P~V; the online
// softmax of "Flash Attention vs Sage Attention: Kernel Comparison",
// section "How FlashAttention reduces memory traffic"):
//
//   per query row, over 128-key tiles j (causal: j <= query tile):
//     A      = q_codes . k_codes_j^T                 (tcgen05 kind::i8, exact;
//                                                     FP8 Q/K: kind::f8f6f4, FP32)
//     t      = A * (s_Q s_K sm_scale log2 e)         (log2 domain; s_Q of the
//                                                     query token, s_K of the
//                                                     key's 32-key block)
//     m_j    = max(m_{j-1}, rowmax t); alpha_j = 2^(m_{j-1} - m_j)
//     p      = e4m3(448 * 2^(t - m_j))               (448 P~, quantized)
//     l      = alpha_j l + sum 448 P~                (unquantized P~)
//     part_j = p . v_codes_j                         (kind::f8f6f4, fresh FP32)
//     O      = alpha_j O + part_j                    (FP32, registers)
//   O_out = O * s_V[c] / l
//
// One CTA owns one 128-row query tile of one (b, h).  The exponentials are
// the throughput limit (the tensor core finishes a 128x128 tile in far fewer
// cycles than the SFU needs for its 16K exponentials; one warp per SM
// sub-partition keeps the SFU only about half busy, two about 80 %), so two
// warpgroups share every tile.  Warp roles (512 threads):
//   warpgroup 0: warp 0 TMA producer (Q once, K_j and V_j^T rings),
//                warp 1 TMEM allocator and single-thread tcgen05 issuer
//   warpgroups 1, 2 ("exp"): key columns 0..63 / 64..127 of every tile.
//                Thread = query row = TMEM lane.  448 P~ as e4m3 codes into
//                a TMEM tile (the A operand of the P~V MMA, read from TMEM)
//                and the row sum.
//   warpgroup 3 ("stats"): per key tile the row max, the running max m_j and
//                alpha_j (published for both exp warpgroups), then the level-2
//                fold of the tile's FP32 partial into the running FP32
//                accumulator (registers); finally normalise and store O.
// TMEM columns: d = 128: S 0..127 (one buffer), PV[0] 128.., PV[1] 256..;
// d = 64: S[0] 0..127, S[1] 128..255, PV[0] 256.., PV[1] 320..; both:
// P~[0] 384..415, P~[1] 416..447 (four e4m3 codes per column, keys
// 64h .. 64h+63 in columns 16h .. 16h+15).  Key tile j uses S[j % SB],
// PV[j % 2] (folded two tiles behind) and P~[j % 2].  The exp warpgroups
// read their S columns first and release S at once, so the next Q K^T runs
// while they work on the exponentials; the MMA thread issues it ahead of
// the P~V of the previous tile.  Each Q K^T overwrites S: the INT8 scores
// are INT32, which the exp warpgroups turn into floats with one integer add
// each (score() in attn_i8f8_common.cuh; TMEM stores are about a third as
// fast as loads, so writing a float bias back into S for the next MMA to
// accumulate onto cost more); the stats warpgroup takes the row maximum on
// the integers.  The FP8 Q/K variant (QF8; the kernel-comparison blog's
// "INT8 or FP8" queries and keys) runs the same pipeline with FP32 scores.
// Dequantization: the Q scale is the row's (one per token), the K scale the
// 32-key chunk's (one per 32 keys), so every thread applies one factor per
// chunk of 32 scores it holds.
// Q smoothing (SMOOTH; SageAttention2 abstract, "smooth Q"): every score
// gains its key's bias qbar . k' of the query block, so the row maximum is
// no longer a scaled integer maximum; the exp warpgroups then take it on the
// biased FP32 scores themselves and exchange the halves, and the stats
// warpgroup only stages the biases and folds (exp_loop_smooth).
// Every barrier wait is bounded; an expired wait sets the device status
// word and makes every role leave its loop.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_i8f8_common.cuh"

namespace sage {

// Optional timeline trace (builds with -DSAGE_TRACE only): %clock64 of
// selected events of one steady-state CTA, read back by sage_trace_read.
#ifdef SAGE_TRACE
// Timestamps go to shared memory while the kernel runs (a global store would
// make the next release-arrive wait for it) and are copied out at the end.
__device__ long long g_sage_trace[16][512];
__shared__ long long s_sage_trace[16][64];
#define SAGE_TRACED_CTA (blockIdx.x == 7 && blockIdx.y == 1)
#define SAGE_TR(ev, j)                                                                  \
  do {                                                                                  \
    if (SAGE_TRACED_CTA && (j) < 64) {                                                  \
      long long t_;                                                                     \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_));                                \
      s_sage_trace[ev][j] = t_;                                                         \
    }                                                                                   \
  } while (0)
#else
#define SAGE_TR(ev, j) \
  do {                 \
  } while (0)
#endif

namespace {

template <int D>
struct Layout {
  static constexpr int KS = D == 128 ? 4 : 6;  // K ring depth
  static constexpr int VS = D == 128 ? 4 : 6;  // V ring depth
  static constexpr int Q_BYTES = 128 * D;
  static constexpr int K_BYTES = 128 * D;
  static constexpr int V_BYTES = D * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * K_BYTES;
  static constexpr int OFF_MISC = OFF_V + VS * V_BYTES;
  static constexpr int OFF_BAR = OFF_MISC;           // barriers (<= 64 x 8 B)
  static constexpr int OFF_TMEM = OFF_MISC + 512;
  static constexpr int OFF_ABORT = OFF_MISC + 528;
  static constexpr int OFF_M = OFF_MISC + 1024;      // [2 slots][m, alpha][128]
  static constexpr int OFF_L = OFF_M + 4 * 128 * 4;  // [2 halves][128] row sums
  static constexpr int OFF_C = OFF_L + 2 * 128 * 4;  // [2 slots][4] s_K sm_scale log2 e per 32 keys
  static constexpr int OFF_VS = OFF_C + 128;         // s_V[D] of the head (bulk-copied with Q)
  // Q smoothing: the score bias of key tile j (log2 units) in slot j % 4;
  // the two exp warpgroups' partial maxima of tile j in slot j % 2; alpha_j
  // for the fold in slot j % 4
  static constexpr int OFF_BIAS = OFF_VS + 4 * D;
  static constexpr int OFF_PM = OFF_BIAS + 4 * 128 * 4;
  static constexpr int OFF_A4 = OFF_PM + 2 * 2 * 128 * 4;
  static constexpr int END = OFF_A4 + 4 * 128 * 4;
  // at least 120 KB so that one CTA (holding all 512 TMEM columns) runs per SM
  static constexpr int SMEM = (END + 1024 > 120 * 1024 ? END + 1024 : 120 * 1024);
  static constexpr uint32_t QK_SBO = 8 * D;  // 8 rows of D bytes
  static constexpr int SB = D == 128 ? 1 : 2;    // S buffers
  static constexpr int PVB = 2;                  // level-1 partial buffers
  static constexpr uint32_t COL_PV = 128 * SB;   // PV[b] at COL_PV + D b
  static constexpr uint32_t COL_P = 384;         // P~[b] at COL_P + 32 b
  static constexpr Swz QK_SWZ = D == 128 ? Swz::k128 : Swz::k64;
};

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* s_init;    // [1] exp -> MMA: the exp warpgroups are running
  uint64_t* s_full;    // [SB] MMA -> stats: S[b] holds Q K_j^T
  uint64_t* s_ready;   // [SB] exp -> MMA: S[b] read
  uint64_t* m_full;    // [2] stats -> exp: m_j, alpha_j of tile j (slot j % 2)
  uint64_t* p_full;    // [2] exp -> MMA: P~[b] written
  uint64_t* p_empty;   // [2] MMA -> exp: P~[b] read by the P~V MMA
  uint64_t* pv_full;   // [PVB] MMA -> stats: PV[b] holds a tile's partial
  uint64_t* pv_empty;  // [PVB] stats -> MMA: PV[b] read
  uint64_t* l_ready;   // [1] exp -> stats: final row sums
  uint64_t* drain;     // MMA drain on abort
  uint64_t* bias_full; // [2] stats -> stats, exp: a tile's bias is in shared memory (Q smoothing)
  uint64_t* pm_full;   // [2] exp <-> exp: both partial maxima of a tile written (Q smoothing)
  uint64_t* a_full;    // [4] exp -> stats: alpha of a tile written (Q smoothing)
};

template <int D>
__device__ __forceinline__ Bars carve_bars(uint8_t* smem) {
  using L = Layout<D>;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  Bars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = r.k_full + L::KS;
  r.v_full = r.k_empty + L::KS;
  r.v_empty = r.v_full + L::VS;
  r.s_init = r.v_empty + L::VS;
  r.s_full = r.s_init + 1;
  r.s_ready = r.s_full + L::SB;
  r.m_full = r.s_ready + L::SB;
  r.p_full = r.m_full + 2;
  r.p_empty = r.p_full + 2;
  r.pv_full = r.p_empty + 2;
  r.pv_empty = r.pv_full + L::PVB;
  r.l_ready = r.pv_empty + L::PVB;
  r.drain = r.l_ready + 1;
  r.bias_full = r.drain + 1;
  r.pm_full = r.bias_full + 2;
  r.a_full = r.pm_full + 2;
  return r;
}

// Exp warpgroup h (0 or 1): key columns 64h .. 64h+63 of every tile.
// RAGGED (non-causal launches of a sequence whose last tile is partial): the
// last key tile masks keys n_tail .. 127.
template <int D, bool CAUSAL, bool QF8, bool RAGGED>
__device__ __forceinline__ void exp_loop(const int h, const int qt, const int nkv, const int n_tail,
                                         const int bh, const int ntiles,
                                         const float* __restrict__ q_scales, const uint32_t tmem,
                                         const Bars& bar, uint8_t* smem,
                                         volatile int* abort_flag, uint32_t* status) {
  using L = Layout<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  const float* m_s = reinterpret_cast<const float*>(smem + L::OFF_M);
  const float* c_s = reinterpret_cast<const float*>(smem + L::OFF_C);
  float* l_s = reinterpret_cast<float*>(smem + L::OFF_L);
  // this row's Q scale (one per token); padding rows of a ragged tile read
  // the scale 0 the pre-pass wrote there
  const float qs = __ldg(q_scales + ((int64_t)bh * ntiles + qt) * 128 + r);

  // (every Q K^T overwrites S: nothing to prepare in TMEM)
  tc_fence_before();
  mbar_arrive(bar.s_init);

  float l = 0.f;
  for (int j = 0; j < nkv; ++j) {
    const int b = j & 1;
    const uint32_t ph = (j >> 1) & 1;
    if (r == 0 && h == 0) SAGE_TR(12, j);
    // m_full(j) is published by the stats warpgroup after it waited for
    // s_full(j) and read S[b]: it orders this warpgroup after the Q K^T too
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&bar.m_full[b], ph, abort_flag, status, kDevTimeoutEpi)))
      return;
    tc_fence_after();
    if (r == 0) SAGE_TR(h, j);
    // dequant factors of this warpgroup's two 32-key chunks (the stats
    // warpgroup forms its maximum from the same products)
    const float ca = qs * c_s[4 * b + 2 * h], cb = qs * c_s[4 * b + 2 * h + 1];
    const float m_j = m_s[(2 * b) * 128 + r];
    const float alpha = m_s[(2 * b + 1) * 128 + r];
    const float neg = kLog2_448 - m_j;  // yields 448 P~ directly
    // masked tiles: the causal diagonal (keys up to the row) and the last
    // tile of a ragged sequence (keys up to n_tail - 1)
    const bool diag = CAUSAL && (j == qt);
    const bool masked = diag || (RAGGED && j == nkv - 1);
    const int lim = diag ? r : n_tail - 1;
    const int sbuf = j % L::SB;
    const uint32_t S = tmem + lanes + 128u * sbuf + 64u * h;
    const uint32_t P = tmem + lanes + L::COL_P + 32u * b + 16u * h;
    uint32_t sa[32], sb[32];
    tmem_ld32(S, sa);
    tmem_ld32(S + 32, sb);
    tmem_wait_ld_regs(sa);
    reg_fence(sb);
    if (r == 0 && h == 0) SAGE_TR(13, j);
    // S read: free for the next Q K^T into it
    tc_fence_before();
    mbar_arrive(&bar.s_ready[sbuf]);
    // P~[b] is free once the P~V MMA of tile j - 2 has read it
    if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.p_empty[b], ph ^ 1, abort_flag, status,
                                                     kDevTimeoutMma)))
      return;
    float sum = masked ? exp_chunk<true, QF8>(sa, 2 * h, ca, neg, lim, P)
                       : exp_chunk<false, QF8>(sa, 2 * h, ca, neg, lim, P);
    if (r == 0 && h == 0) SAGE_TR(14, j);
    sum += masked ? exp_chunk<true, QF8>(sb, 2 * h + 1, cb, neg, lim, P + 8)
                  : exp_chunk<false, QF8>(sb, 2 * h + 1, cb, neg, lim, P + 8);
    l = fmaf(alpha, l, sum);
    if (r == 0 && h == 0) SAGE_TR(10, j);
    tmem_wait_st();
    tc_fence_before();
    if (r == 0) SAGE_TR(2 + h, j);
    mbar_arrive(&bar.p_full[b]);
    if (r == 0 && h == 0) SAGE_TR(11, j);
  }
  l_s[h * 128 + r] = l;
  mbar_arrive(bar.l_ready);
}

// Q smoothing: the exp warpgroups take the row maximum themselves.  Each
// turns its 64 scores of tile j into biased log2-domain scores
// t = A c + bias (in place), takes their maximum, and exchanges it with the
// other warpgroup through shared memory (pm_full); both then form the same
// m_j = max(m_{j-1}, both halves) and alpha_j, warpgroup 0 publishes alpha_j
// for the fold (a_full), and the exponentials take 2^(t - m_j + log2 448).
// The stats warpgroup only stages the bias and folds, so the exact biased
// maximum (about 2.5 instructions a score) no longer sits on one warp per
// SM sub-partition.  Slots: the partial maxima of tile j in j % 2 (a
// warpgroup writes tile j + 2's only after passing tile j + 1's exchange,
// which the other enters only after reading tile j's); alpha in j % 4
// (written for tile j + 4 only after the bias of tile j + 4 is staged, which
// the stats warpgroup does only after reading alpha_j).
template <bool MASKED, bool QF8>
__device__ __forceinline__ float biased32(uint32_t (&s)[32], float c, const float* bias, int col0,
                                          int lim) {
  const float2 c2 = make_float2(c, c);
  const float2 mb = make_float2(-kBias, -kBias);
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const float4 bv = *reinterpret_cast<const float4*>(bias + i);
    float2 x01 = make_float2(score<QF8>(s[i]), score<QF8>(s[i + 1]));
    float2 x23 = make_float2(score<QF8>(s[i + 2]), score<QF8>(s[i + 3]));
    if (!QF8) {
      x01 = __fadd2_rn(x01, mb);
      x23 = __fadd2_rn(x23, mb);
    }
    const float2 t01 = __ffma2_rn(x01, c2, make_float2(bv.x, bv.y));
    const float2 t23 = __ffma2_rn(x23, c2, make_float2(bv.z, bv.w));
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

template <int D, bool CAUSAL, bool QF8, bool RAGGED>
__device__ __forceinline__ void exp_loop_smooth(const int h, const int qt, const int nkv,
                                                const int n_tail, const int bh, const int H,
                                                const int G, const int ntiles,
                                                const float* __restrict__ q_scales,
                                                const float* __restrict__ k_scales,
                                                const float scale_log2, const uint32_t tmem,
                                                const Bars& bar, uint8_t* smem,
                                                volatile int* abort_flag, uint32_t* status) {
  using L = Layout<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  const float* bias_s = reinterpret_cast<const float*>(smem + L::OFF_BIAS);
  float* pm_s = reinterpret_cast<float*>(smem + L::OFF_PM);
  float* a_s = reinterpret_cast<float*>(smem + L::OFF_A4);
  float* l_s = reinterpret_cast<float*>(smem + L::OFF_L);
  const float qs = __ldg(q_scales + ((int64_t)bh * ntiles + qt) * 128 + r);
  // this warpgroup's two K scales of every tile (keys 64h .. 64h + 63)
  const float* ksp = k_scales + (int64_t)kv_head(bh, H, G) * ntiles * 4 + 2 * h;

  tc_fence_before();
  mbar_arrive(bar.s_init);

  float l = 0.f, m = -INFINITY;
  float ks0 = ldg_early(ksp), ks1 = ldg_early(ksp + 1);
  for (int j = 0; j < nkv; ++j) {
    const int b = j & 1;
    const uint32_t ph = (j >> 1) & 1;
    const float ca = qs * (ks0 * scale_log2), cb = qs * (ks1 * scale_log2);
    float ks0n = 0.f, ks1n = 0.f;
    if (j + 1 < nkv) {
      ks0n = ldg_early(ksp + 4 * (j + 1));
      ks1n = ldg_early(ksp + 4 * (j + 1) + 1);
    }
    const int sbuf = j % L::SB;
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[sbuf], (j / L::SB) & 1, abort_flag, status,
                                           kDevTimeoutMma)))
      return;
    tc_fence_after();
    const bool diag = CAUSAL && (j == qt);
    const bool masked = diag || (RAGGED && j == nkv - 1);
    const int lim = diag ? r : n_tail - 1;
    const uint32_t S = tmem + lanes + 128u * sbuf + 64u * h;
    const uint32_t P = tmem + lanes + L::COL_P + 32u * b + 16u * h;
    uint32_t sa[32], sb[32];
    tmem_ld32(S, sa);
    tmem_ld32(S + 32, sb);
    tmem_wait_ld_regs(sa);
    reg_fence(sb);
    // S read: free for the next Q K^T into it
    tc_fence_before();
    mbar_arrive(&bar.s_ready[sbuf]);
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&bar.bias_full[b], ph, abort_flag, status, kDevTimeoutSoftmax)))
      return;
    const float* bias = bias_s + (j & 3) * 128 + 64 * h;
    const float p = masked ? fmaxf(biased32<true, QF8>(sa, ca, bias, 64 * h, lim),
                                   biased32<true, QF8>(sb, cb, bias + 32, 64 * h + 32, lim))
                           : fmaxf(biased32<false, QF8>(sa, ca, bias, 64 * h, lim),
                                   biased32<false, QF8>(sb, cb, bias + 32, 64 * h + 32, lim));
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
    const float neg = kLog2_448 - m_j;  // yields 448 P~ directly
    // P~[b] is free once the P~V MMA of tile j - 2 has read it
    if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.p_empty[b], ph ^ 1, abort_flag, status,
                                                     kDevTimeoutMma)))
      return;
    // the biased scores are plain FP32 now: t - m_j + log2 448 by one FMA
    float sum = masked ? exp_chunk<true, true>(sa, 2 * h, 1.f, neg, lim, P)
                       : exp_chunk<false, true>(sa, 2 * h, 1.f, neg, lim, P);
    sum += masked ? exp_chunk<true, true>(sb, 2 * h + 1, 1.f, neg, lim, P + 8)
                  : exp_chunk<false, true>(sb, 2 * h + 1, 1.f, neg, lim, P + 8);
    l = fmaf(alpha, l, sum);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bar.p_full[b]);
    ks0 = ks0n;
    ks1 = ks1n;
  }
  l_s[h * 128 + r] = l;
  mbar_arrive(bar.l_ready);
}

// Stats warpgroup: row max / running max per key tile, level-2 fold,
// epilogue.
template <int D, bool CAUSAL, typename OutT, bool QF8, bool RAGGED, bool SMOOTH>
__device__ __forceinline__ void stats_loop(const int qt, const int nkv, const int n_tail,
                                           const int bh, const int H, const int G, const int N,
                                           const int ntiles, const uint32_t tmem, const Bars& bar,
                                           uint8_t* smem, volatile int* abort_flag,
                                           uint32_t* status, const float* __restrict__ q_scales,
                                           const float* __restrict__ k_scales,
                                           const float* __restrict__ v_scales,
                                           const float* __restrict__ ds,
                                           OutT* __restrict__ out, const float scale_log2) {
  using L = Layout<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  float* m_s = reinterpret_cast<float*>(smem + L::OFF_M);
  const float* l_s = reinterpret_cast<const float*>(smem + L::OFF_L);
  // this row's Q scale; the K/V head's K scales, four per key tile
  const float qs = __ldg(q_scales + ((int64_t)bh * ntiles + qt) * 128 + r);
  const float* ksp = k_scales + (int64_t)kv_head(bh, H, G) * ntiles * 4;

  float2 o2[D / 2];
#pragma unroll
  for (int c = 0; c < D / 2; ++c) o2[c] = make_float2(0.f, 0.f);
  float m = -INFINITY;
  auto fold = [&](int i, float alpha) -> bool {
    const int b = i % L::PVB;
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.pv_full[b], (i / L::PVB) & 1, abort_flag, status,
                                           kDevTimeoutMma)))
      return false;
    tc_fence_after();
    if (r == 0) SAGE_TR(6, i);
    const uint32_t PV = tmem + lanes + L::COL_PV + (uint32_t)b * (uint32_t)D;
    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t pv[32];
      tmem_ld32(PV + 32 * cc, pv);
      tmem_wait_ld_regs(pv);
#pragma unroll
      for (int k = 0; k < 16; ++k)
        o2[cc * 16 + k] = __ffma2_rn(
            a2, o2[cc * 16 + k], make_float2(__uint_as_float(pv[2 * k]), __uint_as_float(pv[2 * k + 1])));
    }
    if (r == 0) SAGE_TR(7, i);
    tc_fence_before();
    mbar_arrive(&bar.pv_empty[b]);
    return true;
  };

  // The fold lags the max by PVB tiles, so the max of tile j + 1 (which the
  // exp warpgroups wait for) never queues behind the P~V product of tile j.
  float alpha_hist[2] = {0.f, 0.f};
  float* c_s = reinterpret_cast<float*>(smem + L::OFF_C);
  float4 ks_cur = ldg4_early(ksp);
  // Q smoothing: this query block's score bias.  Thread r writes key
  // 128 j + r of tile j (log2 units) into slot j % 4 of the shared bias
  // buffer one tile ahead, after reading alpha_{j-1}, and arrives on
  // bias_full[j % 2]; both exp warpgroups read the whole slot.  A slot is
  // rewritten for tile j + 4 after alpha_{j+3} is published, which both exp
  // warpgroups do only past their reads of tile j's bias.
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
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.a_full[j & 3], (j >> 2) & 1, abort_flag, status,
                                           kDevTimeoutSoftmax)))
      return;
    const float alpha = reinterpret_cast<const float*>(smem + L::OFF_A4)[(j & 3) * 128 + r];
    if (j + 1 < nkv) {
      bias_s[((j + 1) & 3) * 128 + r] = d_nxt * scale_log2;
      mbar_arrive(&bar.bias_full[(j + 1) & 1]);
      if (j + 2 < nkv) d_nxt = ldg_early(dsr + 128 * (j + 2) + r);
    }
    if (j >= L::PVB && !fold(j - L::PVB, alpha_hist[j % L::PVB])) return;
    alpha_hist[j % L::PVB] = alpha;
  }
  for (int j = 0; !SMOOTH && j < nkv; ++j) {
    const int b = j & 1;
    // s_K sm_scale log2 e of the tile's four 32-key chunks; a row's factor
    // is its Q scale times that (the exp warpgroups form the same products)
    const float kl[4] = {ks_cur.x * scale_log2, ks_cur.y * scale_log2, ks_cur.z * scale_log2,
                         ks_cur.w * scale_log2};
    const float4 ks_nxt = j + 1 < nkv ? ldg4_early(ksp + 4 * (j + 1)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const int sbuf = j % L::SB;
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[sbuf], (j / L::SB) & 1, abort_flag,
                                           status, kDevTimeoutMma)))
      return;
    tc_fence_after();
    if (r == 0) SAGE_TR(4, j);
    const bool diag = CAUSAL && (j == qt);
    const bool masked = diag || (RAGGED && j == nkv - 1);
    const int lim = diag ? r : n_tail - 1;
    const uint32_t S = tmem + lanes + (uint32_t)sbuf * 128u;
    float mx = -INFINITY;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t s[2][32];
      tmem_ld32(S + 64 * hh, s[0]);
      tmem_ld32(S + 64 * hh + 32, s[1]);
      tmem_wait_ld_regs(s[0]);
      reg_fence(s[1]);
      // each chunk's factor is >= 0, so its scaled max is the max scaled
      mx = masked ? scaled_max64<true, QF8>(&s[0][0], hh, lim, qs * kl[2 * hh],
                                            qs * kl[2 * hh + 1], mx)
                  : scaled_max64<false, QF8>(&s[0][0], hh, lim, qs * kl[2 * hh],
                                             qs * kl[2 * hh + 1], mx);
    }
    const float m_j = fmaxf(m, mx);
    const float alpha = ex2(m - m_j);
    m = m_j;
    m_s[(2 * b) * 128 + r] = m_j;
    m_s[(2 * b + 1) * 128 + r] = alpha;
    if (r == 0) {
      c_s[4 * b] = kl[0];
      c_s[4 * b + 1] = kl[1];
      c_s[4 * b + 2] = kl[2];
      c_s[4 * b + 3] = kl[3];
    }
    if (r == 0) SAGE_TR(5, j);
    // S[b] has been read: the exp warpgroups may overwrite it with P~ codes
    tc_fence_before();
    mbar_arrive(&bar.m_full[b]);
    if (j >= L::PVB && !fold(j - L::PVB, alpha_hist[j % L::PVB])) return;
    alpha_hist[j % L::PVB] = alpha;
    ks_cur = ks_nxt;
  }
  for (int i = nkv > L::PVB ? nkv - L::PVB : 0; i < nkv; ++i)
    if (!fold(i, alpha_hist[i % L::PVB])) return;
  if (!__all_sync(0xffffffffu,
                  mbar_wait(bar.l_ready, 0, abort_flag, status, kDevTimeoutSoftmax)))
    return;
  const float inv_l = 1.f / (l_s[r] + l_s[128 + r]);
  // s_V arrived in shared memory with Q (q_full has long completed)
  if (!__all_sync(0xffffffffu, mbar_wait(bar.q_full, 0, abort_flag, status, kDevTimeoutEpi)))
    return;
  const float* vs = reinterpret_cast<const float*>(smem + L::OFF_VS);
  // rows past the end of a ragged sequence are padding: not stored
  if (qt * 128 + r >= N) return;
  OutT* dst = out + ((int64_t)bh * N + (int64_t)qt * 128 + r) * D;
#pragma unroll
  for (int cv = 0; cv < D; cv += 8) {
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v = o2[cv / 2 + e];
      w4[e] = pack2<OutT>(v.x * vs[cv + 2 * e] * inv_l, v.y * vs[cv + 2 * e + 1] * inv_l);
    }
    *reinterpret_cast<uint4*>(dst + cv) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

template <int D, bool CAUSAL, typename OutT, bool QF8, bool RAGGED, bool SMOOTH>
__global__ void __launch_bounds__(kThreadsAttn, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scales,
                     const float* __restrict__ k_scales, const float* __restrict__ v_scales,
                     const float* __restrict__ ds, OutT* __restrict__ out, int N, int H, int G,
                     float scale_log2, int head_major, uint32_t* status) {
  using L = Layout<D>;
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
  // head-major grids (x = head) dispatch every head's heaviest causal tile
  // first: longest-first over the whole grid; tile-major grids (x = tile)
  // keep the concurrently running CTAs on few heads (K/V reuse in L2)
  const int bh = head_major ? (int)blockIdx.x : (int)blockIdx.y;
  const int tile_rank = head_major ? (int)blockIdx.y : (int)blockIdx.x;
  // K/V head of this query head (grouped-query attention: G query heads per
  // K/V head; G = 1 is plain multi-head attention)
  const int bhk = kv_head(bh, H, G);
  const int qt = CAUSAL ? (ntiles - 1 - tile_rank) : tile_rank;  // heavy first
  const int nkv = CAUSAL ? qt + 1 : ntiles;

  Bars bar = carve_bars<D>(smem);
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
    for (int i = 0; i < L::SB; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.s_ready[i], 256);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.m_full[i], 128);
      mbar_init(&bar.p_full[i], 256);
      mbar_init(&bar.p_empty[i], 1);
    }
    for (int i = 0; i < L::PVB; ++i) {
      mbar_init(&bar.pv_full[i], 1);
      mbar_init(&bar.pv_empty[i], 128);
    }
    mbar_init(bar.s_init, 256);
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

  const int wg = warp >> 2;
  if (wg == 0) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (elect_one()) {
        mbar_arrive_expect_tx(bar.q_full, L::Q_BYTES + 4 * D);
        tma_load_2d(sQ, &tm_q, 0, bh * Np + qt * 128, bar.q_full);
        bulk_load(smem + L::OFF_VS, v_scales + (int64_t)bhk * D, 4 * D, bar.q_full);
        for (int j = 0; j < nkv; ++j) {
          const int sk = j % L::KS;
          if (!mbar_wait<true>(&bar.k_empty[sk], ((j / L::KS) & 1) ^ 1, abort_flag, status,
                               kDevTimeoutMma))
            break;
          mbar_arrive_expect_tx(&bar.k_full[sk], L::K_BYTES);
          tma_load_2d(sK + sk * L::K_BYTES, &tm_k, 0, bhk * Np + j * 128, &bar.k_full[sk]);
          const int sv = j % L::VS;
          if (!mbar_wait<true>(&bar.v_empty[sv], ((j / L::VS) & 1) ^ 1, abort_flag, status,
                               kDevTimeoutMma))
            break;
          mbar_arrive_expect_tx(&bar.v_full[sv], L::V_BYTES);
          tma_load_2d(sV + sv * L::V_BYTES, &tm_v, j * 128, bhk * D, &bar.v_full[sv]);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------------------------------------------- tcgen05 issuer
      if (elect_one()) {
        constexpr uint32_t idesc_qk = QF8 ? make_idesc(1 /*F32*/, 0 /*e4m3*/, 0 /*e4m3*/, 128, 128)
                                          : make_idesc(2 /*S32*/, 1 /*s8*/, 1 /*s8*/, 128, 128);
        constexpr uint32_t idesc_pv = make_idesc(1 /*F32*/, 0 /*e4m3*/, 0 /*e4m3*/, 128, D);
        const uint64_t qdesc = make_sdesc(smem_u32(sQ), L::QK_SBO, 16, L::QK_SWZ);
        bool ok = mbar_wait(bar.q_full, 0, abort_flag, status, kDevTimeoutTma);
        // S[j % SB] = Q K_j^T
        auto qk = [&](int j) -> bool {
          const int sk = j % L::KS;
          const int sbuf = j % L::SB;
          if (!mbar_wait(&bar.k_full[sk], (j / L::KS) & 1, abort_flag, status, kDevTimeoutTma))
            return false;
          tc_fence_after();
          SAGE_TR(8, j);
          const uint64_t kdesc =
              make_sdesc(smem_u32(sK + sk * L::K_BYTES), L::QK_SBO, 16, L::QK_SWZ);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            if (QF8)
              mma_f8_ss(tmem + (uint32_t)sbuf * 128u, qdesc + 2 * kk, kdesc + 2 * kk, idesc_qk,
                        kk > 0);
            else
              mma_i8_ss(tmem + (uint32_t)sbuf * 128u, qdesc + 2 * kk, kdesc + 2 * kk, idesc_qk,
                        kk > 0);
          }
          mma_commit(&bar.s_full[sbuf]);
          mma_commit(&bar.k_empty[sk]);
          return true;
        };
        // P~_i V_i into PV[i % 2] (level 1)
        auto pv = [&](int i) -> bool {
          const int b = i & 1;
          const int sv = i % L::VS;
          const int pb = i % L::PVB;
          if (!mbar_wait(&bar.p_full[b], (i >> 1) & 1, abort_flag, status, kDevTimeoutSoftmax) ||
              !mbar_wait(&bar.v_full[sv], (i / L::VS) & 1, abort_flag, status, kDevTimeoutTma) ||
              !mbar_wait(&bar.pv_empty[pb], ((i / L::PVB) & 1) ^ 1, abort_flag, status,
                         kDevTimeoutEpi))
            return false;
          tc_fence_after();
          SAGE_TR(9, i);
          const uint64_t vdesc = make_sdesc(smem_u32(sV + sv * L::V_BYTES), 1024, 16, Swz::k128);
          const uint32_t d = tmem + L::COL_PV + (uint32_t)pb * (uint32_t)D;
          const uint32_t pa = tmem + L::COL_P + 32u * (uint32_t)b;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ts(d, pa + 8u * kk, vdesc + 2 * kk, idesc_pv, kk > 0);
          mma_commit(&bar.pv_full[pb]);
          mma_commit(&bar.p_empty[b]);
          mma_commit(&bar.v_empty[sv]);
          return true;
        };
        if (ok) ok = mbar_wait(bar.s_init, 0, abort_flag, status, kDevTimeoutSoftmax);
        for (int j = 0; ok && j < L::SB && j < nkv; ++j) ok = qk(j);
        // The exp warpgroups release S for tile i early in their pass over
        // it: the Q K^T of tile i + SB goes first (the scores the stats
        // warpgroup needs next), the P~V of tile i - 1 (the fold runs two
        // tiles behind) second, so the scores never queue behind it.
        for (int i = 0; ok && i < nkv; ++i) {
          if (i + L::SB < nkv) {
            if (!mbar_wait(&bar.s_ready[i % L::SB], (i / L::SB) & 1, abort_flag, status,
                           kDevTimeoutSoftmax)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (!qk(i + L::SB)) {
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
    exp_loop_smooth<D, CAUSAL, QF8, RAGGED>(wg - 1, qt, nkv, n_tail, bh, H, G, ntiles, q_scales,
                                            k_scales, scale_log2, tmem, bar, smem, abort_flag,
                                            status);
  } else if (wg < 3) {
    // the exp warpgroups keep the 128 registers they were launched with
    exp_loop<D, CAUSAL, QF8, RAGGED>(wg - 1, qt, nkv, n_tail, bh, ntiles, q_scales, tmem, bar, smem,
                                     abort_flag, status);
  } else {
    setmaxnreg_inc<kRegsStats>();
    stats_loop<D, CAUSAL, OutT, QF8, RAGGED, SMOOTH>(qt, nkv, n_tail, bh, H, G, N, ntiles, tmem, bar,
                                                     smem, abort_flag, status, q_scales, k_scales,
                                                     v_scales, ds, out, scale_log2);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
#ifdef SAGE_TRACE
  if (SAGE_TRACED_CTA && threadIdx.x < 64)
    for (int e = 0; e < 16; ++e) g_sage_trace[e][threadIdx.x] = s_sage_trace[e][threadIdx.x];
#endif
}

template <int D, bool CAUSAL, typename OutT, bool QF8, bool RAGGED = false>
cudaError_t launch_typed(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, cudaStream_t st) {
  using L = Layout<D>;
  auto kern = a.ds ? attn_i8f8_kernel<D, CAUSAL, OutT, QF8, RAGGED, true>
                   : attn_i8f8_kernel<D, CAUSAL, OutT, QF8, RAGGED, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)((a.N + 127) / 128);
  const int hm = head_major_grid(a);
  const dim3 grid = hm ? dim3((unsigned)(a.B * a.H), (unsigned)ntiles)
                       : dim3((unsigned)ntiles, (unsigned)(a.B * a.H));
  kern<<<grid, kThreadsAttn, L::SMEM, st>>>(tq, tk, tv, a.q_scales, a.k_scales, a.v_scales, a.ds,
                                           reinterpret_cast<OutT*>(a.o), (int)a.N, (int)a.H,
                                           (int)(a.H / a.Hkv), a.sm_scale * kLog2e, hm,
                                           a.status);
  return cudaGetLastError();
}

template <int D, bool QF8>
cudaError_t launch_d(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, cudaStream_t st) {
  if (a.causal) {
    return a.dtype == 1 ? launch_typed<D, true, __nv_bfloat16, QF8>(a, tq, tk, tv, st)
                        : launch_typed<D, true, __half, QF8>(a, tq, tk, tv, st);
  }
  // causal launches mask the partial last tile through the diagonal already
  if (a.N % 128 != 0)
    return a.dtype == 1 ? launch_typed<D, false, __nv_bfloat16, QF8, true>(a, tq, tk, tv, st)
                        : launch_typed<D, false, __half, QF8, true>(a, tq, tk, tv, st);
  return a.dtype == 1 ? launch_typed<D, false, __nv_bfloat16, QF8>(a, tq, tk, tv, st)
                      : launch_typed<D, false, __half, QF8>(a, tq, tk, tv, st);
}

}  // namespace

cudaError_t launch_attn_i8f8(const AttnArgs& a, cudaStream_t st, const char** detail) {
  if (use_persistent_attention(a)) return launch_attn_i8f8_persist(a, st, detail);
  const uint64_t BH = (uint64_t)(a.B * a.H);
  const uint64_t BHK = (uint64_t)(a.B * a.Hkv);
  const uint64_t N = (uint64_t)((a.N + 127) / 128 * 128);  // codes padded to whole tiles
  const uint64_t D = (uint64_t)a.d;
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_swz =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q_codes, D, BH * N, D, (uint32_t)D, 128,
                      qk_swz, detail) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.k_codes, D, BHK * N, D, (uint32_t)D,
                      128, qk_swz, detail) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.v_codes, N, BHK * D, N, 128, (uint32_t)D,
                      CU_TENSOR_MAP_SWIZZLE_128B, detail))
    return cudaErrorInvalidValue;
  if (a.mode == kModeFp8)
    return D == 128 ? launch_d<128, true>(a, tq, tk, tv, st) : launch_d<64, true>(a, tq, tk, tv, st);
  return D == 128 ? launch_d<128, false>(a, tq, tk, tv, st) : launch_d<64, false>(a, tq, tk, tv, st);
}

}  // namespace sage

#ifdef SAGE_TRACE
extern "C" int sage_trace_read(long long* host) {
  return (int)cudaMemcpyFromSymbol(host, sage::g_sage_trace, sizeof(long long) * 16 * 512);
}

#endif
