// attn_i8f8.cu -- fused quantized attention forward, INT8 Q K^T + FP8 P~V,
// for sm_100a (tcgen05 tensor cores, TMEM accumulators, TMA).
//
// What it computes (SageAttention abstract: INT8 Q K^T; SageAttention2
// abstract: FP8 P~ and V with two-level accumulation of P~V; the online
// softmax of "Flash Attention vs Sage Attention: Kernel Comparison",
// section "How FlashAttention reduces memory traffic"):
//
//   per query row, over 128-key tiles j (causal: j <= query tile):
//     A      = q_codes . k_codes_j^T                 (tcgen05 kind::i8, exact)
//     t      = A * (s_Q s_Kj sm_scale log2 e)        (log2 domain)
//     m_new  = max(m, rowmax t); alpha = 2^(m - m_new)
//     p      = e4m3(448 * 2^(t - m_new))             (448 P~, quantized)
//     l      = alpha l + sum 448 P~                  (unquantized P~)
//     part_j = p . v_codes_j                         (kind::f8f6f4, fresh FP32)
//     O      = alpha O + part_j                      (FP32, registers)
//   O_out = O * s_V[c] / l
//
// One CTA owns one 128-row query tile of one (b, h) and walks all key tiles.
// Warp roles (320 threads):
//   warp 0      TMA producer: Q once, then K_j and V_j^T into 4/6-deep rings
//   warp 1      TMEM allocator and the single-thread tcgen05 issuer
//   warps 2..5  softmax: thread = one query row (TMEM lane); reads S_j from
//               TMEM, writes the e4m3 P~ tile back into TMEM (aliasing the
//               first 32 columns of S_j) as the A operand of the P~V MMA
//   warps 6..9  correction: reads each per-tile FP32 partial from TMEM and
//               folds it into the row's running FP32 accumulator (level 2),
//               then normalises and writes O
// TMEM columns: S[0] 0..127, S[1] 128..255, PV[0] 256.., PV[1] 256+D.. .
// Every barrier wait is bounded; an expired wait sets the device status
// word and makes every role leave its loop.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {
namespace {

constexpr int kThreadsAttn = 320;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)

template <int D>
struct I8F8Layout {
  static constexpr int KS = D == 128 ? 4 : 6;  // K ring depth
  static constexpr int VS = D == 128 ? 4 : 6;  // V ring depth
  static constexpr int Q_BYTES = 128 * D;
  static constexpr int K_BYTES = 128 * D;
  static constexpr int V_BYTES = D * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * K_BYTES;
  static constexpr int OFF_MISC = OFF_V + VS * V_BYTES;
  // misc: barriers (64 x 8 B), tmem slot, abort flag, alpha ring [4][128],
  // l [128]
  static constexpr int OFF_BAR = OFF_MISC;
  static constexpr int OFF_TMEM = OFF_MISC + 512;
  static constexpr int OFF_ABORT = OFF_MISC + 528;
  static constexpr int OFF_ALPHA = OFF_MISC + 1024;
  static constexpr int OFF_L = OFF_ALPHA + 4 * 128 * 4;
  static constexpr int END = OFF_L + 128 * 4;
  // at least 120 KB so that one CTA (holding all 512 TMEM columns) runs per SM
  static constexpr int SMEM = (END + 1024 > 120 * 1024 ? END + 1024 : 120 * 1024);
  // shared-memory descriptor strides
  static constexpr uint32_t QK_SBO = 8 * D;  // 8 rows of D bytes
  static constexpr Swz QK_SWZ = D == 128 ? Swz::k128 : Swz::k64;
};

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* s_full;    // [2] MMA -> softmax
  uint64_t* p_full;    // [2] softmax -> MMA
  uint64_t* pv_full;   // [2] MMA -> correction
  uint64_t* pv_empty;  // [2] correction -> MMA
  uint64_t* a_full;    // [4] softmax -> correction (alpha ring)
  uint64_t* l_ready;   // [1] softmax -> correction (final l)
  uint64_t* drain;     // [1] MMA drain on abort
};

template <int D>
__device__ __forceinline__ Bars carve_bars(uint8_t* smem) {
  using L = I8F8Layout<D>;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  Bars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = r.k_full + L::KS;
  r.v_full = r.k_empty + L::KS;
  r.v_empty = r.v_full + L::VS;
  r.s_full = r.v_empty + L::VS;
  r.p_full = r.s_full + 2;
  r.pv_full = r.p_full + 2;
  r.pv_empty = r.pv_full + 2;
  r.a_full = r.pv_empty + 2;
  r.l_ready = r.a_full + 4;
  r.drain = r.l_ready + 1;
  return r;
}

constexpr uint32_t kBiasBits = 0x4B400000u;  // bit pattern of 1.5 * 2^23
constexpr float kBias = 12582912.0f;

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Max of 128 non-negative floats given as bits: 8 independent 3-input max
// chains, then a short tree.
__device__ __forceinline__ float row_max128(const uint32_t (&s)[128]) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(__uint_as_float(s[k]), __uint_as_float(s[k + 8]));
#pragma unroll
  for (int i = 16; i < 128; i += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k)
      a[k] = fmax3(a[k], __uint_as_float(s[i + k]), __uint_as_float(s[i + 8 + k]));
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

// 448 P~ = 2^((x - bias) c + neg) for the 128 biased scores of a row,
// quantized to e4m3 (four codes per 32-bit word, key i in byte i % 4), and
// the sum of the unquantized values.  MASKED: keys i > r contribute 0.
template <bool MASKED>
__device__ __forceinline__ float exp_quant128(const uint32_t (&s)[128], float c, float neg, int r,
                                              uint32_t (&p)[32]) {
  const float2 c2 = make_float2(c, c);
  const float2 n2 = make_float2(neg, neg);
  const float2 mb = make_float2(-kBias, -kBias);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int i = 0; i < 128; i += 4) {
    const float2 x01 = __fadd2_rn(make_float2(__uint_as_float(s[i]), __uint_as_float(s[i + 1])), mb);
    const float2 x23 =
        __fadd2_rn(make_float2(__uint_as_float(s[i + 2]), __uint_as_float(s[i + 3])), mb);
    const float2 t01 = __ffma2_rn(x01, c2, n2);
    const float2 t23 = __ffma2_rn(x23, c2, n2);
    float f0 = ex2(t01.x), f1 = ex2(t01.y), f2 = ex2(t23.x), f3 = ex2(t23.y);
    if (MASKED) {
      f0 = (i + 0 <= r) ? f0 : 0.f;
      f1 = (i + 1 <= r) ? f1 : 0.f;
      f2 = (i + 2 <= r) ? f2 : 0.f;
      f3 = (i + 3 <= r) ? f3 : 0.f;
    }
    acc[(i >> 2) & 3] = __fadd2_rn(acc[(i >> 2) & 3], make_float2(f0, f1));
    acc[(i >> 2) & 3] = __fadd2_rn(acc[(i >> 2) & 3], make_float2(f2, f3));
    p[i >> 2] = cvt_e4m3x2(f0, f1) | (cvt_e4m3x2(f2, f3) << 16);
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
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

template <int D, bool CAUSAL, typename OutT>
__global__ void __launch_bounds__(kThreadsAttn, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scales,
                     const float* __restrict__ k_scales, const float* __restrict__ v_scales,
                     OutT* __restrict__ out, int N, float scale_log2, uint32_t* status) {
  using L = I8F8Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = N / 128;
  const int bh = blockIdx.y;
  const int qt = CAUSAL ? (ntiles - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int nkv = CAUSAL ? qt + 1 : ntiles;

  Bars bar = carve_bars<D>(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);
  float* alpha_s = reinterpret_cast<float*>(smem + L::OFF_ALPHA);
  float* l_s = reinterpret_cast<float*>(smem + L::OFF_L);

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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.p_full[i], 128);
      mbar_init(&bar.pv_full[i], 1);
      mbar_init(&bar.pv_empty[i], 128);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&bar.a_full[i], 128);
    mbar_init(bar.l_ready, 128);
    mbar_init(bar.drain, 1);
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
  // TMEM column bases of the double-buffered S/P~ and P~V tiles
  auto tS = [tmem](int b) -> uint32_t { return tmem + (uint32_t)b * 128u; };
  auto tPV = [tmem](int b) -> uint32_t { return tmem + 256u + (uint32_t)b * (uint32_t)D; };

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      mbar_arrive_expect_tx(bar.q_full, L::Q_BYTES);
      tma_load_2d(sQ, &tm_q, 0, bh * N + qt * 128, bar.q_full);
      for (int j = 0; j < nkv; ++j) {
        const int sk = j % L::KS;
        if (!mbar_wait(&bar.k_empty[sk], ((j / L::KS) & 1) ^ 1, abort_flag, status, kDevTimeoutMma))
          break;
        mbar_arrive_expect_tx(&bar.k_full[sk], L::K_BYTES);
        tma_load_2d(sK + sk * L::K_BYTES, &tm_k, 0, bh * N + j * 128, &bar.k_full[sk]);
        const int sv = j % L::VS;
        if (!mbar_wait(&bar.v_empty[sv], ((j / L::VS) & 1) ^ 1, abort_flag, status, kDevTimeoutMma))
          break;
        mbar_arrive_expect_tx(&bar.v_full[sv], L::V_BYTES);
        tma_load_2d(sV + sv * L::V_BYTES, &tm_v, j * 128, bh * D, &bar.v_full[sv]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- tcgen05 issuer
    if (elect_one()) {
      constexpr uint32_t idesc_qk = make_idesc(2 /*S32*/, 1 /*s8*/, 1 /*s8*/, 128, 128);
      constexpr uint32_t idesc_pv = make_idesc(1 /*F32*/, 0 /*e4m3*/, 0 /*e4m3*/, 128, D);
      const uint64_t q_desc = make_sdesc(smem_u32(sQ), L::QK_SBO, 16, L::QK_SWZ);
      bool ok = mbar_wait(bar.q_full, 0, abort_flag, status, kDevTimeoutTma);
      auto issue_pv = [&](int jj) -> bool {
        const int b = jj & 1;
        const int sv = jj % L::VS;
        if (!mbar_wait(&bar.p_full[b], (jj >> 1) & 1, abort_flag, status, kDevTimeoutSoftmax))
          return false;
        if (!mbar_wait(&bar.v_full[sv], (jj / L::VS) & 1, abort_flag, status, kDevTimeoutTma))
          return false;
        if (!mbar_wait(&bar.pv_empty[b], ((jj >> 1) & 1) ^ 1, abort_flag, status, kDevTimeoutEpi))
          return false;
        tc_fence_after();
        const uint64_t v_desc = make_sdesc(smem_u32(sV + sv * L::V_BYTES), 1024, 16, Swz::k128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8_ts(tPV(b), tS(b) + kk * 8, v_desc + 2 * kk, idesc_pv, kk > 0);
        mma_commit(&bar.pv_full[b]);
        mma_commit(&bar.v_empty[sv]);
        return true;
      };
      for (int j = 0; ok && j < nkv; ++j) {
        const int sk = j % L::KS;
        if (!mbar_wait(&bar.k_full[sk], (j / L::KS) & 1, abort_flag, status, kDevTimeoutTma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int b = j & 1;
        const uint64_t k_desc = make_sdesc(smem_u32(sK + sk * L::K_BYTES), L::QK_SBO, 16, L::QK_SWZ);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tS(b), q_desc + 2 * kk, k_desc + 2 * kk, idesc_qk, kk > 0);
        mma_commit(&bar.s_full[b]);
        mma_commit(&bar.k_empty[sk]);
        if (j > 0 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) ok = issue_pv(nkv - 1);
      if (!ok) {
        // let every MMA already issued finish before TMEM is released
        mma_commit(bar.drain);
        volatile int no_abort = 0;
        mbar_wait(bar.drain, 0, &no_abort, status, kDevTimeoutMma);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float qs = __ldg(q_scales + (int64_t)bh * ntiles + qt);
    const float* ksp = k_scales + (int64_t)bh * ntiles;
    float m = -INFINITY;
    float l = 0.f;
    float ks_next = __ldg(ksp);
    for (int j = 0; j < nkv; ++j) {
      const int b = j & 1;
      const float ks = ks_next;
      if (j + 1 < nkv) ks_next = __ldg(ksp + j + 1);
      // warp-uniform decision: the tcgen05.ld/st below are .sync.aligned
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&bar.s_full[b], (j >> 1) & 1, abort_flag, status, kDevTimeoutMma)))
        break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(lane_base + tS(b) + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(lane_base + tS(b) + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(lane_base + tS(b) + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(lane_base + tS(b) + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_wait_ld();
      const bool diag = CAUSAL && (j == qt);
      const float c = qs * ks * scale_log2;
      // Integer scores -> floats without a conversion instruction: with the
      // bias 1.5 * 2^23 added, the bit pattern is the float 1.5 * 2^23 + A
      // exactly (|A| <= 127^2 * 128 < 2^22); subtracting the bias back is
      // exact too.  The biased floats are ordered like A, so the row max is
      // taken on them directly.
#pragma unroll
      for (int i = 0; i < 128; ++i) s[i] += kBiasBits;
      if (diag) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > r) s[i] = 0u;  // masked keys: +0.0, below every biased score
      }
      const float m_new = fmaxf(m, (row_max128(s) - kBias) * c);
      const float alpha = ex2(m - m_new);
      const float neg = kLog2_448 - m_new;  // yields 448 P~ directly
      uint32_t p[32];
      const float sum = diag ? exp_quant128<true>(s, c, neg, r, p)
                             : exp_quant128<false>(s, c, neg, r, p);
      l = fmaf(alpha, l, sum);
      m = m_new;
      alpha_s[(j & 3) * 128 + r] = alpha;
      mbar_arrive(&bar.a_full[j & 3]);
      tmem_st32(lane_base + tS(b), p);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.p_full[b]);
    }
    l_s[r] = l;
    mbar_arrive(bar.l_ready);
  } else {
    // ---------------------------------------------------------- correction
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float2 o2[D / 2];
#pragma unroll
    for (int c = 0; c < D / 2; ++c) o2[c] = make_float2(0.f, 0.f);
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int b = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.a_full[j & 3], (j >> 2) & 1, abort_flag,
                                             status, kDevTimeoutSoftmax))) {
        ok = false;
        break;
      }
      const float alpha = alpha_s[(j & 3) * 128 + r];
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.pv_full[b], (j >> 1) & 1, abort_flag, status,
                                             kDevTimeoutMma))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t t[32];
        tmem_ld32(lane_base + tPV(b) + cc * 32, t);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          o2[cc * 16 + i] = __ffma2_rn(
              a2, o2[cc * 16 + i], make_float2(__uint_as_float(t[2 * i]), __uint_as_float(t[2 * i + 1])));
      }
      tc_fence_before();
      mbar_arrive(&bar.pv_empty[b]);
    }
    if (ok && mbar_wait(bar.l_ready, 0, abort_flag, status, kDevTimeoutSoftmax)) {
      const float inv_l = 1.f / l_s[r];
      const float* vs = v_scales + (int64_t)bh * D;
      OutT* dst = out + ((int64_t)bh * N + (int64_t)qt * 128 + r) * D;
#pragma unroll
      for (int c = 0; c < D; c += 8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = o2[c / 2 + e];
          w[e] = pack2<OutT>(v.x * __ldg(vs + c + 2 * e) * inv_l,
                             v.y * __ldg(vs + c + 2 * e + 1) * inv_l);
        }
        *reinterpret_cast<uint4*>(dst + c) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool CAUSAL, typename OutT>
cudaError_t launch_typed(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, cudaStream_t st) {
  using L = I8F8Layout<D>;
  auto kern = attn_i8f8_kernel<D, CAUSAL, OutT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)(a.N / 128);
  dim3 grid((unsigned)ntiles, (unsigned)(a.B * a.H));
  kern<<<grid, kThreadsAttn, L::SMEM, st>>>(tq, tk, tv, a.q_scales, a.k_scales, a.v_scales,
                                           reinterpret_cast<OutT*>(a.o), (int)a.N,
                                           a.sm_scale * kLog2e, a.status);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, cudaStream_t st) {
  if (a.causal) {
    return a.dtype == 1 ? launch_typed<D, true, __nv_bfloat16>(a, tq, tk, tv, st)
                        : launch_typed<D, true, __half>(a, tq, tk, tv, st);
  }
  return a.dtype == 1 ? launch_typed<D, false, __nv_bfloat16>(a, tq, tk, tv, st)
                      : launch_typed<D, false, __half>(a, tq, tk, tv, st);
}

}  // namespace

cudaError_t launch_attn_i8f8(const AttnArgs& a, cudaStream_t st, const char** detail) {
  const uint64_t BH = (uint64_t)(a.B * a.H);
  const uint64_t N = (uint64_t)a.N;
  const uint64_t D = (uint64_t)a.d;
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_swz =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q_codes, D, BH * N, D, (uint32_t)D, 128,
                      qk_swz, detail) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.k_codes, D, BH * N, D, (uint32_t)D, 128,
                      qk_swz, detail) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.v_codes, N, BH * D, N, 128, (uint32_t)D,
                      CU_TENSOR_MAP_SWIZZLE_128B, detail))
    return cudaErrorInvalidValue;
  return D == 128 ? launch_d<128>(a, tq, tk, tv, st) : launch_d<64>(a, tq, tk, tv, st);
}

}  // namespace sage
