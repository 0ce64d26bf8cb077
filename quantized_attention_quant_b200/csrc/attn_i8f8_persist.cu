// attn_i8f8_persist.cu -- the INT8 (or FP8) Q K^T + FP8 P~V attention
// forward of attn_i8f8.cu as a persistent kernel, for sm_100a.
//
// Same computation, same warp roles and per-tile pipeline as attn_i8f8.cu
// (SageAttention abstract: INT8 Q K^T; SageAttention2 abstract: FP8 P~ and
// V, two-level P~V accumulation; the online softmax of "Flash Attention vs
// Sage Attention: Kernel Comparison"), but each CTA (one per SM) works
// through a list of work items (query tile, b*h).  A CTA pays its start-up
// once, and an item's epilogue overlaps the next item's tiles:
//   - the key tiles of consecutive items form one stream through the K/V
//     rings, S, P~ and PV buffers (all indexed by the CTA's tile count);
//   - Q is double-buffered (the next item's Q loads during this one);
//   - the row sums of an item are triple-buffered, its s_V copy too;
//   - the stats warpgroup folds each tile two behind its max; after an
//     item's last fold it normalises O into a 128-byte-swizzled staging
//     tile, and one thread stores it with a TMA tensor store, which clips
//     the rows past N of a ragged sequence.
// It pays off where items are short (causal prefill of a few thousand
// tokens: a CTA's start-up and epilogue cost about as much as three key
// tiles); long items use the one-item-per-CTA kernel.

#include "attn_i8f8_common.cuh"

namespace sage {
namespace {

template <int D>
struct Layout {
  static constexpr int KS = D == 128 ? 4 : 6;  // K ring depth
  static constexpr int VS = D == 128 ? 4 : 6;  // V ring depth
  static constexpr int Q_BYTES = 128 * D;
  static constexpr int K_BYTES = 128 * D;
  static constexpr int V_BYTES = D * 128;
  static constexpr int O_BYTES = 128 * D * 2;        // one 16-bit O tile, staged for the TMA store
  static constexpr int OFF_Q = 0;                    // Q[2]: this item's and the next one's
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * K_BYTES;
  static constexpr int OFF_O = OFF_V + VS * V_BYTES;
  static constexpr int OFF_MISC = OFF_O + O_BYTES;
  static constexpr int OFF_BAR = OFF_MISC;           // barriers (<= 64 x 8 B)
  static constexpr int OFF_TMEM = OFF_MISC + 512;
  static constexpr int OFF_ABORT = OFF_MISC + 528;
  static constexpr int OFF_M = OFF_MISC + 1024;      // [2 slots][m, alpha][128]
  static constexpr int OFF_L = OFF_M + 4 * 128 * 4;  // [3 items][2 halves][128] row sums
  static constexpr int OFF_C = OFF_L + 6 * 128 * 4;  // [2 slots][4] s_K sm_scale log2 e per 32 keys
  static constexpr int OFF_VS = OFF_C + 128;         // [3][D] s_V of an item (bulk-copied)
  static constexpr int END = OFF_VS + 3 * 4 * D;
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
  uint64_t* q_full;    // [2] producer -> MMA: Q of an item landed
  uint64_t* q_empty;   // [2] MMA (after the item's last Q K^T) -> producer
  uint64_t* vs_full;   // [3] producer -> stats: s_V of an item landed
  uint64_t* vs_empty;  // [3] stats (epilogue done) -> producer
  uint64_t* o_free;    // [1] stats leader -> stats: the O staging buffer is free
  uint64_t* o_full;    // [1] stats warps -> stats leader: O rows staged
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
  uint64_t* l_ready;   // [3] exp -> stats: an item's final row sums
  uint64_t* drain;     // MMA drain on abort
};

template <int D>
__device__ __forceinline__ Bars carve_bars(uint8_t* smem) {
  using L = Layout<D>;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  Bars r;
  r.q_full = b;
  r.q_empty = b + 2;
  r.vs_full = b + 4;
  r.vs_empty = b + 7;
  r.o_free = b + 10;
  r.o_full = b + 11;
  r.k_full = b + 12;
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
  r.drain = r.l_ready + 3;
  return r;
}

// ----------------------------------------------------------------- schedule
// The kernel is persistent: G CTAs (one per SM at most) share the W work
// items (query tile, b*h).  Items are dealt in rounds of G, alternating
// direction: round r gives CTA c the item r*G + c when r is even and
// r*G + G-1-c when odd.  In item order the causal tiles run from the
// heaviest down (head-major order when every head's K/V codes fit in L2,
// see head_major_grid), so each CTA's share of work is balanced, and every
// role of a CTA derives the same item list without communicating.
struct Sched {
  int W, G, ntiles, BH, head_major;
  __device__ __forceinline__ int count(int c) const {
    const int R = W / G, rem = W % G;
    return R + ((((R & 1) ? G - 1 - c : c) < rem) ? 1 : 0);
  }
  __device__ __forceinline__ int item(int c, int r) const {
    return r * G + ((r & 1) ? G - 1 - c : c);
  }
};

// One work item of this CTA, and a walk over its key tiles.
template <bool CAUSAL>
struct Cursor {
  int it = -1;  // item index in this CTA's list
  int j = 0;    // key tile within the item
  int nkv = 0, qt = 0, bh = 0;
  __device__ __forceinline__ void load(const Sched& s, int c, int item_idx) {
    it = item_idx;
    j = 0;
    const int k = s.item(c, item_idx);
    const int rank = s.head_major ? k / s.BH : k % s.ntiles;
    bh = s.head_major ? k % s.BH : k / s.ntiles;
    qt = CAUSAL ? s.ntiles - 1 - rank : rank;
    nkv = CAUSAL ? qt + 1 : s.ntiles;
  }
  // to the next key tile (the first tile of the next item past the last)
  __device__ __forceinline__ void next(const Sched& s, int c) {
    if (++j == nkv) load(s, c, it + 1);
  }
};

// Exp warpgroup h (0 or 1): key columns 64h .. 64h+63 of every tile of every
// item.  RAGGED (non-causal launches of a sequence whose last tile is
// partial): the last key tile of an item masks keys n_tail .. 127.
template <int D, bool CAUSAL, bool QF8, bool RAGGED>
__device__ __forceinline__ void exp_loop(const int h, const Sched& sch, const int T,
                                         const int n_tail, const float* __restrict__ q_scales,
                                         const uint32_t tmem, const Bars& bar,
                                         uint8_t* smem, volatile int* abort_flag,
                                         uint32_t* status) {
  using L = Layout<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  const float* m_s = reinterpret_cast<const float*>(smem + L::OFF_M);
  const float* c_s = reinterpret_cast<const float*>(smem + L::OFF_C);
  float* l_s = reinterpret_cast<float*>(smem + L::OFF_L);

  // (every Q K^T overwrites S: nothing to prepare in TMEM)
  tc_fence_before();
  mbar_arrive(bar.s_init);

  Cursor<CAUSAL> cur;
  cur.load(sch, blockIdx.x, 0);
  const int nitems = sch.count(blockIdx.x);
  // this row's Q scale in the current item; the next item's is loaded at
  // the start of the current item's last tile, a tile ahead of its use
  float qs = ldg_early(q_scales + ((int64_t)cur.bh * sch.ntiles + cur.qt) * 128 + r);
  float qs_next = 0.f;
  // l restarts at every item by itself: the first tile's alpha is 0
  float l = 0.f;
  for (int g = 0; g < T; ++g, cur.next(sch, blockIdx.x)) {
    const int j = cur.j;
    const int b = g & 1;
    const uint32_t ph = (g >> 1) & 1;
    if (j == cur.nkv - 1 && cur.it + 1 < nitems) {
      Cursor<CAUSAL> nx;
      nx.load(sch, blockIdx.x, cur.it + 1);
      qs_next = ldg_early(q_scales + ((int64_t)nx.bh * sch.ntiles + nx.qt) * 128 + r);
    }
    // m_full(g) is published by the stats warpgroup after it waited for
    // s_full(g) and read S[b]: it orders this warpgroup after the Q K^T too
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&bar.m_full[b], ph, abort_flag, status, kDevTimeoutEpi)))
      return;
    tc_fence_after();
    // dequant factors of this warpgroup's two 32-key chunks (the stats
    // warpgroup forms its maximum from the same products)
    const float ca = qs * c_s[4 * b + 2 * h], cb = qs * c_s[4 * b + 2 * h + 1];
    const float m_j = m_s[(2 * b) * 128 + r];
    const float alpha = m_s[(2 * b + 1) * 128 + r];
    const float neg = kLog2_448 - m_j;  // yields 448 P~ directly
    // masked tiles: the causal diagonal (keys up to the row) and the last
    // tile of a ragged sequence (keys up to n_tail - 1)
    const bool diag = CAUSAL && (j == cur.qt);
    const bool masked = diag || (RAGGED && j == cur.nkv - 1);
    const int lim = diag ? r : n_tail - 1;
    const int sbuf = g % L::SB;
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
    // P~[b] is free once the P~V MMA of tile g - 2 has read it
    if (g >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.p_empty[b], ph ^ 1, abort_flag, status,
                                                     kDevTimeoutMma)))
      return;
    float sum = masked ? exp_chunk<true, QF8>(sa, 2 * h, ca, neg, lim, P)
                       : exp_chunk<false, QF8>(sa, 2 * h, ca, neg, lim, P);
    sum += masked ? exp_chunk<true, QF8>(sb, 2 * h + 1, cb, neg, lim, P + 8)
                  : exp_chunk<false, QF8>(sb, 2 * h + 1, cb, neg, lim, P + 8);
    l = fmaf(alpha, l, sum);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bar.p_full[b]);
    if (j == cur.nkv - 1) {
      // the item's row sums, for its epilogue (three buffers: the stats
      // warpgroup reads item i's before this one can reach item i + 3)
      const int lb = cur.it % 3;
      l_s[(lb * 2 + h) * 128 + r] = l;
      mbar_arrive(&bar.l_ready[lb]);
      qs = qs_next;
    }
  }
}

// Stats warpgroup: row max / running max per key tile, level-2 fold (two
// tiles behind), and each item's epilogue once its last tile is folded.
template <int D, bool CAUSAL, typename OutT, bool QF8, bool RAGGED>
__device__ __forceinline__ void stats_loop(const Sched& sch, const int T, const int n_tail,
                                           const int H, const int G,
                                           const uint32_t tmem, const Bars& bar, uint8_t* smem,
                                           volatile int* abort_flag, uint32_t* status,
                                           const float* __restrict__ q_scales,
                                           const float* __restrict__ k_scales,
                                           const CUtensorMap* tm_o, const float scale_log2) {
  using L = Layout<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const bool leader = (threadIdx.x == 3 * 128);  // issues the O stores
  const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
  const int ntiles = sch.ntiles;
  float* m_s = reinterpret_cast<float*>(smem + L::OFF_M);
  const float* l_s = reinterpret_cast<const float*>(smem + L::OFF_L);
  float* c_s = reinterpret_cast<float*>(smem + L::OFF_C);

  float2 o2[D / 2];
#pragma unroll
  for (int c = 0; c < D / 2; ++c) o2[c] = make_float2(0.f, 0.f);

  // O of a finished item: normalise, stage (128-byte swizzled rows, the
  // TMA layout) and store with the tensor map (rows past N are clipped).
  // Every wait here is a bounded mbarrier wait (no named barrier), so an
  // abort elsewhere cannot leave part of the warpgroup waiting for the rest.
  auto epilogue = [&](const Cursor<CAUSAL>& f) -> bool {
    const int lb = f.it % 3;
    const uint32_t ph = f.it & 1;  // one epilogue per item, in order
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.l_ready[lb], (f.it / 3) & 1, abort_flag, status,
                                           kDevTimeoutSoftmax) &&
                                     mbar_wait(&bar.vs_full[lb], (f.it / 3) & 1, abort_flag,
                                               status, kDevTimeoutTma)))
      return false;
    const float inv_l = 1.f / (l_s[(lb * 2) * 128 + r] + l_s[(lb * 2 + 1) * 128 + r]);
    const float* vs = reinterpret_cast<const float*>(smem + L::OFF_VS + lb * 4 * D);
    // the staging buffer is free once the previous item's store has read it
    if (leader) {
      bulk_wait_read();
      mbar_arrive(bar.o_free);
    }
    if (!__all_sync(0xffffffffu, mbar_wait(bar.o_free, ph, abort_flag, status, kDevTimeoutEpi)))
      return false;
    uint8_t* stage = smem + L::OFF_O;
#pragma unroll
    for (int cv = 0; cv < D; cv += 8) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 v = o2[cv / 2 + e];
        w4[e] = pack2<OutT>(v.x * vs[cv + 2 * e] * inv_l, v.y * vs[cv + 2 * e + 1] * inv_l);
      }
      const int box = cv / 64, chunk = (cv % 64) / 8;
      *reinterpret_cast<uint4*>(stage + box * (128 * 128) + r * 128 + ((chunk ^ (r & 7)) << 4)) =
          make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    // the rows are visible to the TMA (async proxy), and s_V was read
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar.o_full);
    bool good = true;
    if (leader) {
      good = mbar_wait(bar.o_full, ph, abort_flag, status, kDevTimeoutEpi);
      if (good) {
#pragma unroll
        for (int box = 0; box < D / 64; ++box)
          tma_store_3d(tm_o, stage + box * (128 * 128), box * 64, f.qt * 128, f.bh);
        bulk_commit();
        mbar_arrive(&bar.vs_empty[lb]);
      }
    }
    // warp-uniform result (the leader's warp decides with its lane 0)
    return __shfl_sync(0xffffffffu, good, 0);
  };

  auto fold = [&](int i, float alpha) -> bool {
    const int b = i % L::PVB;
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.pv_full[b], (i / L::PVB) & 1, abort_flag, status,
                                           kDevTimeoutMma)))
      return false;
    tc_fence_after();
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
    tc_fence_before();
    mbar_arrive(&bar.pv_empty[b]);
    return true;
  };

  // the fold lags the max by PVB tiles (an item's first fold has alpha = 0,
  // which clears the accumulator of the previous item)
  Cursor<CAUSAL> fc;  // tile being folded
  fc.load(sch, blockIdx.x, 0);

  float alpha_hist[2] = {0.f, 0.f};
  Cursor<CAUSAL> mc;  // tile whose max is taken
  mc.load(sch, blockIdx.x, 0);
  const int nitems = sch.count(blockIdx.x);
  // this row's Q scale and the K/V head's K scales (four per key tile) of
  // the current item; the next item's are loaded at the start of the
  // current item's last tile, a tile ahead of their use
  const float* ksp = k_scales + (int64_t)kv_head(mc.bh, H, G) * ntiles * 4;
  const float* ksp_next = ksp;
  float qs = ldg_early(q_scales + ((int64_t)mc.bh * ntiles + mc.qt) * 128 + r);
  float qs_next = 0.f;
  float4 ks_cur = ldg4_early(ksp);
  float m = -INFINITY;
  // one pass: the max of tile g (g < T), then the fold of tile g - PVB
  for (int g = 0; g < T + L::PVB; ++g) {
    float alpha = 0.f;
    if (g < T) {
      const int j = mc.j;
      const int b = g & 1;
      if (j == 0) m = -INFINITY;  // a new item: a fresh running max
      // s_K sm_scale log2 e of the tile's four 32-key chunks; a row's factor
      // is its Q scale times that (the exp warpgroups form the same products)
      const float kl[4] = {ks_cur.x * scale_log2, ks_cur.y * scale_log2, ks_cur.z * scale_log2,
                           ks_cur.w * scale_log2};
      float4 ks_nxt = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j + 1 < mc.nkv) {
        ks_nxt = ldg4_early(ksp + 4 * (j + 1));
      } else if (mc.it + 1 < nitems) {
        Cursor<CAUSAL> nx;
        nx.load(sch, blockIdx.x, mc.it + 1);
        ksp_next = k_scales + (int64_t)kv_head(nx.bh, H, G) * ntiles * 4;
        ks_nxt = ldg4_early(ksp_next);
        qs_next = ldg_early(q_scales + ((int64_t)nx.bh * ntiles + nx.qt) * 128 + r);
      }
      const int sbuf = g % L::SB;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[sbuf], (g / L::SB) & 1, abort_flag,
                                             status, kDevTimeoutMma)))
        break;
      tc_fence_after();
      const bool diag = CAUSAL && (j == mc.qt);
      const bool masked = diag || (RAGGED && j == mc.nkv - 1);
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
      alpha = ex2(m - m_j);
      m = m_j;
      m_s[(2 * b) * 128 + r] = m_j;
      m_s[(2 * b + 1) * 128 + r] = alpha;
      if (r == 0) {
        c_s[4 * b] = kl[0];
        c_s[4 * b + 1] = kl[1];
        c_s[4 * b + 2] = kl[2];
        c_s[4 * b + 3] = kl[3];
      }
      // S[b] has been read: the exp warpgroups may overwrite it with P~ codes
      tc_fence_before();
      mbar_arrive(&bar.m_full[b]);
      ks_cur = ks_nxt;
      if (j == mc.nkv - 1) {
        qs = qs_next;
        ksp = ksp_next;
      }
      mc.next(sch, blockIdx.x);
    }
    if (g >= L::PVB) {
      const int i = g - L::PVB;
      if (!fold(i, alpha_hist[i % L::PVB])) break;
      if (fc.j == fc.nkv - 1 && !epilogue(fc)) break;
      fc.next(sch, blockIdx.x);
    }
    if (g < T) alpha_hist[g % L::PVB] = alpha;
  }
  // every O store has completed before the CTA leaves
  if (leader) bulk_wait_all();
}

template <int D, bool CAUSAL, typename OutT, bool QF8, bool RAGGED>
__global__ void __launch_bounds__(kThreadsAttn, 1)
    attn_i8f8_persist_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_o, const float* __restrict__ q_scales,
                     const float* __restrict__ k_scales, const float* __restrict__ v_scales,
                     int N, int H, int G, float scale_log2, Sched sch, uint32_t* status) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // N tokens in ntiles 128-token tiles (codes padded to Np = 128 ntiles);
  // the last tile holds n_tail of them
  const int ntiles = sch.ntiles;
  const int Np = ntiles * 128;
  const int n_tail = N - (ntiles - 1) * 128;
  const int c = blockIdx.x;
  const int nitems = sch.count(c);
  // key tiles of all of this CTA's items
  int T = 0;
  for (int i = 0; i < nitems; ++i) {
    Cursor<CAUSAL> t;
    t.load(sch, c, i);
    T += t.nkv;
  }

  Bars bar = carve_bars<D>(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.q_full[i], 1);
      mbar_init(&bar.q_empty[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&bar.vs_full[i], 1);
      mbar_init(&bar.vs_empty[i], 1);
    }
    mbar_init(bar.o_free, 1);
    mbar_init(bar.o_full, 4);
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
    for (int i = 0; i < 3; ++i) mbar_init(&bar.l_ready[i], 256);
    mbar_init(bar.s_init, 256);
    mbar_init(bar.drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
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
        int g = 0;  // key tiles of the earlier items
        for (int it = 0; it < nitems; ++it) {
          Cursor<CAUSAL> cu;
          cu.load(sch, c, it);
          const int bhk = kv_head(cu.bh, H, G);
          const int qb = it & 1;
          // Q buffer qb is free once item it - 2 is done with it
          if (!mbar_wait<true>(&bar.q_empty[qb], ((it >> 1) & 1) ^ 1, abort_flag, status,
                               kDevTimeoutSoftmax))
            break;
          mbar_arrive_expect_tx(&bar.q_full[qb], L::Q_BYTES);
          tma_load_2d(sQ + qb * L::Q_BYTES, &tm_q, 0, cu.bh * Np + cu.qt * 128, &bar.q_full[qb]);
          // s_V buffer it % 3 is free once the epilogue of item it - 3 is done
          const int vb = it % 3;
          if (!mbar_wait<true>(&bar.vs_empty[vb], ((it / 3) & 1) ^ 1, abort_flag, status,
                               kDevTimeoutEpi))
            break;
          mbar_arrive_expect_tx(&bar.vs_full[vb], 4 * D);
          bulk_load(smem + L::OFF_VS + vb * 4 * D, v_scales + (int64_t)bhk * D, 4 * D,
                    &bar.vs_full[vb]);
          bool ok = true;
          for (int j = 0; j < cu.nkv; ++j) {
            const int gj = g + j;
            const int sk = gj % L::KS;
            if (!mbar_wait<true>(&bar.k_empty[sk], ((gj / L::KS) & 1) ^ 1, abort_flag, status,
                                 kDevTimeoutMma)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bar.k_full[sk], L::K_BYTES);
            tma_load_2d(sK + sk * L::K_BYTES, &tm_k, 0, bhk * Np + j * 128, &bar.k_full[sk]);
            const int sv = gj % L::VS;
            if (!mbar_wait<true>(&bar.v_empty[sv], ((gj / L::VS) & 1) ^ 1, abort_flag, status,
                                 kDevTimeoutMma)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bar.v_full[sv], L::V_BYTES);
            tma_load_2d(sV + sv * L::V_BYTES, &tm_v, j * 128, bhk * D, &bar.v_full[sv]);
          }
          if (!ok) break;
          g += cu.nkv;
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------------------------------------------- tcgen05 issuer
      if (elect_one()) {
        constexpr uint32_t idesc_qk = QF8 ? make_idesc(1 /*F32*/, 0 /*e4m3*/, 0 /*e4m3*/, 128, 128)
                                          : make_idesc(2 /*S32*/, 1 /*s8*/, 1 /*s8*/, 128, 128);
        constexpr uint32_t idesc_pv = make_idesc(1 /*F32*/, 0 /*e4m3*/, 0 /*e4m3*/, 128, D);
        Cursor<CAUSAL> qc;  // item of the next Q K^T
        qc.load(sch, c, 0);
        // S[g % SB] = Q K_g^T (Q of the tile's item)
        auto qk = [&](int g) -> bool {
          const int sk = g % L::KS;
          const int sbuf = g % L::SB;
          const int qb = qc.it & 1;
          if (qc.j == 0 && !mbar_wait(&bar.q_full[qb], (qc.it >> 1) & 1, abort_flag, status,
                                      kDevTimeoutTma))
            return false;
          if (!mbar_wait(&bar.k_full[sk], (g / L::KS) & 1, abort_flag, status, kDevTimeoutTma))
            return false;
          tc_fence_after();
          const uint64_t qdesc = make_sdesc(smem_u32(sQ + qb * L::Q_BYTES), L::QK_SBO, 16, L::QK_SWZ);
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
          // the item's last Q K^T: its Q buffer may be refilled
          if (qc.j == qc.nkv - 1) mma_commit(&bar.q_empty[qb]);
          qc.next(sch, c);
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
        bool ok = mbar_wait(bar.s_init, 0, abort_flag, status, kDevTimeoutSoftmax);
        for (int g = 0; ok && g < L::SB && g < T; ++g) ok = qk(g);
        // The exp warpgroups release S for tile i early in their pass over
        // it: the Q K^T of tile i + SB goes first (the scores the stats
        // warpgroup needs next), the P~V of tile i - 1 (the fold runs two
        // tiles behind) second, so the scores never queue behind it.  The
        // tiles of consecutive items form one stream.
        for (int i = 0; ok && i < T; ++i) {
          if (i + L::SB < T) {
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
        if (ok && T > 0) ok = pv(T - 1);
        if (!ok) {
          // let every MMA already issued finish before TMEM is released
          mma_commit(bar.drain);
          volatile int no_abort = 0;
          mbar_wait(bar.drain, 0, &no_abort, status, kDevTimeoutMma);
        }
      }
      __syncwarp();
    }
  } else if (wg < 3) {
    // the exp warpgroups keep the 128 registers they were launched with
    exp_loop<D, CAUSAL, QF8, RAGGED>(wg - 1, sch, T, n_tail, q_scales, tmem, bar, smem, abort_flag,
                                     status);
  } else {
    setmaxnreg_inc<kRegsStats>();
    stats_loop<D, CAUSAL, OutT, QF8, RAGGED>(sch, T, n_tail, H, G, tmem, bar, smem, abort_flag,
                                            status, q_scales, k_scales, &tm_o, scale_log2);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool CAUSAL, typename OutT, bool QF8, bool RAGGED = false>
cudaError_t launch_typed(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t st) {
  using L = Layout<D>;
  Sched sch;
  sch.ntiles = (int)((a.N + 127) / 128);
  sch.BH = (int)(a.B * a.H);
  sch.W = sch.ntiles * sch.BH;
  sch.G = sm_count() < sch.W ? sm_count() : sch.W;
  sch.head_major = head_major_grid(a);
  auto kern = attn_i8f8_persist_kernel<D, CAUSAL, OutT, QF8, RAGGED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)sch.G), kThreadsAttn, L::SMEM, st>>>(
      tq, tk, tv, to, a.q_scales, a.k_scales, a.v_scales, (int)a.N, (int)a.H,
      (int)(a.H / a.Hkv), a.sm_scale * kLog2e, sch, a.status);
  return cudaGetLastError();
}

template <int D, bool QF8>
cudaError_t launch_d(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t st) {
  if (a.causal) {
    return a.dtype == 1 ? launch_typed<D, true, __nv_bfloat16, QF8>(a, tq, tk, tv, to, st)
                        : launch_typed<D, true, __half, QF8>(a, tq, tk, tv, to, st);
  }
  // causal launches mask the partial last tile through the diagonal already
  if (a.N % 128 != 0)
    return a.dtype == 1 ? launch_typed<D, false, __nv_bfloat16, QF8, true>(a, tq, tk, tv, to, st)
                        : launch_typed<D, false, __half, QF8, true>(a, tq, tk, tv, to, st);
  return a.dtype == 1 ? launch_typed<D, false, __nv_bfloat16, QF8>(a, tq, tk, tv, to, st)
                      : launch_typed<D, false, __half, QF8>(a, tq, tk, tv, to, st);
}

}  // namespace

cudaError_t launch_attn_i8f8_persist(const AttnArgs& a, cudaStream_t st, const char** detail) {
  const uint64_t BH = (uint64_t)(a.B * a.H);
  const uint64_t BHK = (uint64_t)(a.B * a.Hkv);
  const uint64_t N = (uint64_t)((a.N + 127) / 128 * 128);  // codes padded to whole tiles
  const uint64_t D = (uint64_t)a.d;
  CUtensorMap tq, tk, tv, to;
  const CUtensorMapSwizzle qk_swz =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  // O [B*H][N][d] in the output dtype, stored as 128-row x 64-column boxes
  // (128-byte swizzled rows); rows past N are clipped by the tensor map
  const CUtensorMapDataType odt =
      a.dtype == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q_codes, D, BH * N, D, (uint32_t)D, 128,
                      qk_swz, detail) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.k_codes, D, BHK * N, D, (uint32_t)D,
                      128, qk_swz, detail) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.v_codes, N, BHK * D, N, 128, (uint32_t)D,
                      CU_TENSOR_MAP_SWIZZLE_128B, detail) ||
      !encode_tmap_3d(&to, odt, a.o, D, (uint64_t)a.N, BH, D * 2, (uint64_t)a.N * D * 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B, detail))
    return cudaErrorInvalidValue;
  if (a.mode == kModeFp8)
    return D == 128 ? launch_d<128, true>(a, tq, tk, tv, to, st)
                    : launch_d<64, true>(a, tq, tk, tv, to, st);
  return D == 128 ? launch_d<128, false>(a, tq, tk, tv, to, st)
                  : launch_d<64, false>(a, tq, tk, tv, to, st);
}

}  // namespace sage
