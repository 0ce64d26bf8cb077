// sage_internal.h -- launcher argument blocks shared by the C-ABI layer and
// the kernels (host side only).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace sage {

// sage_mode_t values (include/sage.h)
constexpr int kModeInt8Fp8 = 0;  // INT8 Q/K, FP8 P~ and V
constexpr int kModeFp4 = 1;      // FP4 Q/K/P~/V
constexpr int kModeFp8 = 2;      // FP8 Q/K, FP8 P~ and V

struct QuantQKArgs {
  const void* q;
  const void* k;
  int dtype;  // 0 = f16, 1 = bf16
  int mode;   // kModeInt8Fp8 / kModeFp4 / kModeFp8 (sage_mode_t values)
  int64_t B, H, N, d;
  int64_t Hkv;  // K heads (H % Hkv == 0; Hkv == H without grouped-query attention)
  void* q_codes;
  float* q_scales;
  void* q_sf;
  void* k_codes;
  float* k_scales;
  void* k_sf;
  float* k_mean;
  double* ws_ksum;  // [B*H, N/128, d] FP64 chunk partial sums (workspace)
  uint32_t* ws_cnt;  // [2][65536] per-head statistics counters: zero before the
                     // call, zero again after it (workspace)
  uint32_t* status = nullptr;  // device status word (bounded waits of the fused pre-pass)
  // Q smoothing (8-bit modes): when q_mean is set, Q loses its per-128-token
  // block mean before quantization (q_mean [B*H, N/128, d] FP32 receives
  // it) and ds [B*H, N/128, Np] FP32 receives the score bias qbar . k'
  float* q_mean = nullptr;
  float* ds = nullptr;
};

struct QuantVArgs {
  const void* v;
  int dtype;
  int mode;  // as above; V is FP8 in both 8-bit modes
  int64_t B, H, N, d;
  void* v_codes;
  float* v_scales;
  void* v_sf;
  double* ws_ksum;  // scratch the V statistics pass may write (same size as above)
  float* ws_vmax;   // [B*H, N/128, d] per-chunk |V| maxima (workspace)
  uint32_t* ws_cnt;  // as in QuantQKArgs
};

// The per-head counters at the start of every workspace: K counters at
// [0, kMaxStatHeads), V counters at [kMaxStatHeads, 2 kMaxStatHeads).
constexpr int kMaxStatHeads = 65536;
constexpr size_t kStatsCounterBytes = size_t(2) * kMaxStatHeads * 4;

struct AttnArgs {
  int mode;
  const void* q_codes;
  const float* q_scales;
  const void* q_sf;
  const void* k_codes;
  const float* k_scales;
  const void* k_sf;
  const void* v_codes;
  const float* v_scales;
  const void* v_sf;
  void* o;
  int dtype;
  int64_t B, H, N, d;
  int64_t Hkv;  // K/V heads: query head h reads K/V head h / (H / Hkv)
  int causal;
  float sm_scale;
  uint32_t* status;  // device status word
  // Q smoothing: the score bias [B*H, N/128, Np] of sage_quant_qk_smooth
  // (null: none)
  const float* ds = nullptr;
};

cudaError_t launch_quant_qk(const QuantQKArgs& a, cudaStream_t st);
cudaError_t launch_quant_v(const QuantVArgs& a, cudaStream_t st);
// The whole 8-bit pre-pass (Q, K and V) in one cluster launch, for sequences
// whose K / V head slices fit in one cluster's shared memory.
bool fused_prepass_fits(const QuantQKArgs& a);
cudaError_t launch_prepass_fused(const QuantQKArgs& qa, const QuantVArgs& va, cudaStream_t st);

// Returns cudaSuccess, or an error; `detail` receives a message on failure
// of something other than a CUDA call (e.g. tensor-map encoding).
cudaError_t launch_attn_i8f8(const AttnArgs& a, cudaStream_t st, const char** detail);
cudaError_t launch_attn_fp4(const AttnArgs& a, cudaStream_t st, const char** detail);

// Grouped-query attention: the key/value head read by flattened query head
// bh = b * H + h, with G query heads per key/value head (G = 1: multi-head).
__host__ __device__ __forceinline__ int kv_head(int bh, int H, int G) {
  return (bh / H) * (H / G) + (bh % H) / G;
}

// Grid order of the attention kernels.  Causal query tiles differ in work
// (tile t sees t + 1 key tiles); CTAs start in grid order, so a head-major
// grid (every head's heaviest tile first) runs longest-first over the whole
// launch, which keeps the tail short.  It also spreads the running CTAs over
// all heads, so it is used only while every head's K and V codes fit in L2
// together (at most 64 MB); otherwise the grid stays tile-major, where the
// running CTAs share the K/V tiles of a few heads.
inline int head_major_grid(const AttnArgs& a) {
  if (!a.causal) return 0;
  const int64_t np = (a.N + 127) / 128 * 128;
  const int64_t kv_bytes = 2 * a.B * a.Hkv * np * a.d;  // 8-bit K and V codes
  return kv_bytes <= (int64_t(64) << 20) ? 1 : 0;
}

// The INT8/FP8 attention runs as a persistent kernel (one CTA per SM
// working through a list of (query tile, b*h) items) when the items are
// short: a CTA's start-up and epilogue then cost as much as a few key tiles,
// and the persistent kernel overlaps them with the next item.  Long items
// keep one CTA each, which the hardware balances itself.
int sm_count();
inline bool use_persistent_attention(const AttnArgs& a) {
  if (a.ds) return false;  // Q smoothing runs in the one-item-per-CTA kernel
  const int64_t ntiles = (a.N + 127) / 128;
  const int64_t mean_tiles = a.causal ? (ntiles + 1) / 2 : ntiles;
  return mean_tiles <= 64 && ntiles * a.B * a.H > sm_count();
}
cudaError_t launch_attn_i8f8_persist(const AttnArgs& a, cudaStream_t st, const char** detail);

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library does not link libcuda).  Returns false with a message on failure.
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t dim0,
                    uint64_t dim1, uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                    CUtensorMapSwizzle swz, const char** detail);
// The same for a 3-D tensor (box depth 1 in dimension 2).
bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t dim0,
                    uint64_t dim1, uint64_t dim2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                    uint32_t box0, uint32_t box1, CUtensorMapSwizzle swz, const char** detail);
// Streaming multiprocessors of the current device (cached per device):
// declared above.

}  // namespace sage
