// api.cu -- the C ABI (include/sage.h): argument checks, buffer sizing, the
// per-(device, stream) workspace, tensor-map encoding and the device status
// word.  No exception crosses the ABI.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/sage.h"
#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {

__device__ uint32_t g_device_status;  // bits from sage_ptx.cuh, per device

// Self-test of the bounded waits: an mbarrier that nothing arrives on, so
// the wait runs out (after kWaitLimitNs), records its bit in the status word
// and returns; the kernel then exits normally.
__global__ void wait_selftest_kernel(uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, kDevTimeoutSoftmax);
  __syncthreads();
}

namespace {

thread_local int t_last_status = 0;
thread_local std::string t_last_detail;

int fail(int status, const std::string& detail) {
  t_last_status = status;
  t_last_detail = detail;
  return status;
}

int fail_cuda(cudaError_t e, const char* where) {
  std::string d = std::string(where) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) +
                  ")";
  return fail(SAGE_ERR_CUDA, d);
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device facts, looked up once.
struct DeviceInfo {
  bool checked = false;
  bool sm100 = false;
  uint32_t* status = nullptr;
};
std::mutex g_mu;
std::map<int, DeviceInfo> g_dev;

int device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.checked) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute");
    di.sm100 = (major == 10 && minor == 0);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_status);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(status)");
    di.status = static_cast<uint32_t*>(p);
    di.checked = true;
  }
  if (!di.sm100)
    return fail(SAGE_ERR_UNSUPPORTED, "the current device is not compute capability 10.0 (sm_100)");
  *out = &di;
  return SAGE_OK;
}

// Stream-ordered workspace, one per (device, stream): a call on stream S
// only ever touches the workspace of S, so calls on different streams
// never share scratch memory.  Its first kStatsCounterBytes hold the
// per-head statistics counters of the pre-pass: zeroed when the workspace
// is (re)allocated, and left at zero by every pre-pass.
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

// Workspace allocations still to fail on purpose (sage_debug_fail_allocations):
// the failure is made on the host, in place of the allocation call.
int g_fail_allocs = 0;

int workspace(cudaStream_t st, size_t need, void** out, uint32_t** counters) {
  need += kStatsCounterBytes;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[{dev, st}];
  if (w.bytes < need) {
    if (w.ptr) {
      e = cudaFreeAsync(w.ptr, st);
      if (e != cudaSuccess) return fail_cuda(e, "cudaFreeAsync(workspace)");
      w.ptr = nullptr;
      w.bytes = 0;
    }
    const size_t grow = need + need / 4;
    if (g_fail_allocs > 0) {
      --g_fail_allocs;
      return fail(SAGE_ERR_CUDA,
                  "cudaMallocAsync(workspace): injected failure (sage_debug_fail_allocations)");
    }
    e = cudaMallocAsync(&w.ptr, grow, st);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMallocAsync(workspace)");
    w.bytes = grow;
    e = cudaMemsetAsync(w.ptr, 0, kStatsCounterBytes, st);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(workspace counters)");
  }
  *counters = static_cast<uint32_t*>(w.ptr);
  *out = static_cast<char*>(w.ptr) + kStatsCounterBytes;
  return SAGE_OK;
}

// A second stream per device.  The pre-pass is two independent chains:
// Q codes + K statistics then K codes, and V statistics then V codes; the
// V chain runs on this stream, forked from and joined back to the caller's
// stream by events (a pattern stream capture records as a fork and a join).
// The two chains use disjoint parts of the workspace (K sums and counters
// vs. V maxima and counters).
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex mu;  // one fork/join at a time: the events are shared
};
std::map<int, SideStream*> g_side;

int side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  SideStream*& ss = g_side[dev];
  if (!ss) {
    auto* n = new SideStream;
    if ((e = cudaStreamCreateWithFlags(&n->s, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&n->fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&n->join, cudaEventDisableTiming)) != cudaSuccess) {
      delete n;
      return fail_cuda(e, "side stream setup");
    }
    ss = n;
  }
  *out = ss;
  return SAGE_OK;
}

// Q/K chain on st, V chain on the side stream; st continues after both.
// Sequences short enough for the cluster-fused pre-pass take one launch on st.
int prepass_forked(const QuantQKArgs& qa, const QuantVArgs& va, cudaStream_t st) {
  if (fused_prepass_fits(qa)) {
    const cudaError_t e = launch_prepass_fused(qa, va, st);
    if (e != cudaSuccess) return fail_cuda(e, "fused pre-pass launch");
    return SAGE_OK;
  }

  SideStream* ss = nullptr;
  const int got = side_stream(&ss);
  if (got != SAGE_OK) return got;
  std::lock_guard<std::mutex> lk(ss->mu);
  cudaError_t e;
  if ((e = cudaEventRecord(ss->fork, st)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess)
    return fail_cuda(e, "pre-pass fork");
  if ((e = launch_quant_v(va, ss->s)) != cudaSuccess) return fail_cuda(e, "quant_v launch");
  if ((e = cudaEventRecord(ss->join, ss->s)) != cudaSuccess)
    return fail_cuda(e, "pre-pass join");
  // the caller's stream waits for the V chain even if the Q/K launch fails
  const cudaError_t eq = launch_quant_qk(qa, st);
  if ((e = cudaStreamWaitEvent(st, ss->join, 0)) != cudaSuccess)
    return fail_cuda(e, "pre-pass join");
  if (eq != cudaSuccess) return fail_cuda(eq, "quant_qk launch");
  return SAGE_OK;
}

struct WorkspaceReleaser {
  ~WorkspaceReleaser() {
    // Best effort at unload; during process teardown the runtime may already
    // be gone, in which case the calls fail harmlessly.
    for (auto& kv : g_ws)
      if (kv.second.ptr) cudaFree(kv.second.ptr);
  }
} g_ws_releaser;

// ---------------------------------------------------------------- checks

int check_common(int dtype, int mode, int64_t B, int64_t H, int64_t N, int64_t d, bool* empty) {
  if (dtype != SAGE_DTYPE_F16 && dtype != SAGE_DTYPE_BF16)
    return fail(SAGE_ERR_INVALID_ARG, "dtype must be SAGE_DTYPE_F16 or SAGE_DTYPE_BF16");
  if (mode != SAGE_MODE_INT8_FP8 && mode != SAGE_MODE_FP4 && mode != SAGE_MODE_FP8)
    return fail(SAGE_ERR_INVALID_ARG,
                "mode must be SAGE_MODE_INT8_FP8, SAGE_MODE_FP4 or SAGE_MODE_FP8");
  if (B < 0 || H < 0 || N < 0 || d < 0) return fail(SAGE_ERR_INVALID_ARG, "negative size");
  *empty = (B == 0 || H == 0 || N == 0);
  if (d != 64 && d != 128) return fail(SAGE_ERR_UNSUPPORTED, "head dim d must be 64 or 128");
  if (mode == SAGE_MODE_FP4 && d != 128)
    return fail(SAGE_ERR_UNSUPPORTED, "FP4 mode supports d == 128 only");
  if (!*empty) {
    // code buffers hold N rounded up to whole 128-token tiles per head
    const int64_t Np = (N + 127) / 128 * 128;
    if (B * H > 65535) return fail(SAGE_ERR_UNSUPPORTED, "B*H must be <= 65535");
    if (B * H * Np > 2147483647LL)
      return fail(SAGE_ERR_UNSUPPORTED, "B*H*N (N rounded up to a multiple of 128) must be < 2^31");
  }
  return SAGE_OK;
}

int check_ptr(const void* p, const char* name, bool required) {
  if (!p) {
    if (required) return fail(SAGE_ERR_INVALID_ARG, std::string(name) + " is NULL");
    return SAGE_OK;
  }
  if (!aligned16(p)) return fail(SAGE_ERR_UNSUPPORTED, std::string(name) + " is not 16-byte aligned");
  return SAGE_OK;
}

int check_unused(const void* p, const char* name) {
  if (p) return fail(SAGE_ERR_INVALID_ARG, std::string(name) + " must be NULL outside FP4 mode");
  return SAGE_OK;
}

#define SAGE_TRY(x)           \
  do {                        \
    int _s = (x);             \
    if (_s != SAGE_OK) return _s; \
  } while (0)

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn(const char** detail) {
  static std::once_flag once;
  static EncodeFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  if (!fn && detail) *detail = "cuTensorMapEncodeTiled is not available from the driver";
  return fn;
}

size_t ws_ksum_bytes(int64_t BH, int64_t N, int64_t d) {
  return (size_t)(BH * ((N + 127) / 128) * d * 8);
}
size_t ws_vmax_bytes(int64_t BH, int64_t N, int64_t d) {
  return (size_t)(BH * ((N + 127) / 128) * d * 4);
}

}  // namespace

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t dim0,
                    uint64_t dim1, uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                    CUtensorMapSwizzle swz, const char** detail) {
  EncodeFn fn = encode_fn(detail);
  if (!fn) return false;
  const cuuint64_t dims[2] = {dim0, dim1};
  const cuuint64_t strides[1] = {stride1_bytes};
  const cuuint32_t box[2] = {box0, box1};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (detail) *detail = "cuTensorMapEncodeTiled rejected a tensor map";
    return false;
  }
  return true;
}

bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t dim0,
                    uint64_t dim1, uint64_t dim2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                    uint32_t box0, uint32_t box1, CUtensorMapSwizzle swz, const char** detail) {
  EncodeFn fn = encode_fn(detail);
  if (!fn) return false;
  const cuuint64_t dims[3] = {dim0, dim1, dim2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (detail) *detail = "cuTensorMapEncodeTiled rejected a tensor map";
    return false;
  }
  return true;
}

int sm_count() {
  static std::mutex mu;
  static std::map<int, int> counts;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(mu);
  auto it = counts.find(dev);
  if (it != counts.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  counts[dev] = n;
  return n;
}

}  // namespace sage

using namespace sage;

extern "C" size_t sage_buffer_bytes(int mode, int which, int64_t B, int64_t H, int64_t N,
                                    int64_t d);

namespace {

// H >= 0 is already checked; no query heads means no key/value heads
int check_kv_heads(int64_t H, int64_t Hkv) {
  if (H == 0 ? Hkv != 0 : (Hkv < 1 || Hkv > H || H % Hkv != 0))
    return fail(SAGE_ERR_INVALID_ARG, "Hkv must be >= 1 and divide H");
  return SAGE_OK;
}

// Q-side buffers are per query head, K/V-side ones per key/value head
int64_t heads_of(int which, int64_t H, int64_t Hkv) {
  return which == SAGE_BUF_Q_CODES || which == SAGE_BUF_Q_SCALES || which == SAGE_BUF_Q_SF ||
                 which == SAGE_BUF_Q_MEAN || which == SAGE_BUF_DS
             ? H
             : Hkv;
}

// The whole pipeline (pre-pass, then attention) with every buffer carved
// from the per-stream workspace. Q and O have H heads, K and V have Hkv heads
// (Hkv divides H; Hkv == H is plain multi-head attention).
// Workspace layout of one forward pass (codes, scales, statistics partials,
// and with Q smoothing the Q means and the score bias), relative to the
// workspace base.
struct FwdLayout {
  size_t off[SAGE_BUF_V_SF + 1];
  size_t ksum, vmax, qmean, ds, total;
};

FwdLayout fwd_layout(int mode, bool smooth, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                     int64_t d) {
  FwdLayout L{};
  size_t total = 0;
  for (int w = 0; w <= SAGE_BUF_V_SF; ++w) {
    L.off[w] = total;
    total += align_up(sage_buffer_bytes(mode, w, B, heads_of(w, H, Hkv), N, d));
  }
  L.ksum = total;
  total += align_up(ws_ksum_bytes(B * Hkv, N, d));
  L.vmax = total;
  total += align_up(ws_vmax_bytes(B * Hkv, N, d));
  L.qmean = total;
  if (smooth) total += align_up(sage_buffer_bytes(mode, SAGE_BUF_Q_MEAN, B, H, N, d));
  L.ds = total;
  if (smooth) total += align_up(sage_buffer_bytes(mode, SAGE_BUF_DS, B, H, N, d));
  L.total = total;
  return L;
}

// The pre-pass and the attention of one forward pass on `st`, every buffer
// carved from `base` (laid out by fwd_layout) and the statistics counters
// `cnt`.  Arguments are already checked.
int run_fwd(const void* q, const void* k, const void* v, void* o, int dtype, int64_t B, int64_t H,
            int64_t Hkv, int64_t N, int64_t d, int causal, float sm_scale, int mode, bool smooth,
            char* base, uint32_t* cnt, uint32_t* status, cudaStream_t st) {
  const FwdLayout L = fwd_layout(mode, smooth, B, H, Hkv, N, d);
  auto at = [&](int w) -> void* {
    return sage_buffer_bytes(mode, w, B, heads_of(w, H, Hkv), N, d) ? base + L.off[w] : nullptr;
  };
  QuantQKArgs qa{q, k, dtype, mode, B, H, N, d, Hkv,
                 at(SAGE_BUF_Q_CODES), (float*)at(SAGE_BUF_Q_SCALES), at(SAGE_BUF_Q_SF),
                 at(SAGE_BUF_K_CODES), (float*)at(SAGE_BUF_K_SCALES), at(SAGE_BUF_K_SF),
                 (float*)at(SAGE_BUF_K_MEAN), reinterpret_cast<double*>(base + L.ksum), cnt};
  QuantVArgs va{v, dtype, mode, B, Hkv, N, d,
                at(SAGE_BUF_V_CODES), (float*)at(SAGE_BUF_V_SCALES), at(SAGE_BUF_V_SF),
                reinterpret_cast<double*>(base + L.ksum),
                reinterpret_cast<float*>(base + L.vmax), cnt};
  qa.status = status;
  if (smooth) {
    qa.q_mean = reinterpret_cast<float*>(base + L.qmean);
    qa.ds = reinterpret_cast<float*>(base + L.ds);
  }
  SAGE_TRY(prepass_forked(qa, va, st));
  AttnArgs aa{mode, at(SAGE_BUF_Q_CODES), (float*)at(SAGE_BUF_Q_SCALES), at(SAGE_BUF_Q_SF),
              at(SAGE_BUF_K_CODES), (float*)at(SAGE_BUF_K_SCALES), at(SAGE_BUF_K_SF),
              at(SAGE_BUF_V_CODES), (float*)at(SAGE_BUF_V_SCALES), at(SAGE_BUF_V_SF),
              o, dtype, B, H, N, d, Hkv, causal != 0, sm_scale, status};
  aa.ds = qa.ds;
  const char* detail = nullptr;
  const cudaError_t e =
      mode == SAGE_MODE_FP4 ? launch_attn_fp4(aa, st, &detail) : launch_attn_i8f8(aa, st, &detail);
  if (detail) return fail(SAGE_ERR_CUDA, detail);
  if (e != cudaSuccess) return fail_cuda(e, "attention launch");
  return SAGE_OK;
}

// The whole pipeline (pre-pass, then attention) with every buffer carved
// from the per-stream workspace. Q and O have H heads, K and V have Hkv heads
// (Hkv divides H; Hkv == H is plain multi-head attention).
int attn_fwd_full(const void* q, const void* k, const void* v, void* o, int dtype, int64_t B,
                  int64_t H, int64_t Hkv, int64_t N, int64_t d, int causal, float sm_scale,
                  int mode, sage_stream_t stream) {
  const bool smooth = (mode & SAGE_FLAG_SMOOTH_Q) != 0;
  mode &= ~SAGE_FLAG_SMOOTH_Q;
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_kv_heads(H, Hkv));
  SAGE_TRY(check_ptr(q, "q", true));
  SAGE_TRY(check_ptr(k, "k", true));
  SAGE_TRY(check_ptr(v, "v", true));
  SAGE_TRY(check_ptr(o, "o", true));
  if (!(sm_scale > 0.f)) sm_scale = 1.0f / std::sqrt((float)d);
  if (!std::isfinite(sm_scale)) return fail(SAGE_ERR_INVALID_ARG, "sm_scale must be finite");
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  uint32_t* cnt = nullptr;
  SAGE_TRY(workspace(st, fwd_layout(mode, smooth, B, H, Hkv, N, d).total, &ws, &cnt));
  return run_fwd(q, k, v, o, dtype, B, H, Hkv, N, d, causal, sm_scale, mode, smooth,
                 static_cast<char*>(ws), cnt, di->status, st);
}

// Two more streams per device for sage_attn_fwd_host: host -> device copies
// of a chunk's Q, K, V and device -> host copies of its O, each ordered
// against the compute on the caller's stream by events (two slots of staging
// buffers, so chunk i + 1 is copied in and chunk i - 1 copied out while
// chunk i computes).
struct CopyStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t in_ready[2] = {nullptr, nullptr}, done[2] = {nullptr, nullptr},
              out_read[2] = {nullptr, nullptr};
  std::mutex mu;  // one pipelined call at a time per device: the events are shared
};
std::map<int, CopyStreams*> g_copy;

int copy_streams(CopyStreams** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  CopyStreams*& cs = g_copy[dev];
  if (!cs) {
    auto* n = new CopyStreams;
    e = cudaStreamCreateWithFlags(&n->h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&n->d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n->start, cudaEventDisableTiming);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&n->in_ready[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n->done[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n->out_read[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
      delete n;
      return fail_cuda(e, "copy stream setup");
    }
    cs = n;
  }
  *out = cs;
  return SAGE_OK;
}

// Heads per chunk of sage_attn_fwd_host: about 16 chunks, none smaller than
// 32 MB of inputs (fewer, larger chunks for small problems).  The copy in of
// the first chunk and the compute and copy out of the last are not
// overlapped, so more chunks shorten the pass while each still fills the GPU.
int64_t host_chunk_heads(int64_t BH, int64_t N, int64_t d) {
  const int64_t head_bytes = 3 * N * d * 2;
  int64_t c = (BH + 15) / 16;
  const int64_t min_heads = (int64_t(32) << 20) / (head_bytes > 0 ? head_bytes : 1);
  if (c < min_heads) c = min_heads;
  if (c > BH) c = BH;
  return c < 1 ? 1 : c;
}

}  // namespace

extern "C" {

size_t sage_buffer_bytes(int mode, int which, int64_t B, int64_t H, int64_t N, int64_t d) {
  if (B < 0 || H < 0 || N < 0 || d < 0) return 0;
  const int64_t BH = B * H;
  const int64_t nt = (N + 127) / 128;
  const bool fp4 = mode == SAGE_MODE_FP4;
  switch (which) {
    case SAGE_BUF_Q_CODES:
    case SAGE_BUF_K_CODES:
    case SAGE_BUF_V_CODES:
      // padded to whole 128-token tiles (the padding holds zero codes)
      return (size_t)(fp4 ? BH * nt * 128 * d / 2 : BH * nt * 128 * d);
    case SAGE_BUF_Q_SCALES:
      // 8-bit modes: one scale per token; FP4: one tile scale per 128 tokens
      return (size_t)(fp4 ? BH * nt * 4 : BH * nt * 128 * 4);
    case SAGE_BUF_K_SCALES:
      // 8-bit modes: one scale per 32 tokens; FP4: one tile scale per 128
      return (size_t)(fp4 ? BH * nt * 4 : BH * nt * 4 * 4);
    case SAGE_BUF_Q_SF:
    case SAGE_BUF_K_SF:
      return fp4 ? (size_t)(BH * nt * ((d + 63) / 64) * 512) : 0;
    case SAGE_BUF_K_MEAN:
      return (size_t)(BH * d * 4);
    case SAGE_BUF_V_SCALES:
      return (size_t)(fp4 ? BH * nt * 4 : BH * d * 4);
    case SAGE_BUF_V_SF:
      return fp4 ? (size_t)(BH * nt * 2 * 512) : 0;
    case SAGE_BUF_Q_MEAN:
      return (size_t)(BH * nt * d * 4);
    case SAGE_BUF_DS:
      return (size_t)(BH * nt * nt * 128 * 4);
    default:
      return 0;
  }
}

int sage_quant_qk(const void* q, const void* k, int dtype, int64_t B, int64_t H, int64_t N,
                  int64_t d, int mode, void* q_codes, float* q_scales, void* q_sf, void* k_codes,
                  float* k_scales, void* k_sf, float* k_mean, sage_stream_t stream) {
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_ptr(q, "q", true));
  SAGE_TRY(check_ptr(k, "k", true));
  SAGE_TRY(check_ptr(q_codes, "q_codes", true));
  SAGE_TRY(check_ptr(q_scales, "q_scales", true));
  SAGE_TRY(check_ptr(k_codes, "k_codes", true));
  SAGE_TRY(check_ptr(k_scales, "k_scales", true));
  SAGE_TRY(check_ptr(k_mean, "k_mean", true));
  if (mode == SAGE_MODE_FP4) {
    SAGE_TRY(check_ptr(q_sf, "q_sf", true));
    SAGE_TRY(check_ptr(k_sf, "k_sf", true));
  } else {
    SAGE_TRY(check_unused(q_sf, "q_sf"));
    SAGE_TRY(check_unused(k_sf, "k_sf"));
  }
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  uint32_t* cnt = nullptr;
  SAGE_TRY(workspace(st, ws_ksum_bytes(B * H, N, d), &ws, &cnt));
  QuantQKArgs a{q, k, dtype, mode, B, H, N, d, H, q_codes, q_scales, q_sf,
                k_codes, k_scales, k_sf, k_mean, static_cast<double*>(ws), cnt};
  cudaError_t e = launch_quant_qk(a, st);
  if (e != cudaSuccess) return fail_cuda(e, "quant_qk launch");
  return SAGE_OK;
}

int sage_quant_qk_smooth(const void* q, const void* k, int dtype, int64_t B, int64_t H, int64_t N,
                         int64_t d, int mode, void* q_codes, float* q_scales, void* q_sf,
                         void* k_codes, float* k_scales, void* k_sf, float* k_mean, float* q_mean,
                         float* ds, sage_stream_t stream) {
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_ptr(q, "q", true));
  SAGE_TRY(check_ptr(k, "k", true));
  SAGE_TRY(check_ptr(q_codes, "q_codes", true));
  SAGE_TRY(check_ptr(q_scales, "q_scales", true));
  SAGE_TRY(check_ptr(k_codes, "k_codes", true));
  SAGE_TRY(check_ptr(k_scales, "k_scales", true));
  SAGE_TRY(check_ptr(k_mean, "k_mean", true));
  SAGE_TRY(check_ptr(q_mean, "q_mean", true));
  SAGE_TRY(check_ptr(ds, "ds", true));
  if (mode == SAGE_MODE_FP4) {
    SAGE_TRY(check_ptr(q_sf, "q_sf", true));
    SAGE_TRY(check_ptr(k_sf, "k_sf", true));
  } else {
    SAGE_TRY(check_unused(q_sf, "q_sf"));
    SAGE_TRY(check_unused(k_sf, "k_sf"));
  }
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  uint32_t* cnt = nullptr;
  SAGE_TRY(workspace(st, ws_ksum_bytes(B * H, N, d), &ws, &cnt));
  QuantQKArgs a{q, k, dtype, mode, B, H, N, d, H, q_codes, q_scales, q_sf,
                k_codes, k_scales, k_sf, k_mean, static_cast<double*>(ws), cnt};
  a.q_mean = q_mean;
  a.ds = ds;
  cudaError_t e = launch_quant_qk(a, st);
  if (e != cudaSuccess) return fail_cuda(e, "quant_qk_smooth launch");
  return SAGE_OK;
}

int sage_quant_v(const void* v, int dtype, int64_t B, int64_t H, int64_t N, int64_t d, int mode,
                 void* v_codes, float* v_scales, void* v_sf, sage_stream_t stream) {
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_ptr(v, "v", true));
  SAGE_TRY(check_ptr(v_codes, "v_codes", true));
  SAGE_TRY(check_ptr(v_scales, "v_scales", true));
  if (mode == SAGE_MODE_FP4) SAGE_TRY(check_ptr(v_sf, "v_sf", true));
  else SAGE_TRY(check_unused(v_sf, "v_sf"));
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  uint32_t* cnt = nullptr;
  const size_t ks = align_up(ws_ksum_bytes(B * H, N, d));
  if (mode != SAGE_MODE_FP4)
    SAGE_TRY(workspace(st, ks + ws_vmax_bytes(B * H, N, d), &ws, &cnt));
  QuantVArgs a{v, dtype, mode, B, H, N, d, v_codes, v_scales, v_sf,
               static_cast<double*>(ws),
               ws ? reinterpret_cast<float*>(static_cast<char*>(ws) + ks) : nullptr, cnt};
  cudaError_t e = launch_quant_v(a, st);
  if (e != cudaSuccess) return fail_cuda(e, "quant_v launch");
  return SAGE_OK;
}

int sage_quant_qkv(const void* q, const void* k, const void* v, int dtype, int64_t B, int64_t H,
                   int64_t N, int64_t d, int mode, void* q_codes, float* q_scales, void* q_sf,
                   void* k_codes, float* k_scales, void* k_sf, float* k_mean, void* v_codes,
                   float* v_scales, void* v_sf, sage_stream_t stream) {
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_ptr(q, "q", true));
  SAGE_TRY(check_ptr(k, "k", true));
  SAGE_TRY(check_ptr(v, "v", true));
  SAGE_TRY(check_ptr(q_codes, "q_codes", true));
  SAGE_TRY(check_ptr(q_scales, "q_scales", true));
  SAGE_TRY(check_ptr(k_codes, "k_codes", true));
  SAGE_TRY(check_ptr(k_scales, "k_scales", true));
  SAGE_TRY(check_ptr(k_mean, "k_mean", true));
  SAGE_TRY(check_ptr(v_codes, "v_codes", true));
  SAGE_TRY(check_ptr(v_scales, "v_scales", true));
  if (mode == SAGE_MODE_FP4) {
    SAGE_TRY(check_ptr(q_sf, "q_sf", true));
    SAGE_TRY(check_ptr(k_sf, "k_sf", true));
    SAGE_TRY(check_ptr(v_sf, "v_sf", true));
  } else {
    SAGE_TRY(check_unused(q_sf, "q_sf"));
    SAGE_TRY(check_unused(k_sf, "k_sf"));
    SAGE_TRY(check_unused(v_sf, "v_sf"));
  }
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  uint32_t* cnt = nullptr;
  const size_t ks = align_up(ws_ksum_bytes(B * H, N, d));
  SAGE_TRY(workspace(st, ks + ws_vmax_bytes(B * H, N, d), &ws, &cnt));
  QuantQKArgs qa{q, k, dtype, mode, B, H, N, d, H, q_codes, q_scales, q_sf,
                 k_codes, k_scales, k_sf, k_mean, static_cast<double*>(ws), cnt};
  QuantVArgs va{v, dtype, mode, B, H, N, d, v_codes, v_scales, v_sf,
                static_cast<double*>(ws), reinterpret_cast<float*>(static_cast<char*>(ws) + ks),
                cnt};
  qa.status = di->status;
  return prepass_forked(qa, va, st);
}

int sage_attn_fwd_quantized(int mode, const void* q_codes, const float* q_scales, const void* q_sf,
                            const void* k_codes, const float* k_scales, const void* k_sf,
                            const void* v_codes, const float* v_scales, const void* v_sf, void* o,
                            int dtype, int64_t B, int64_t H, int64_t N, int64_t d, int causal,
                            float sm_scale, sage_stream_t stream) {
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_ptr(q_codes, "q_codes", true));
  SAGE_TRY(check_ptr(q_scales, "q_scales", true));
  SAGE_TRY(check_ptr(k_codes, "k_codes", true));
  SAGE_TRY(check_ptr(k_scales, "k_scales", true));
  SAGE_TRY(check_ptr(v_codes, "v_codes", true));
  SAGE_TRY(check_ptr(v_scales, "v_scales", true));
  SAGE_TRY(check_ptr(o, "o", true));
  if (mode == SAGE_MODE_FP4) {
    SAGE_TRY(check_ptr(q_sf, "q_sf", true));
    SAGE_TRY(check_ptr(k_sf, "k_sf", true));
    SAGE_TRY(check_ptr(v_sf, "v_sf", true));
  } else {
    SAGE_TRY(check_unused(q_sf, "q_sf"));
    SAGE_TRY(check_unused(k_sf, "k_sf"));
    SAGE_TRY(check_unused(v_sf, "v_sf"));
  }
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale))
    return fail(SAGE_ERR_INVALID_ARG, "sm_scale must be positive and finite");
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  AttnArgs a{mode, q_codes, q_scales, q_sf, k_codes, k_scales, k_sf, v_codes, v_scales, v_sf,
             o, dtype, B, H, N, d, H, causal != 0, sm_scale, di->status};
  const char* detail = nullptr;
  cudaError_t e = mode == SAGE_MODE_FP4 ? launch_attn_fp4(a, st, &detail)
                                        : launch_attn_i8f8(a, st, &detail);
  if (detail) return fail(SAGE_ERR_CUDA, detail);
  if (e != cudaSuccess) return fail_cuda(e, "attention launch");
  return SAGE_OK;
}

int sage_attn_fwd_quantized_smooth(int mode, const void* q_codes, const float* q_scales,
                                   const void* q_sf, const void* k_codes, const float* k_scales,
                                   const void* k_sf, const void* v_codes, const float* v_scales,
                                   const void* v_sf, const float* ds, void* o, int dtype,
                                   int64_t B, int64_t H, int64_t N, int64_t d, int causal,
                                   float sm_scale, sage_stream_t stream) {
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_ptr(q_codes, "q_codes", true));
  SAGE_TRY(check_ptr(q_scales, "q_scales", true));
  SAGE_TRY(check_ptr(k_codes, "k_codes", true));
  SAGE_TRY(check_ptr(k_scales, "k_scales", true));
  SAGE_TRY(check_ptr(v_codes, "v_codes", true));
  SAGE_TRY(check_ptr(v_scales, "v_scales", true));
  SAGE_TRY(check_ptr(ds, "ds", true));
  SAGE_TRY(check_ptr(o, "o", true));
  if (mode == SAGE_MODE_FP4) {
    SAGE_TRY(check_ptr(q_sf, "q_sf", true));
    SAGE_TRY(check_ptr(k_sf, "k_sf", true));
    SAGE_TRY(check_ptr(v_sf, "v_sf", true));
  } else {
    SAGE_TRY(check_unused(q_sf, "q_sf"));
    SAGE_TRY(check_unused(k_sf, "k_sf"));
    SAGE_TRY(check_unused(v_sf, "v_sf"));
  }
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale))
    return fail(SAGE_ERR_INVALID_ARG, "sm_scale must be positive and finite");
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  AttnArgs a{mode, q_codes, q_scales, q_sf, k_codes, k_scales, k_sf, v_codes, v_scales,
             v_sf, o, dtype, B, H, N, d, H, causal != 0, sm_scale, di->status};
  a.ds = ds;
  const char* detail = nullptr;
  cudaError_t e = mode == SAGE_MODE_FP4 ? launch_attn_fp4(a, st, &detail)
                                        : launch_attn_i8f8(a, st, &detail);
  if (detail) return fail(SAGE_ERR_CUDA, detail);
  if (e != cudaSuccess) return fail_cuda(e, "attention launch");
  return SAGE_OK;
}

int sage_attn_fwd_host(const void* q, const void* k, const void* v, void* o, int dtype,
                       int64_t B, int64_t H, int64_t N, int64_t d, int causal, float sm_scale,
                       int mode, sage_stream_t stream) {
  const bool smooth = (mode & SAGE_FLAG_SMOOTH_Q) != 0;
  const int base_mode = mode & ~SAGE_FLAG_SMOOTH_Q;
  bool empty = false;
  SAGE_TRY(check_common(dtype, base_mode, B, H, N, d, &empty));
  if (!q || !k || !v || !o) return fail(SAGE_ERR_INVALID_ARG, "q, k, v and o must not be NULL");
  if (!(sm_scale > 0.f)) sm_scale = 1.0f / std::sqrt((float)d);
  if (!std::isfinite(sm_scale)) return fail(SAGE_ERR_INVALID_ARG, "sm_scale must be finite");
  if (empty) return SAGE_OK;
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t BH = B * H;
  const int64_t ch = host_chunk_heads(BH, N, d);
  const size_t head_bytes = (size_t)(N * d * 2);
  const size_t in_bytes = align_up(head_bytes * ch);   // one tensor of a chunk
  // staging: two slots of Q, K, V and O; then the chunk pipeline's workspace
  const size_t stage = 2 * 4 * in_bytes;
  void* ws = nullptr;
  uint32_t* cnt = nullptr;
  SAGE_TRY(workspace(st, stage + fwd_layout(base_mode, smooth, 1, ch, ch, N, d).total, &ws, &cnt));
  char* base = static_cast<char*>(ws);
  auto slot = [&](int s, int t) { return base + (size_t)(4 * s + t) * in_bytes; };  // t: q k v o
  CopyStreams* cs = nullptr;
  SAGE_TRY(copy_streams(&cs));
  std::lock_guard<std::mutex> lk(cs->mu);
  cudaError_t e;
  // the copy streams start after everything already queued on st (the
  // workspace may have been in use there)
  if ((e = cudaEventRecord(cs->start, st)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(cs->h2d, cs->start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(cs->d2h, cs->start, 0)) != cudaSuccess)
    return fail_cuda(e, "host pipeline fork");
  const char* hq = static_cast<const char*>(q);
  const char* hk = static_cast<const char*>(k);
  const char* hv = static_cast<const char*>(v);
  char* ho = static_cast<char*>(o);
  int status = SAGE_OK;
  const int64_t nchunks = (BH + ch - 1) / ch;
  for (int64_t i = 0; i < nchunks && status == SAGE_OK; ++i) {
    const int s = (int)(i & 1);
    const int64_t h0 = i * ch, nh = (BH - h0 < ch) ? BH - h0 : ch;
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)nh * head_bytes;
    // copy in (slot s is free once chunk i - 2 has computed)
    if ((i >= 2 && (e = cudaStreamWaitEvent(cs->h2d, cs->done[s], 0)) != cudaSuccess) ||
        (e = cudaMemcpyAsync(slot(s, 0), hq + off, bytes, cudaMemcpyDefault, cs->h2d)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(slot(s, 1), hk + off, bytes, cudaMemcpyDefault, cs->h2d)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(slot(s, 2), hv + off, bytes, cudaMemcpyDefault, cs->h2d)) !=
            cudaSuccess ||
        (e = cudaEventRecord(cs->in_ready[s], cs->h2d)) != cudaSuccess) {
      status = fail_cuda(e, "host pipeline copy in");
      break;
    }
    // compute (O slot s is free once chunk i - 2 has been copied out)
    if ((e = cudaStreamWaitEvent(st, cs->in_ready[s], 0)) != cudaSuccess ||
        (i >= 2 && (e = cudaStreamWaitEvent(st, cs->out_read[s], 0)) != cudaSuccess)) {
      status = fail_cuda(e, "host pipeline order");
      break;
    }
    status = run_fwd(slot(s, 0), slot(s, 1), slot(s, 2), slot(s, 3), dtype, 1, nh, nh, N, d,
                     causal, sm_scale, base_mode, smooth, base + stage, cnt, di->status, st);
    if (status != SAGE_OK) break;
    if ((e = cudaEventRecord(cs->done[s], st)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(cs->d2h, cs->done[s], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(ho + off, slot(s, 3), bytes, cudaMemcpyDefault, cs->d2h)) !=
            cudaSuccess ||
        (e = cudaEventRecord(cs->out_read[s], cs->d2h)) != cudaSuccess) {
      status = fail_cuda(e, "host pipeline copy out");
      break;
    }
  }
  // st continues after every copy of this call (also when a step failed)
  for (cudaStream_t cpy : {cs->h2d, cs->d2h}) {
    if ((e = cudaEventRecord(cs->start, cpy)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(st, cs->start, 0)) != cudaSuccess)
      return status != SAGE_OK ? status : fail_cuda(e, "host pipeline join");
  }
  return status;
}

int sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int dtype, int64_t B,
                  int64_t H, int64_t N, int64_t d, int causal, float sm_scale, int mode,
                  sage_stream_t stream) {
  return attn_fwd_full(q, k, v, o, dtype, B, H, H, N, d, causal, sm_scale, mode, stream);
}

int sage_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, int dtype, int64_t B,
                      int64_t H, int64_t Hkv, int64_t N, int64_t d, int causal, float sm_scale,
                      int mode, sage_stream_t stream) {
  return attn_fwd_full(q, k, v, o, dtype, B, H, Hkv, N, d, causal, sm_scale, mode, stream);
}

int sage_get_last_device_status(void) {
  DeviceInfo* di = nullptr;
  int s = device_info(&di);
  if (s != SAGE_OK) return s;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceSynchronize");
  uint32_t v = 0;
  e = cudaMemcpy(&v, di->status, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e, "read status");
  const uint32_t zero = 0;
  e = cudaMemcpy(di->status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail_cuda(e, "clear status");
  if (v == 0) return SAGE_OK;
  char bits[96];
  std::snprintf(bits, sizeof bits, "a bounded wait expired in a kernel (status bits 0x%x)", v);
  return fail(SAGE_ERR_DEVICE_TIMEOUT, bits);
}

int sage_selftest_bounded_wait(sage_stream_t stream) {
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  sage::wait_selftest_kernel<<<1, 32, 0, st>>>(di->status);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail_cuda(e, "self-test launch");
  return SAGE_OK;
}

const char* sage_status_string(int status) {
  static thread_local std::string s;
  const char* base = "unknown status";
  switch (status) {
    case SAGE_OK: base = "ok"; break;
    case SAGE_ERR_INVALID_ARG: base = "invalid argument"; break;
    case SAGE_ERR_UNSUPPORTED: base = "unsupported"; break;
    case SAGE_ERR_CUDA: base = "CUDA error"; break;
    case SAGE_ERR_DEVICE_TIMEOUT: base = "device wait timed out"; break;
    default: break;
  }
  s = base;
  if (status != SAGE_OK && status == t_last_status && !t_last_detail.empty())
    s += ": " + t_last_detail;
  return s.c_str();
}

const char* sage_version(void) { return "sage-b200 0.1 (sm_100a)"; }

int sage_debug_fail_allocations(int count) {
  if (count < 0) return fail(SAGE_ERR_INVALID_ARG, "count must be >= 0");
  std::lock_guard<std::mutex> lk(g_mu);
  g_fail_allocs = count;
  return SAGE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation variant of sage_attn_fwd.
//
// Some callers cannot allocate device memory at call time: code running
// under a memory-pool policy that forbids new allocations, allocators that
// own every byte of the device, or real-time callers that may not take the
// driver's allocation locks.  For them the whole forward pass can run out of
// one fixed scratch area that is part of the library's device image: a
// file-scope array of kNoAllocScratchBytes, reserved on every GPU that loads
// the library and held until the process exits.
// ---------------------------------------------------------------------------

namespace sage {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device with that
// device current (in host code the array's name is only a host-side stand-in,
// never a device address).
std::map<int, void*> g_noalloc_addr;

// One-time set-up per device: the array's device address, and the side
// stream (with its fork/join events) that the two-launch pre-pass uses, so
// that no later call of any shape creates a CUDA object.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_noalloc_addr.find(dev);
    if (it != g_noalloc_addr.end()) {
      *out = it->second;
      return SAGE_OK;
    }
  }
  SideStream* ss = nullptr;
  SAGE_TRY(side_stream(&ss));
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(no-allocation scratch)");
  std::lock_guard<std::mutex> lk(g_mu);
  g_noalloc_addr[dev] = p;
  *out = p;
  return SAGE_OK;
}

}  // namespace
}  // namespace sage

static_assert(sage::kNoAllocScratchBytes == SAGE_NOALLOC_SCRATCH_BYTES,
              "the header states the scratch size");

extern "C" {

int sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, int dtype,
                          int64_t B, int64_t H, int64_t N, int64_t d, int causal, float sm_scale,
                          int mode, sage_stream_t stream) {
  bool empty = false;
  SAGE_TRY(check_common(dtype, mode, B, H, N, d, &empty));
  SAGE_TRY(check_ptr(q, "q", true));
  SAGE_TRY(check_ptr(k, "k", true));
  SAGE_TRY(check_ptr(v, "v", true));
  SAGE_TRY(check_ptr(o, "o", true));
  if (!(sm_scale > 0.f)) sm_scale = 1.0f / std::sqrt((float)d);
  if (!std::isfinite(sm_scale)) return fail(SAGE_ERR_INVALID_ARG, "sm_scale must be finite");
  if (empty) return SAGE_OK;
  // scratch layout: every quantized buffer, then the statistics partials
  size_t off[SAGE_BUF_V_SF + 1];
  size_t total = 0;
  for (int w = 0; w <= SAGE_BUF_V_SF; ++w) {
    off[w] = total;
    total += align_up(sage_buffer_bytes(mode, w, B, H, N, d));
  }
  const size_t off_ksum = total;
  total += align_up(ws_ksum_bytes(B * H, N, d));
  const size_t off_vmax = total;
  total += align_up(ws_vmax_bytes(B * H, N, d));
  total += kStatsCounterBytes;  // the per-head statistics counters, first
  if (total > kNoAllocScratchBytes) {
    return fail(SAGE_ERR_UNSUPPORTED,
                "this shape needs " + std::to_string(total) +
                    " bytes of scratch; the no-allocation entry point has " +
                    std::to_string(kNoAllocScratchBytes) + " (use sage_attn_fwd)");
  }
  DeviceInfo* di = nullptr;
  SAGE_TRY(device_info(&di));
  void* ws = nullptr;
  SAGE_TRY(noalloc_scratch(&ws));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* cnt = static_cast<uint32_t*>(ws);
  char* base = static_cast<char*>(ws) + kStatsCounterBytes;
  auto at = [&](int w) -> void* {
    return sage_buffer_bytes(mode, w, B, H, N, d) ? base + off[w] : nullptr;
  };
  // Every scratch byte the kernels read is written earlier in the same call
  // (codes, scales, statistics partials), except the per-head counters of
  // the statistics pass.  A pre-pass leaves them at zero, but a call that
  // overlapped another one on the GPU may not have: clear the counters of
  // the heads in use (K, then V) first, in stream order, so that one such
  // race cannot spoil the calls after it.
  cudaError_t e = cudaMemsetAsync(cnt, 0, (size_t)(B * H) * sizeof(uint32_t), st);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(cnt + kMaxStatHeads, 0, (size_t)(B * H) * sizeof(uint32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(no-allocation counters)");
  QuantQKArgs qa{q, k, dtype, mode, B, H, N, d, H,
                 at(SAGE_BUF_Q_CODES), (float*)at(SAGE_BUF_Q_SCALES), at(SAGE_BUF_Q_SF),
                 at(SAGE_BUF_K_CODES), (float*)at(SAGE_BUF_K_SCALES), at(SAGE_BUF_K_SF),
                 (float*)at(SAGE_BUF_K_MEAN), reinterpret_cast<double*>(base + off_ksum), cnt};
  QuantVArgs va{v, dtype, mode, B, H, N, d,
                at(SAGE_BUF_V_CODES), (float*)at(SAGE_BUF_V_SCALES), at(SAGE_BUF_V_SF),
                reinterpret_cast<double*>(base + off_ksum),
                reinterpret_cast<float*>(base + off_vmax), cnt};
  qa.status = di->status;
  SAGE_TRY(prepass_forked(qa, va, st));
  AttnArgs aa{mode, at(SAGE_BUF_Q_CODES), (float*)at(SAGE_BUF_Q_SCALES), at(SAGE_BUF_Q_SF),
              at(SAGE_BUF_K_CODES), (float*)at(SAGE_BUF_K_SCALES), at(SAGE_BUF_K_SF),
              at(SAGE_BUF_V_CODES), (float*)at(SAGE_BUF_V_SCALES), at(SAGE_BUF_V_SF),
              o, dtype, B, H, N, d, H, causal != 0, sm_scale, di->status};
  const char* detail = nullptr;
  e = mode == SAGE_MODE_FP4 ? launch_attn_fp4(aa, st, &detail) : launch_attn_i8f8(aa, st, &detail);
  if (detail) return fail(SAGE_ERR_CUDA, detail);
  if (e != cudaSuccess) return fail_cuda(e, "attention launch");
  return SAGE_OK;
}

}  // extern "C"
