// ubench.cu -- measurement kernels behind the design choices of the
// attention kernels (libsage_ubench.so, include/sage_ubench.h):
//   - tcgen05 MMA throughput per kind (8-bit, and block-scaled FP4),
//     accumulator type and tile width N
//     (is an FP16 accumulator faster than FP32 for FP8 P~V, as the
//     SageAttention2++ page reports for its GPUs; how much narrower is an
//     N = 128 tile than N = 256);
//   - SFU exponential throughput, FP32 against packed FP16x2;
//   - the FMA-pipe 2^t of the attention kernels on given arguments (for an
//     accuracy check against an exact exponential).
// One CTA per SM; every wait is bounded (a timeout sets a flag the host
// reads and returns as an error).  No other code of the library uses this.

#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/sage_ubench.h"
#include "exp2_poly.cuh"
#include "sage_ptx.cuh"

namespace sage {
namespace {

// M = 128, N = 128 or 256; K = 32 for the 8-bit kinds (32 bytes of K per
// row), 64 for block-scaled FP4 (E2M1 operands, one UE4M3 scale per 16
// elements of K, the scales in TMEM); operands and scales zero (the rate
// does not depend on the values).
template <int KIND>
constexpr int kUbenchK = KIND == SAGE_UBENCH_NVF4 ? 64 : 32;
template <int KIND, int N>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int iters, uint32_t* flag) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t slot;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  // A: 128 rows, B: N rows, 128 bytes each (128-byte swizzle atoms)
  for (int i = threadIdx.x; i < (128 + N) * 128 / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem)[i] = 0u;
  fence_proxy_async_smem();
  // the accumulator in columns 0 .. N-1; FP4 scale factors of A from
  // column kColSfA, of B from kColSfB
  constexpr uint32_t kColSfA = 384, kColSfB = 416;
  if (warp == 0) {
    tmem_alloc(&slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = slot;
  if (KIND == SAGE_UBENCH_NVF4) {
    // zero scale factors: each warp its 32 lanes of columns 384 .. 447
    const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;
#pragma unroll
    for (int c = 0; c < 64; c += 8) tmem_st8(tmem + lanes + kColSfA + (uint32_t)c, z);
    tmem_wait_st();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0 && elect_one()) {
    constexpr uint32_t idesc = KIND == SAGE_UBENCH_F8_F32 ? make_idesc(1, 0, 0, 128, N)
                             : KIND == SAGE_UBENCH_F8_F16 ? make_idesc(0, 0, 0, 128, N)
                             : KIND == SAGE_UBENCH_NVF4   ? make_idesc_nvf4(128, N)
                                                          : make_idesc(2, 1, 1, 128, N);
    // 8-bit kinds: 128-byte rows, 128-byte swizzle; FP4: 64-byte rows
    // (128 E2M1 elements, two K steps), 64-byte swizzle, first K step
    const uint64_t a = KIND == SAGE_UBENCH_NVF4
                           ? make_sdesc(smem_u32(smem), 8 * 64, 16, Swz::k64)
                           : make_sdesc(smem_u32(smem), 1024, 16, Swz::k128);
    const uint64_t b = KIND == SAGE_UBENCH_NVF4
                           ? make_sdesc(smem_u32(smem + 128 * 128), 8 * 64, 16, Swz::k64)
                           : make_sdesc(smem_u32(smem + 128 * 128), 1024, 16, Swz::k128);
    for (int i = 0; i < iters; ++i) {
      if (KIND == SAGE_UBENCH_I8_S32) mma_i8_ss(tmem, a, b, idesc, i > 0);
      else if (KIND == SAGE_UBENCH_NVF4)
        mma_nvf4_ss(tmem, a, b, idesc, tmem + kColSfA, tmem + kColSfB, i > 0);
      else mma_f8_ss(tmem, a, b, idesc, i > 0);
    }
    mma_commit(&bar);
    volatile int no_abort = 0;
    mbar_wait(&bar, 0, &no_abort, flag, 1u);  // an expired wait sets *flag
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// 8 independent exponentials per thread and round, each fed by the
// previous round (y = 2^(y - 1) converges to 1): FP32 ex2, or packed
// FP16x2 ex2 (two values per instruction).
template <int MODE>
__global__ void exp_rate_kernel(int iters, float* sink, long long* cycles) {
  const long long t0 = clock64();
  float acc = 0.f;
  if (MODE == SAGE_UBENCH_EXP_F32) {
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = 1.0f + 0.001f * (float)(threadIdx.x + i);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float r;
        asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y[i] - 1.0f));
        y[i] = r;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc += y[i];
  } else {
    uint32_t y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = 0x3C003C00u;  // (1, 1) in f16x2
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t d, r;
        asm volatile("sub.f16x2 %0, %1, %2;" : "=r"(d) : "r"(y[i]), "r"(0x3C003C00u));
        asm volatile("ex2.approx.f16x2 %0, %1;" : "=r"(r) : "r"(d));
        y[i] = r;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc += (float)(y[i] & 0xFFFFu);
  }
  const long long t1 = clock64();
  sink[blockIdx.x * blockDim.x + threadIdx.x] = acc;
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// FP64 FMA throughput: 8 independent chains per thread (the Q smoothing
// bias kernel's arithmetic); cycles as in exp_rate_kernel.
__global__ void dfma_rate_kernel(int iters, double* sink, long long* cycles) {
  const long long t0 = clock64();
  double y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = 1e-3 * (double)(threadIdx.x + i);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fma_rn(y[i], 1.0000001, 1e-9);
  }
  double acc = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) acc += y[i];
  const long long t1 = clock64();
  sink[blockIdx.x * blockDim.x + threadIdx.x] = acc;
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// The attention kernels' FMA-pipe 2^t (exp2_poly.cuh) on given arguments,
// two per thread through the packed path, so the host can check it against
// an exact exponential.
__global__ void exp2_poly_kernel(const float* t, float* out, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = exp2_poly2(make_float2(t[i], i + 1 < n ? t[i + 1] : 0.f));
  out[i] = v.x;
  if (i + 1 < n) out[i + 1] = v.y;
}

int sms_of_device(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? 0 : -1;
}

template <int KIND, int N>
int run_mma(int iters, int reps, double* tops) {
  int sms = 0;
  if (sms_of_device(&sms) != 0) return SAGE_UBENCH_ERR_CUDA;
  auto k = mma_rate_kernel<KIND, N>;
  const int smem = (128 + N) * 128 + 1024;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SAGE_UBENCH_ERR_CUDA;
  uint32_t* flag = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  int status = SAGE_UBENCH_ERR_CUDA;
  float ms = 0.f;
  if (cudaMalloc(&flag, 4) != cudaSuccess) return SAGE_UBENCH_ERR_CUDA;
  if (cudaMemset(flag, 0, 4) == cudaSuccess && cudaEventCreate(&e0) == cudaSuccess &&
      cudaEventCreate(&e1) == cudaSuccess) {
    k<<<sms, 128, smem>>>(iters, flag);  // warm-up
    cudaEventRecord(e0);
    for (int r = 0; r < reps; ++r) k<<<sms, 128, smem>>>(iters, flag);
    cudaEventRecord(e1);
    uint32_t h = 0;
    if (cudaEventSynchronize(e1) == cudaSuccess && cudaEventElapsedTime(&ms, e0, e1) == cudaSuccess &&
        cudaMemcpy(&h, flag, 4, cudaMemcpyDeviceToHost) == cudaSuccess)
      status = h ? SAGE_UBENCH_ERR_TIMEOUT : SAGE_UBENCH_OK;
  }
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  cudaFree(flag);
  if (status == SAGE_UBENCH_OK)
    *tops = 2.0 * 128 * N * kUbenchK<KIND> * (double)iters * sms * reps / (ms * 1e-3) / 1e12;
  return status;
}

template <int MODE>
int run_exp(int threads, int iters, double* per_clk) {
  int sms = 0;
  if (sms_of_device(&sms) != 0) return SAGE_UBENCH_ERR_CUDA;
  float* sink = nullptr;
  long long* cyc = nullptr;
  int status = SAGE_UBENCH_ERR_CUDA;
  if (cudaMalloc(&sink, (size_t)sms * threads * 4) == cudaSuccess &&
      cudaMalloc(&cyc, (size_t)sms * 8) == cudaSuccess) {
    exp_rate_kernel<MODE><<<sms, threads>>>(iters, sink, cyc);  // warm-up
    exp_rate_kernel<MODE><<<sms, threads>>>(iters, sink, cyc);
    long long* h = new long long[sms];
    if (cudaMemcpy(h, cyc, (size_t)sms * 8, cudaMemcpyDeviceToHost) == cudaSuccess) {
      double c = 0;
      for (int i = 0; i < sms; ++i) c += (double)h[i];
      c /= sms;
      const double values = (double)threads * 8 * iters * (MODE == SAGE_UBENCH_EXP_F32 ? 1 : 2);
      *per_clk = values / c;
      status = SAGE_UBENCH_OK;
    }
    delete[] h;
  }
  cudaFree(sink);
  cudaFree(cyc);
  return status;
}

int run_dfma(int threads, int iters, double* per_clk) {
  int sms = 0;
  if (sms_of_device(&sms) != 0) return SAGE_UBENCH_ERR_CUDA;
  double* sink = nullptr;
  long long* cyc = nullptr;
  int status = SAGE_UBENCH_ERR_CUDA;
  if (cudaMalloc(&sink, (size_t)sms * threads * 8) == cudaSuccess &&
      cudaMalloc(&cyc, (size_t)sms * 8) == cudaSuccess) {
    dfma_rate_kernel<<<sms, threads>>>(iters, sink, cyc);  // warm-up
    dfma_rate_kernel<<<sms, threads>>>(iters, sink, cyc);
    long long* h = new long long[sms];
    if (cudaMemcpy(h, cyc, (size_t)sms * 8, cudaMemcpyDeviceToHost) == cudaSuccess) {
      double c = 0;
      for (int i = 0; i < sms; ++i) c += (double)h[i];
      c /= sms;
      *per_clk = (double)threads * 8 * iters / c;
      status = SAGE_UBENCH_OK;
    }
    delete[] h;
  }
  cudaFree(sink);
  cudaFree(cyc);
  return status;
}

}  // namespace
}  // namespace sage

extern "C" {

int sage_ubench_dfma(int threads, int iters, double* per_clk_per_sm) {
  using namespace sage;
  if (!per_clk_per_sm || iters <= 0 || threads <= 0 || threads > 1024 || threads % 32)
    return SAGE_UBENCH_ERR_ARG;
  return run_dfma(threads, iters, per_clk_per_sm);
}

int sage_ubench_mma(int kind, int n, int iters, int reps, double* tops) {
  using namespace sage;
  if (!tops || iters <= 0 || reps <= 0 || (n != 128 && n != 256)) return SAGE_UBENCH_ERR_ARG;
  switch (kind) {
    case SAGE_UBENCH_F8_F32:
      return n == 128 ? run_mma<SAGE_UBENCH_F8_F32, 128>(iters, reps, tops)
                      : run_mma<SAGE_UBENCH_F8_F32, 256>(iters, reps, tops);
    case SAGE_UBENCH_F8_F16:
      return n == 128 ? run_mma<SAGE_UBENCH_F8_F16, 128>(iters, reps, tops)
                      : run_mma<SAGE_UBENCH_F8_F16, 256>(iters, reps, tops);
    case SAGE_UBENCH_I8_S32:
      return n == 128 ? run_mma<SAGE_UBENCH_I8_S32, 128>(iters, reps, tops)
                      : run_mma<SAGE_UBENCH_I8_S32, 256>(iters, reps, tops);
    case SAGE_UBENCH_NVF4:
      return n == 128 ? run_mma<SAGE_UBENCH_NVF4, 128>(iters, reps, tops)
                      : run_mma<SAGE_UBENCH_NVF4, 256>(iters, reps, tops);
    default:
      return SAGE_UBENCH_ERR_ARG;
  }
}

int sage_ubench_exp2_poly(const float* t, float* out, int n) {
  using namespace sage;
  if (!t || !out || n <= 0) return SAGE_UBENCH_ERR_ARG;
  float* dt = nullptr;
  float* dout = nullptr;
  int status = SAGE_UBENCH_ERR_CUDA;
  const size_t bytes = (size_t)n * 4;
  if (cudaMalloc(&dt, bytes) == cudaSuccess && cudaMalloc(&dout, bytes) == cudaSuccess &&
      cudaMemcpy(dt, t, bytes, cudaMemcpyHostToDevice) == cudaSuccess) {
    const int pairs = (n + 1) / 2;
    exp2_poly_kernel<<<(pairs + 255) / 256, 256>>>(dt, dout, n);
    if (cudaGetLastError() == cudaSuccess &&
        cudaMemcpy(out, dout, bytes, cudaMemcpyDeviceToHost) == cudaSuccess)
      status = SAGE_UBENCH_OK;
  }
  cudaFree(dt);
  cudaFree(dout);
  return status;
}

int sage_ubench_exp(int mode, int threads, int iters, double* per_clk_per_sm) {
  using namespace sage;
  if (!per_clk_per_sm || iters <= 0 || threads <= 0 || threads > 1024 || threads % 32)
    return SAGE_UBENCH_ERR_ARG;
  if (mode == SAGE_UBENCH_EXP_F32) return run_exp<SAGE_UBENCH_EXP_F32>(threads, iters, per_clk_per_sm);
  if (mode == SAGE_UBENCH_EXP_F16X2)
    return run_exp<SAGE_UBENCH_EXP_F16X2>(threads, iters, per_clk_per_sm);
  return SAGE_UBENCH_ERR_ARG;
}

}  // extern "C"
