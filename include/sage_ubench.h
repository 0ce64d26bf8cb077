/*
 * sage_ubench.h -- C ABI of libsage_ubench.so: the microbenchmarks behind
 * the design of the attention kernels.  Not part of the attention path (no
 * counterpart on the pages); bench.py --ubench prints their results.
 *
 * All calls run on the current CUDA device, synchronise it, allocate and
 * free their own small buffers, and return SAGE_UBENCH_OK or a negative
 * status.  Every device wait is bounded.
 */
#ifndef SAGE_UBENCH_H
#define SAGE_UBENCH_H

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SAGE_UBENCH_OK = 0,
  SAGE_UBENCH_ERR_ARG = -1,      /* bad argument                         */
  SAGE_UBENCH_ERR_CUDA = -3,     /* a CUDA call failed                   */
  SAGE_UBENCH_ERR_TIMEOUT = -4   /* a bounded wait in the kernel expired */
};

/* tcgen05.mma kinds measured by sage_ubench_mma. */
enum {
  SAGE_UBENCH_F8_F32 = 0,  /* kind::f8f6f4, e4m3 x e4m3, FP32 accumulator */
  SAGE_UBENCH_F8_F16 = 1,  /* kind::f8f6f4, e4m3 x e4m3, FP16 accumulator */
  SAGE_UBENCH_I8_S32 = 2,  /* kind::i8, s8 x s8, INT32 accumulator        */
  SAGE_UBENCH_NVF4 = 3     /* kind::mxf4nvf4.block_scale.block16, e2m1 x
                              e2m1 with UE4M3 scales per 16 elements of K
                              (in TMEM), FP32 accumulator                  */
};

/* Exponential variants measured by sage_ubench_exp. */
enum { SAGE_UBENCH_EXP_F32 = 0, SAGE_UBENCH_EXP_F16X2 = 1 };

/* Dense MMA throughput: one CTA per SM issues `iters` MMAs of M = 128,
 * N = n (128 or 256), K = 32 (K = 64 for SAGE_UBENCH_NVF4) from shared
 * memory onto one TMEM accumulator, `reps` launches timed with CUDA
 * events.  *tops receives 2 M N K iters SMs reps / time, in 10^12
 * operations per second.  The SageAttention2++
 * page reports an FP8 MMA with FP16 accumulation twice as fast as with
 * FP32 on its GPUs; this measures the same question on this one. */
int sage_ubench_mma(int kind, int n, int iters, int reps, double* tops);

/* Exponential throughput: one CTA of `threads` threads per SM, each with 8
 * independent chains of `iters` rounds; *per_clk_per_sm receives the
 * exponentials (values, two per FP16x2 instruction) per SM clock cycle. */
int sage_ubench_exp(int mode, int threads, int iters, double* per_clk_per_sm);

/* FP64 FMA throughput: one CTA of `threads` threads per SM, each with 8
 * independent chains of `iters` FMAs; *per_clk_per_sm receives the FP64
 * FMAs per SM clock cycle.  The denominator of the Q smoothing bias
 * kernel, which sums q-bar . k' in FP64 (sage.h, sage_quant_qk_smooth). */
int sage_ubench_dfma(int threads, int iters, double* per_clk_per_sm);
/* The attention kernels' FMA-pipe exponential (a degree-4 polynomial after
 * a rint split, on the packed FP32 pipe) evaluated on the device at the n
 * host values t[i] (t <= 128; arguments below -125 are clamped there), the
 * results copied to out[i], so that a test can hold it to its stated
 * relative error (2^-18.5) against an exact exponential. */
int sage_ubench_exp2_poly(const float* t, float* out, int n);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_UBENCH_H */
