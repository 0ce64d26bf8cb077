/*
 * sage.h -- C ABI of the B200 (sm_100a) quantized attention forward pass.
 *
 * The library computes O = softmax(Q K^T * sm_scale) V the SageAttention
 * way:
 *   - K is smoothed by subtracting its per-channel mean over tokens
 *     (SageAttention abstract, dblp author page on taxoreview.com: accurate
 *     8-bit attention; softmax is unchanged by a per-row shift);
 *   - Q and K are quantized per block of tokens to INT8 or FP8
 *     ("Flash Attention vs Sage Attention: Kernel Comparison", section "How
 *     SageAttention uses quantization for more throughput") -- one scale
 *     per query token and one per 32 keys, the granularity of the kernel's
 *     threads (SageAttention2 abstract: "hardware-friendly thread-level
 *     granularity") -- or to FP4 with one UE4M3 scale per 16 elements
 *     (SageAttention3 abstract: FP4 tensor cores of Blackwell GPUs);
 *   - Q K^T runs on the tensor cores and is dequantized by the product of
 *     the scales;
 *   - an online (flash-style) softmax follows (kernel-comparison blog,
 *     section "How FlashAttention reduces memory traffic");
 *   - the unnormalised P~ and V are quantized to FP8 (SageAttention2
 *     abstract) or FP4, and P~V accumulates in two levels: a fresh FP32
 *     partial per 128-key tile folded into an FP32 running accumulator
 *     (SageAttention2 abstract: "two-level accumulation strategy").
 *
 * Conventions shared by every entry point
 *   - Tensors are row-major and contiguous.  Q, K, V, O are [B, H, N, d] in
 *     the input dtype (fp16 or bf16).
 *   - All pointers are DEVICE pointers of the current CUDA device, owned by
 *     the caller, and must be 16-byte aligned.  `stream` is a cudaStream_t
 *     (NULL = legacy default stream).  Every call is asynchronous on
 *     `stream`; the library never synchronises it.
 *   - Supported shapes: d in {64, 128} (FP4 mode: d == 128); any N >= 0.
 *     A call with B, H or N equal to zero does nothing and returns SAGE_OK.
 *   - Ragged sequences: every code buffer is laid out for Np = N rounded
 *     up to a multiple of 128 (the rows or columns of the missing tokens
 *     hold zero codes); the last quantization block (32 K tokens, a 128-token
 *     tile in FP4 mode) may be partial and its scale covers the real tokens
 *     only; a block of missing tokens has scale 0; keys past N are masked
 *     out of the softmax.
 *   - Return value: SAGE_OK (0) or a negative sage_status_t.  No exception
 *     or process exit crosses the ABI.  sage_status_string() describes the
 *     most recent error of the calling thread.
 *   - Quantized buffers (sizes from sage_buffer_bytes):
 *       INT8/FP8 and FP8 modes
 *         q_codes, k_codes  int8 (FP8 mode: e4m3) [B, H, Np, d]
 *         q_scales          float [B, H, Np]        one scale per token
 *         k_scales          float [B, H, Np/32]     one scale per 32 tokens
 *         k_mean            float [B, H, d]
 *         v_codes           e4m3  [B, H, d, Np]     V transposed
 *         v_scales          float [B, H, d]         one scale per channel
 *       FP4 mode
 *         q_codes, k_codes  e2m1x2 [B, H, Np, d/2]  low nibble = even channel
 *         q_scales, k_scales float [B, H, Np/128]   tile scale g
 *         q_sf, k_sf        ue4m3 per 16 channels, tensor-core layout (below)
 *         v_codes           e2m1x2 [B, H, d, Np/2]  V transposed, low nibble =
 *                                                    even token
 *         v_scales          float [B, H, Np/128]    tile scale g
 *         v_sf              ue4m3 per 16 tokens, tensor-core layout (below)
 *       Tensor-core scale layout: for each (b, h, 128-token tile t, 64-wide
 *       chunk c of the contraction axis) one 512-byte block; inside it byte
 *       16*l + 4*j + s holds the scale of row 32*j + l (row = token for
 *       Q/K, channel for V; rows >= d are zero) and 16-element group
 *       4*c + s.  Blocks are ordered (b, h, t, c).
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                         /* == cudaStream_t */
typedef struct CUstream_st* sage_stream_t;

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = -1,     /* null pointer, negative size, bad enum   */
  SAGE_ERR_UNSUPPORTED = -2,     /* shape/alignment/device not supported    */
  SAGE_ERR_CUDA = -3,            /* a CUDA runtime/driver call failed       */
  SAGE_ERR_DEVICE_TIMEOUT = -4   /* a bounded wait inside a kernel expired  */
} sage_status_t;

/* INT8_FP8: INT8 Q/K, FP8 P~ and V.  FP4: FP4 Q/K/P~/V.  FP8: FP8 Q/K
 * (e4m3, block scale amax/448 with the INT8 mode's blocks), FP8 P~ and V;
 * its Q K^T accumulates in FP32 on the tensor cores instead of exactly in
 * INT32. */
typedef enum { SAGE_MODE_INT8_FP8 = 0, SAGE_MODE_FP4 = 1, SAGE_MODE_FP8 = 2 } sage_mode_t;
typedef enum { SAGE_DTYPE_F16 = 0, SAGE_DTYPE_BF16 = 1 } sage_dtype_t;

typedef enum {
  SAGE_BUF_Q_CODES = 0, SAGE_BUF_Q_SCALES, SAGE_BUF_Q_SF,
  SAGE_BUF_K_CODES, SAGE_BUF_K_SCALES, SAGE_BUF_K_SF, SAGE_BUF_K_MEAN,
  SAGE_BUF_V_CODES, SAGE_BUF_V_SCALES, SAGE_BUF_V_SF,
  /* Q smoothing: the per-block Q means, FP32 [B, H, ceil(N/128), d], and
   * the score bias, FP32 [B, H, ceil(N/128), 128 ceil(N/128)] */
  SAGE_BUF_Q_MEAN, SAGE_BUF_DS
} sage_buffer_t;

/* OR'ed into the mode of sage_attn_fwd / sage_attn_fwd_gqa: Q smoothing
 * (SageAttention2 abstract, "we propose a method to smooth Q"; see
 * sage_quant_qk_smooth), in every mode. */
#define SAGE_FLAG_SMOOTH_Q 0x100

/* Bytes of one quantized buffer for the given mode and shape (0 for a
 * buffer the mode does not use, e.g. *_SF outside FP4 mode). */
size_t sage_buffer_bytes(int mode, int which, int64_t B, int64_t H, int64_t N, int64_t d);

/* Q/K pre-pass: K channel mean (FP64 accumulation: per 128-token chunk in
 * token order, then over chunks; mean = fp32(sum / N)), K smoothing
 * (one FP32 subtraction), then block quantization of Q (8-bit modes: one
 * scale per token) and of smoothed K (8-bit modes: one scale per 32
 * tokens), amax taken over the block's tokens and all d channels.
 *   INT8 mode: s = fp32(amax / 127); code = clamp(rne(fp32(x / s)), +-127);
 *              q_sf, k_sf must be NULL.
 *   FP8 mode:  s = fp32(amax / 448); code = e4m3(fp32(x / s)); q_sf, k_sf
 *              must be NULL.
 *   FP4 mode:  g = fp32(amax_tile / 2688); per 16 channels
 *              s16 = ue4m3(fp32(amax16 / fp32(6 g))),
 *              code = e2m1(fp32(x / fp32(s16 * g))); q_scales/k_scales
 *              receive g.
 * All divisions are IEEE FP32 divisions; all casts round to nearest-even
 * and saturate.  Codes and scales are bit-identical to the CPU oracle.
 * Uses a stream-ordered library workspace for the mean partial sums. */
int sage_quant_qk(const void* q, const void* k, int dtype,
                  int64_t B, int64_t H, int64_t N, int64_t d, int mode,
                  void* q_codes, float* q_scales, void* q_sf,
                  void* k_codes, float* k_scales, void* k_sf,
                  float* k_mean, sage_stream_t stream);

/* The Q/K pre-pass with Q smoothing, in every mode.  Before Q is quantized,
 * each (b, h) and 128-token block of queries loses its mean:
 *   qbar = fp32(FP64 sum of the block's tokens in token order / count)
 *   (the last block of a ragged sequence: its own tokens), written to
 *   q_mean [B, H, ceil(N/128), d];
 *   Q' = fp32(Q) - qbar (one FP32 subtraction) is quantized as Q is in
 *   sage_quant_qk.
 * What qbar takes out comes back as a bias on the block's scores,
 *   ds[b, h, blk, j] = fp32( sum over c in order of qbar[blk, c] *
 *                           (fp32(K[j, c]) - k_mean[c]) ),
 * the sum in FP64 (every product exact), written to
 * ds [B, H, ceil(N/128), 128 ceil(N/128)] (keys past N hold 0); it costs
 * B H N^2 d / 128 FP64 multiply-adds.  K, its mean and its codes are as in
 * sage_quant_qk.  Everything is bit-identical to the CPU oracle.  Buffer
 * sizes: sage_buffer_bytes with SAGE_BUF_Q_MEAN and SAGE_BUF_DS. */
int sage_quant_qk_smooth(const void* q, const void* k, int dtype,
                         int64_t B, int64_t H, int64_t N, int64_t d, int mode,
                         void* q_codes, float* q_scales, void* q_sf,
                         void* k_codes, float* k_scales, void* k_sf,
                         float* k_mean, float* q_mean, float* ds, sage_stream_t stream);

/* V pre-pass.
 *   INT8_FP8 and FP8 modes: s_V[c] = fp32(amax_c / 448) over all N tokens
 *             of the (b, h);
 *             code = e4m3(fp32(V / s_V)); written transposed; v_sf NULL.
 *   FP4 mode: per 128-token tile g = fp32(amax_tile / 2688); per channel
 *             and 16 tokens s16 = ue4m3(fp32(amax16 / fp32(6 g))),
 *             code = e2m1(fp32(V / fp32(s16 * g))); v_scales receive g.
 * (SageAttention2 abstract: V to FP8; SageAttention3 abstract: FP4.) */
int sage_quant_v(const void* v, int dtype,
                 int64_t B, int64_t H, int64_t N, int64_t d, int mode,
                 void* v_codes, float* v_scales, void* v_sf, sage_stream_t stream);

/* The Q/K and V pre-passes in one call, with the arguments of both (Q, K
 * and V share B, H, N, d).  Results are those of the two separate calls, bit
 * for bit.  Two launch forms:
 *   - 8-bit modes with N <= 1024 and B * H <= 16: one launch on `stream`
 *     (clusters of 8 CTAs per head and tensor hold the head in shared memory
 *     and reduce the K mean and V scales across the cluster).  Its wait for
 *     the input copy is bounded: if it expires, the codes are not valid and
 *     sage_get_last_device_status reports SAGE_ERR_DEVICE_TIMEOUT.
 *   - otherwise the two pre-passes are independent: the V pre-pass runs on
 *     a library-owned second stream, forked from `stream` and joined back to
 *     it with events (stream capture records the fork and the join), so the
 *     two overlap on the GPU.  That second stream is one per device, shared
 *     by every caller stream: callers on different streams that reach this
 *     point at the same time have their V pre-passes serialised on it (the
 *     results are unaffected; only the overlap between them is lost). */
int sage_quant_qkv(const void* q, const void* k, const void* v, int dtype,
                   int64_t B, int64_t H, int64_t N, int64_t d, int mode,
                   void* q_codes, float* q_scales, void* q_sf,
                   void* k_codes, float* k_scales, void* k_sf, float* k_mean,
                   void* v_codes, float* v_scales, void* v_sf, sage_stream_t stream);

/* Attention on already-quantized operands (the buffers written by the two
 * pre-pass calls); writes O [B, H, N, d] in `dtype`.  causal != 0 applies
 * the top-left-aligned causal mask (query t sees keys 0..t).  sm_scale is
 * applied at dequantization, not folded into the stored scales.
 * P~ is quantized inside the kernel: INT8_FP8 and FP8 modes e4m3(448 P~);
 * FP4 mode per 16 keys s16 = ue4m3(448 amax16), code = e2m1(2688 P~ / s16). */
int sage_attn_fwd_quantized(int mode,
                            const void* q_codes, const float* q_scales, const void* q_sf,
                            const void* k_codes, const float* k_scales, const void* k_sf,
                            const void* v_codes, const float* v_scales, const void* v_sf,
                            void* o, int dtype,
                            int64_t B, int64_t H, int64_t N, int64_t d,
                            int causal, float sm_scale, sage_stream_t stream);

/* Attention with Q smoothing on the buffers of sage_quant_qk_smooth and
 * sage_quant_v: every score of query block blk and key j is dequantized as
 * in sage_attn_fwd_quantized and gains ds[b, h, blk, j] sm_scale before the
 * online softmax.  Other arguments and errors as in
 * sage_attn_fwd_quantized. */
int sage_attn_fwd_quantized_smooth(int mode,
                                   const void* q_codes, const float* q_scales, const void* q_sf,
                                   const void* k_codes, const float* k_scales, const void* k_sf,
                                   const void* v_codes, const float* v_scales, const void* v_sf,
                                   const float* ds, void* o, int dtype,
                                   int64_t B, int64_t H, int64_t N, int64_t d,
                                   int causal, float sm_scale, sage_stream_t stream);

/* The whole forward pass: pre-pass into a library-owned workspace (grown
 * on demand with stream-ordered allocation, one per (device, stream),
 * freed at unload; the pre-pass takes the launch forms of sage_quant_qkv),
 * then the attention kernel.  sm_scale <= 0 means 1/sqrt(d).  An allocation
 * failure returns SAGE_ERR_CUDA before any kernel is launched.  mode may
 * carry SAGE_FLAG_SMOOTH_Q: the pre-pass is then that of
 * sage_quant_qk_smooth (chained form only) and the attention that of
 * sage_attn_fwd_quantized_smooth. */
int sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int dtype,
                  int64_t B, int64_t H, int64_t N, int64_t d,
                  int causal, float sm_scale, int mode, sage_stream_t stream);

/* The whole forward pass on HOST buffers: q, k, v and o point to host
 * memory holding [B, H, N, d] in `dtype` (any host memory; page-locked
 * memory lets the copies overlap the compute).  The heads are cut into
 * about 16 chunks (none smaller than 32 MB of inputs); chunk i + 1 is copied
 * in and chunk i - 1 copied out on two library-owned copy streams (one pair
 * per device, shared by callers, one call at a time) while chunk i runs the
 * pre-pass and attention of sage_attn_fwd on `stream`.  Heads are
 * independent, so O equals sage_attn_fwd's bit for bit.  Every copy of the
 * call is ordered before later work on `stream`: synchronise `stream`
 * before reading o.  mode may carry SAGE_FLAG_SMOOTH_Q.  Device memory
 * comes from the same per-(device, stream) workspace as sage_attn_fwd (two
 * chunks of Q, K, V and O plus one chunk's pipeline); errors as in
 * sage_attn_fwd (a NULL pointer is SAGE_ERR_INVALID_ARG). */
int sage_attn_fwd_host(const void* q, const void* k, const void* v, void* o, int dtype,
                       int64_t B, int64_t H, int64_t N, int64_t d,
                       int causal, float sm_scale, int mode, sage_stream_t stream);

/* Grouped-query (and multi-query) attention: the kernel-comparison blog
 * ("Attention kernel benchmarks: speed and memory use") notes that
 * grouped-query attention changes the shape of the K/V tensors being
 * quantized.  Here Q and O are [B, H, N, d] while K and V are
 * [B, Hkv, N, d]; query head h reads key/value head h / (H / Hkv).
 * Hkv must divide H (Hkv == 1 is multi-query attention; Hkv == H is
 * exactly sage_attn_fwd).  K is smoothed and K and V are quantized once
 * per key/value head, so the result equals sage_attn_fwd on K and V
 * repeated across each group of H / Hkv query heads, bit for bit.  Other
 * arguments, the workspace and the errors are those of sage_attn_fwd; a
 * bad Hkv is SAGE_ERR_INVALID_ARG. */
int sage_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, int dtype,
                      int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                      int causal, float sm_scale, int mode, sage_stream_t stream);

/* The same forward pass for callers that cannot allocate device memory
 * while they run (a memory pool that admits no new allocations, an
 * allocator that owns the whole device, a caller that may not take the
 * driver's allocation locks).  The paper has no counterpart: this is a
 * deployment variant of sage_attn_fwd.
 *
 * All scratch (codes, scales, statistics partials) lives in one fixed
 * array of SAGE_NOALLOC_SCRATCH_BYTES inside the library's device image,
 * reserved on every GPU that loads the library and held until the process
 * exits; the call itself allocates and frees nothing.  The caller still
 * passes Q, K, V and O as with sage_attn_fwd (same arguments, same result).
 *   - A shape whose scratch exceeds the array is rejected with
 *     SAGE_ERR_UNSUPPORTED and a message giving both sizes (about 3.1 bytes
 *     per element of Q in INT8/FP8 mode: B*H*N*d up to about 21 million).
 *   - The first call on a device does its one-time set-up with that device
 *     current: it looks up the array's device address and creates the
 *     library's second stream (and two events) that the pre-pass forks onto
 *     for long sequences.  Make that first call, of any shape, before any
 *     stream capture; later calls create nothing.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind: calls whose GPU work overlaps (different streams, or threads)
 *     race on it and must be serialised by the caller.  Each call clears the
 *     statistics counters it uses (a stream-ordered memset, which allocates
 *     nothing) before its pre-pass, so an overlap spoils only the calls that
 *     overlapped.
 *   - The second stream is shared by every caller stream of a device: two
 *     callers that run this pre-pass at once on different streams have their
 *     V chains serialised (results are unaffected). */
/* (mode as in sage_attn_fwd, without SAGE_FLAG_SMOOTH_Q: a mode carrying
 * it is SAGE_ERR_INVALID_ARG here.) */
#define SAGE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
int sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, int dtype,
                          int64_t B, int64_t H, int64_t N, int64_t d,
                          int causal, float sm_scale, int mode, sage_stream_t stream);

/* Reads and clears the device status word written by the kernels' bounded
 * waits: SAGE_OK when no wait expired since the last call, else
 * SAGE_ERR_DEVICE_TIMEOUT (sage_status_string then gives the status bits).
 * Synchronises the current device. */
int sage_get_last_device_status(void);

/* Self-test of the kernels' bounded waits: launches a kernel whose
 * mbarrier wait can never complete.  The wait gives up after about one
 * second and records a timeout in the device status word (read it with
 * sage_get_last_device_status); the kernel exits normally and the context
 * stays usable.  No counterpart on the pages: a failure-detection check. */
int sage_selftest_bounded_wait(sage_stream_t stream);

/* Failure injection for tests: the next `count` workspace allocations (the
 * stream-ordered growth of the workspace of sage_attn_fwd, sage_attn_fwd_gqa
 * and the pre-pass calls) fail as if the allocation call had failed, without
 * making it: the entry point returns SAGE_ERR_CUDA with a message naming the
 * injected failure and launches nothing, and the workspace stays
 * unallocated, so a later call allocates it again.  count = 0 clears the
 * injection; a negative count is SAGE_ERR_INVALID_ARG.  No counterpart on
 * the pages: a failure-detection check made on the host. */
int sage_debug_fail_allocations(int count);

/* Human-readable text of a status, with the detail of the calling thread's
 * most recent error when `status` is that error. */
const char* sage_status_string(int status);

/* Library version string. */
const char* sage_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H */
