"""Python binding of libsage_b200.so (SageAttention-style quantized attention
forward for B200 / sm_100a).

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step of the computation runs in the library's
CUDA kernels.  There is no CPU fallback -- if the shared library is missing
or cannot be loaded, every call raises.

Entry points (same names as the C ABI in include/sage.h):

    sage_quant_qk(q, k, mode="int8_fp8")      -> dict of code/scale tensors
    sage_quant_v(v, mode="int8_fp8")          -> dict of code/scale tensors
    sage_quant_qkv(q, k, v, mode="int8_fp8")  -> (Q/K dict, V dict), the two overlapped
    sage_attn_fwd_quantized(qk, vq, mode, causal, sm_scale, out_dtype) -> O
    sage_attn_fwd(q, k, v, causal=False, sm_scale=None, mode="int8_fp8") -> O
    sage_attn_fwd_gqa(q, k, v, ...)           -> O  (K/V with fewer heads than Q)
    sage_quant_qk_smooth(q, k, mode)          -> dict, with Q smoothing (q_mean, ds)
    sage_attn_fwd_quantized_smooth(qk, vq, shape, mode, ...) -> O, with Q smoothing
    (sage_attn_fwd(..., smooth_q=True) runs the whole pass with Q smoothing)
    sage_attn_fwd_host(q, k, v, ...)          -> O  (host tensors in and out, copies overlapped)
"""

import ctypes
import math
import os

__all__ = ["sage_quant_qk", "sage_quant_v", "sage_quant_qkv", "sage_attn_fwd", "sage_attn_fwd_gqa",
           "sage_attn_fwd_quantized", "sage_attn_fwd_noalloc",
           "sage_quant_qk_smooth", "sage_attn_fwd_quantized_smooth", "SMOOTH_Q", "sage_attn_fwd_host",
           "buffer_bytes", "library", "library_path", "SageError", "MODES", "EXPORTS",
           "selftest_bounded_wait"]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libsage_b200.so")

MODES = {"int8_fp8": 0, "fp4": 1, "fp8": 2}
SMOOTH_Q = 0x100  # SAGE_FLAG_SMOOTH_Q, OR'ed into the mode of sage_attn_fwd
DTYPES = {"f16": 0, "bf16": 1}
BUF = {name: i for i, name in enumerate(
    ["q_codes", "q_scales", "q_sf", "k_codes", "k_scales", "k_sf", "k_mean",
     "v_codes", "v_scales", "v_sf", "q_mean", "ds"])}

# every symbol include/sage.h declares
EXPORTS = ["sage_buffer_bytes", "sage_quant_qk", "sage_quant_v", "sage_quant_qkv",
           "sage_attn_fwd_quantized", "sage_quant_qk_smooth", "sage_attn_fwd_quantized_smooth",
           "sage_attn_fwd", "sage_attn_fwd_gqa", "sage_attn_fwd_noalloc", "sage_attn_fwd_host",
           "sage_get_last_device_status",
           "sage_selftest_bounded_wait", "sage_status_string", "sage_version",
           "sage_debug_fail_allocations"]

_lib = None


class SageError(RuntimeError):
    def __init__(self, status, text):
        super().__init__(f"sage status {status}: {text}")
        self.status = status


def library():
    """The loaded ctypes library (loads it on first use; raises if missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(
            f"{library_path} is missing: build it with "
            "`python -m quantized_attention_quant_b200.build` (there is no fallback path)")
    lib = ctypes.CDLL(library_path)
    i64, vp, fp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
    lib.sage_buffer_bytes.restype = ctypes.c_size_t
    lib.sage_buffer_bytes.argtypes = [i32, i32, i64, i64, i64, i64]
    lib.sage_quant_qk.restype = i32
    lib.sage_quant_qk.argtypes = [vp, vp, i32, i64, i64, i64, i64, i32,
                                  vp, fp, vp, vp, fp, vp, fp, vp]
    lib.sage_quant_qk_smooth.restype = i32
    lib.sage_quant_qk_smooth.argtypes = [vp, vp, i32, i64, i64, i64, i64, i32,
                                         vp, fp, vp, vp, fp, vp, fp, fp, fp, vp]
    lib.sage_attn_fwd_quantized_smooth.restype = i32
    lib.sage_attn_fwd_quantized_smooth.argtypes = [i32, vp, fp, vp, vp, fp, vp, vp, fp, vp, fp,
                                                   vp, i32, i64, i64, i64, i64, i32,
                                                   ctypes.c_float, vp]
    lib.sage_quant_v.restype = i32
    lib.sage_quant_v.argtypes = [vp, i32, i64, i64, i64, i64, i32, vp, fp, vp, vp]
    lib.sage_quant_qkv.restype = i32
    lib.sage_quant_qkv.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i32,
                                   vp, fp, vp, vp, fp, vp, fp, vp, fp, vp, vp]
    lib.sage_attn_fwd_quantized.restype = i32
    lib.sage_attn_fwd_quantized.argtypes = [i32, vp, fp, vp, vp, fp, vp, vp, fp, vp, vp, i32,
                                            i64, i64, i64, i64, i32, ctypes.c_float, vp]
    lib.sage_attn_fwd.restype = i32
    lib.sage_attn_fwd.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i32,
                                  ctypes.c_float, i32, vp]
    lib.sage_attn_fwd_gqa.restype = i32
    lib.sage_attn_fwd_gqa.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, i32,
                                      ctypes.c_float, i32, vp]
    lib.sage_attn_fwd_host.restype = i32
    lib.sage_attn_fwd_host.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i32,
                                       ctypes.c_float, i32, vp]
    lib.sage_attn_fwd_noalloc.restype = i32
    lib.sage_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i32,
                                          ctypes.c_float, i32, vp]
    lib.sage_get_last_device_status.restype = i32
    lib.sage_get_last_device_status.argtypes = []
    lib.sage_selftest_bounded_wait.restype = i32
    lib.sage_selftest_bounded_wait.argtypes = [vp]
    lib.sage_status_string.restype = ctypes.c_char_p
    lib.sage_status_string.argtypes = [i32]
    lib.sage_version.restype = ctypes.c_char_p
    lib.sage_version.argtypes = []
    lib.sage_debug_fail_allocations.restype = i32
    lib.sage_debug_fail_allocations.argtypes = [i32]
    _lib = lib
    return lib


def _check(status):
    if status != 0:
        raise SageError(status, library().sage_status_string(status).decode())


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return DTYPES["bf16"]
    if t.dtype == torch.float16:
        return DTYPES["f16"]
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or f16)")


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _shape(x):
    if x.dim() != 4 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor of shape [B, H, N, d]")
    return tuple(int(s) for s in x.shape)


def buffer_bytes(mode, which, B, H, N, d):
    return int(library().sage_buffer_bytes(MODES[mode], BUF[which], B, H, N, d))


def _alloc(mode, names, B, H, N, d, device):
    import torch
    out = {}
    for n in names:
        nbytes = buffer_bytes(mode, n, B, H, N, d)
        out[n] = torch.empty(nbytes, dtype=torch.uint8, device=device) if nbytes else None
    return out


def _f(t):
    return None if t is None else t.data_ptr()


def sage_quant_qk(q, k, mode="int8_fp8"):
    """Q/K pre-pass.  Returns {q_codes, q_scales, q_sf, k_codes, k_scales, k_sf,
    k_mean} as raw uint8 tensors laid out as include/sage.h describes."""
    B, H, N, d = _shape(q)
    if _shape(k) != (B, H, N, d) or k.dtype != q.dtype:
        raise ValueError("q and k must have the same shape and dtype")
    bufs = _alloc(mode, ["q_codes", "q_scales", "q_sf", "k_codes", "k_scales", "k_sf", "k_mean"],
                  B, H, N, d, q.device)
    _check(library().sage_quant_qk(
        _ptr(q), _ptr(k), _dtype_code(q), B, H, N, d, MODES[mode],
        _f(bufs["q_codes"]), _f(bufs["q_scales"]), _f(bufs["q_sf"]),
        _f(bufs["k_codes"]), _f(bufs["k_scales"]), _f(bufs["k_sf"]), _f(bufs["k_mean"]),
        _stream()))
    return bufs


def sage_quant_qk_smooth(q, k, mode="int8_fp8"):
    """Q/K pre-pass with Q smoothing.  Returns {q_codes, q_scales, q_sf,
    k_codes, k_scales, k_sf, k_mean, q_mean, ds} as raw uint8 tensors laid
    out as include/sage.h describes."""
    B, H, N, d = _shape(q)
    if _shape(k) != (B, H, N, d) or k.dtype != q.dtype:
        raise ValueError("q and k must have the same shape and dtype")
    bufs = _alloc(mode, ["q_codes", "q_scales", "q_sf", "k_codes", "k_scales", "k_sf", "k_mean",
                         "q_mean", "ds"], B, H, N, d, q.device)
    _check(library().sage_quant_qk_smooth(
        _ptr(q), _ptr(k), _dtype_code(q), B, H, N, d, MODES[mode],
        _f(bufs["q_codes"]), _f(bufs["q_scales"]), _f(bufs["q_sf"]),
        _f(bufs["k_codes"]), _f(bufs["k_scales"]), _f(bufs["k_sf"]),
        _f(bufs["k_mean"]), _f(bufs["q_mean"]), _f(bufs["ds"]), _stream()))
    return bufs


def sage_quant_v(v, mode="int8_fp8"):
    """V pre-pass.  Returns {v_codes, v_scales, v_sf} as raw uint8 tensors."""
    B, H, N, d = _shape(v)
    bufs = _alloc(mode, ["v_codes", "v_scales", "v_sf"], B, H, N, d, v.device)
    _check(library().sage_quant_v(
        _ptr(v), _dtype_code(v), B, H, N, d, MODES[mode],
        _f(bufs["v_codes"]), _f(bufs["v_scales"]), _f(bufs["v_sf"]), _stream()))
    return bufs


def sage_quant_qkv(q, k, v, mode="int8_fp8"):
    """Both pre-passes in one call: one cluster-fused launch for short heads
    in the 8-bit modes, else the V pass overlapped with the Q/K pass on a
    library stream.  Returns (qk, vq) as sage_quant_qk and sage_quant_v do,
    bit for bit."""
    B, H, N, d = _shape(q)
    if _shape(k) != (B, H, N, d) or _shape(v) != (B, H, N, d):
        raise ValueError("q, k, v must have the same shape")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must have the same dtype")
    qk = _alloc(mode, ["q_codes", "q_scales", "q_sf", "k_codes", "k_scales", "k_sf", "k_mean"],
                B, H, N, d, q.device)
    vq = _alloc(mode, ["v_codes", "v_scales", "v_sf"], B, H, N, d, v.device)
    _check(library().sage_quant_qkv(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, H, N, d, MODES[mode],
        _f(qk["q_codes"]), _f(qk["q_scales"]), _f(qk["q_sf"]),
        _f(qk["k_codes"]), _f(qk["k_scales"]), _f(qk["k_sf"]), _f(qk["k_mean"]),
        _f(vq["v_codes"]), _f(vq["v_scales"]), _f(vq["v_sf"]), _stream()))
    return qk, vq


def sage_attn_fwd_quantized(qk, vq, shape, mode="int8_fp8", causal=False, sm_scale=None,
                            out_dtype=None, out=None):
    """Attention on pre-quantized operands (the dicts returned above)."""
    import torch
    B, H, N, d = shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype or torch.bfloat16,
                          device=qk["q_codes"].device)
    _check(library().sage_attn_fwd_quantized(
        MODES[mode], _f(qk["q_codes"]), _f(qk["q_scales"]), _f(qk["q_sf"]),
        _f(qk["k_codes"]), _f(qk["k_scales"]), _f(qk["k_sf"]),
        _f(vq["v_codes"]), _f(vq["v_scales"]), _f(vq["v_sf"]),
        _ptr(out), _dtype_code(out), B, H, N, d, int(bool(causal)), float(sm_scale), _stream()))
    return out


def sage_attn_fwd_quantized_smooth(qk, vq, shape, mode="int8_fp8", causal=False, sm_scale=None,
                                   out_dtype=None, out=None):
    """Attention with Q smoothing on the dicts of sage_quant_qk_smooth and
    sage_quant_v."""
    import torch
    B, H, N, d = shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype or torch.bfloat16,
                          device=qk["q_codes"].device)
    _check(library().sage_attn_fwd_quantized_smooth(
        MODES[mode], _f(qk["q_codes"]), _f(qk["q_scales"]), _f(qk["q_sf"]),
        _f(qk["k_codes"]), _f(qk["k_scales"]), _f(qk["k_sf"]),
        _f(vq["v_codes"]), _f(vq["v_scales"]), _f(vq["v_sf"]), _f(qk["ds"]),
        _ptr(out), _dtype_code(out), B, H, N, d, int(bool(causal)), float(sm_scale), _stream()))
    return out


def sage_attn_fwd(q, k, v, causal=False, sm_scale=None, mode="int8_fp8", out=None,
                  smooth_q=False):
    """O = softmax(Q K^T sm_scale) V through the quantized path; O has q's dtype.
    K and V with fewer heads than Q (grouped-query attention) go to
    sage_attn_fwd_gqa.  smooth_q: Q smoothing (SAGE_FLAG_SMOOTH_Q)."""
    import torch
    B, H, N, d = _shape(q)
    if _shape(k)[1] != H:
        return sage_attn_fwd_gqa(q, k, v, causal=causal, sm_scale=sm_scale, mode=mode, out=out,
                                 smooth_q=smooth_q)
    if _shape(k) != (B, H, N, d) or _shape(v) != (B, H, N, d):
        raise ValueError("q, k, v must have the same shape")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must have the same dtype")
    if out is None:
        out = torch.empty_like(q)
    _check(library().sage_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, H, N, d,
        int(bool(causal)), float(sm_scale or 0.0), MODES[mode] | (SMOOTH_Q if smooth_q else 0),
        _stream()))
    return out


def sage_attn_fwd_gqa(q, k, v, causal=False, sm_scale=None, mode="int8_fp8", out=None,
                      smooth_q=False):
    """Grouped-query attention: q is [B, H, N, d], k and v are [B, Hkv, N, d]
    with Hkv dividing H; query head h reads key/value head h // (H // Hkv)."""
    import torch
    B, H, N, d = _shape(q)
    Hkv = _shape(k)[1]
    if _shape(k) != (B, Hkv, N, d) or _shape(v) != (B, Hkv, N, d):
        raise ValueError("k and v must be [B, Hkv, N, d] with q's B, N and d")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must have the same dtype")
    if out is None:
        out = torch.empty_like(q)
    _check(library().sage_attn_fwd_gqa(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, H, Hkv, N, d,
        int(bool(causal)), float(sm_scale or 0.0), MODES[mode] | (SMOOTH_Q if smooth_q else 0),
        _stream()))
    return out


def sage_attn_fwd_host(q, k, v, causal=False, sm_scale=None, mode="int8_fp8", out=None,
                       smooth_q=False):
    """The whole forward pass on host (CPU) tensors: the library copies the
    heads in chunks to the device, computes, and copies O back, overlapping
    the copies with the compute (pinned tensors overlap best).  Returns O on
    the host once the current CUDA stream has finished it (this call
    synchronises that stream)."""
    import torch
    for t in (q, k, v):
        if t.dim() != 4 or t.is_cuda or not t.is_contiguous():
            raise ValueError("expected contiguous host tensors of shape [B, H, N, d]")
    B, H, N, d = (int(x) for x in q.shape)
    if tuple(k.shape) != (B, H, N, d) or tuple(v.shape) != (B, H, N, d):
        raise ValueError("q, k, v must have the same shape")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must have the same dtype")
    if out is None:
        out = torch.empty_like(q, pin_memory=q.is_pinned())
    _check(library().sage_attn_fwd_host(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, H, N, d,
        int(bool(causal)), float(sm_scale or 0.0), MODES[mode] | (SMOOTH_Q if smooth_q else 0),
        _stream()))
    torch.cuda.current_stream().synchronize()
    return out


def sage_attn_fwd_noalloc(q, k, v, causal=False, sm_scale=None, mode="int8_fp8", out=None):
    """sage_attn_fwd for callers that cannot allocate device memory while they
    run: all scratch lives in the library's fixed per-device array (see
    include/sage.h).  `out` should be passed (pre-allocated) by such callers;
    calls that overlap on the GPU share the array and must be serialised."""
    import torch
    B, H, N, d = _shape(q)
    if _shape(k) != (B, H, N, d) or _shape(v) != (B, H, N, d):
        raise ValueError("q, k, v must have the same shape")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must have the same dtype")
    if out is None:
        out = torch.empty_like(q)
    _check(library().sage_attn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, H, N, d,
        int(bool(causal)), float(sm_scale or 0.0), MODES[mode], _stream()))
    return out


def device_status():
    """Reads and clears the kernels' bounded-wait status: 0 when no wait
    expired, else raises SageError (SAGE_ERR_DEVICE_TIMEOUT)."""
    s = library().sage_get_last_device_status()
    if s < 0:
        _check(s)
    return s


def selftest_bounded_wait():
    """Launches the bounded-wait self-test kernel on the current stream (its
    wait expires after about a second; device_status() then reports it)."""
    import torch
    _check(library().sage_selftest_bounded_wait(
        torch.cuda.current_stream().cuda_stream))
