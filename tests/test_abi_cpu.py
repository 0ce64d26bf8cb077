"""The C-ABI library builds for sm_100a, loads without a GPU, exports every
symbol include/sage.h declares, and rejects bad arguments before touching a
device (CPU only: no compute call is made)."""

import ctypes
import os
import re

import pytest

from quantized_attention_quant_b200 import build as qb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    qb.build()
    import quantized_attention_quant_b200 as q
    return q.library()


def header_functions():
    text = open(os.path.join(ROOT, "include", "sage.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))


def test_exports_match_header(lib):
    import quantized_attention_quant_b200 as q
    names = header_functions()
    assert names == sorted(q.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.sage_version().decode().startswith("sage-b200")


def test_ubench_library_exports_its_header():
    # the microbenchmark library exports every function include/sage_ubench.h
    # declares, and rejects bad arguments before touching a device
    import ctypes

    from quantized_attention_quant_b200 import build as qb
    qb.build()
    text = open(os.path.join(ROOT, "include", "sage_ubench.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))
    assert names == ["sage_ubench_dfma", "sage_ubench_exp", "sage_ubench_exp2_poly",
                     "sage_ubench_mma"]
    ub = ctypes.CDLL(qb.UBENCH_LIB)
    for n in names:
        assert hasattr(ub, n), n
    v = ctypes.c_double(0.0)
    ub.sage_ubench_mma.argtypes = [ctypes.c_int] * 4 + [ctypes.POINTER(ctypes.c_double)]
    ub.sage_ubench_exp.argtypes = [ctypes.c_int] * 3 + [ctypes.POINTER(ctypes.c_double)]
    assert ub.sage_ubench_mma(0, 96, 10, 1, ctypes.byref(v)) == -1      # N must be 128 or 256
    assert ub.sage_ubench_mma(7, 128, 10, 1, ctypes.byref(v)) == -1     # unknown kind
    assert ub.sage_ubench_mma(3, 64, 10, 1, ctypes.byref(v)) == -1      # FP4 kind: N 128 or 256 too
    assert ub.sage_ubench_exp(0, 100, 10, ctypes.byref(v)) == -1        # not whole warps
    assert ub.sage_ubench_exp(5, 128, 10, ctypes.byref(v)) == -1        # unknown mode
    ub.sage_ubench_dfma.argtypes = [ctypes.c_int] * 2 + [ctypes.POINTER(ctypes.c_double)]
    assert ub.sage_ubench_dfma(100, 10, ctypes.byref(v)) == -1          # not whole warps
    assert ub.sage_ubench_dfma(128, 0, ctypes.byref(v)) == -1           # no rounds
    ub.sage_ubench_exp2_poly.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    assert ub.sage_ubench_exp2_poly(None, None, 4) == -1               # null buffers


def test_allocation_failure_injection_arguments(lib):
    # the injection is a host-side counter: no device call
    assert lib.sage_debug_fail_allocations(2) == 0
    assert lib.sage_debug_fail_allocations(0) == 0
    assert lib.sage_debug_fail_allocations(-1) == -1


def test_buffer_bytes(lib):
    import quantized_attention_quant_b200 as q
    B, H, N, d = 2, 3, 256, 128
    assert q.buffer_bytes("int8_fp8", "q_codes", B, H, N, d) == B * H * N * d
    # 8-bit modes: one Q scale per token, one K scale per 32 tokens, over
    # the padded length (N = 200 pads to 256)
    assert q.buffer_bytes("int8_fp8", "q_scales", B, H, N, d) == B * H * N * 4
    assert q.buffer_bytes("int8_fp8", "k_scales", B, H, N, d) == B * H * (N // 32) * 4
    assert q.buffer_bytes("fp8", "q_scales", B, H, 200, d) == B * H * 256 * 4
    assert q.buffer_bytes("fp8", "k_scales", B, H, 200, d) == B * H * 8 * 4
    assert q.buffer_bytes("fp4", "q_scales", B, H, N, d) == B * H * 2 * 4
    assert q.buffer_bytes("fp4", "k_scales", B, H, N, d) == B * H * 2 * 4
    assert q.buffer_bytes("int8_fp8", "q_sf", B, H, N, d) == 0
    assert q.buffer_bytes("int8_fp8", "v_scales", B, H, N, d) == B * H * d * 4
    assert q.buffer_bytes("fp4", "q_codes", B, H, N, d) == B * H * N * d // 2
    assert q.buffer_bytes("fp4", "q_sf", B, H, N, d) == B * H * 2 * 2 * 512
    assert q.buffer_bytes("fp4", "v_sf", B, H, N, d) == B * H * 2 * 2 * 512
    assert q.buffer_bytes("fp4", "v_scales", B, H, N, d) == B * H * 2 * 4
    assert lib.sage_buffer_bytes(0, 0, -1, 1, 1, 1) == 0


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def call_attn(lib, **kw):
    a = dict(mode=0, qc=FAKE, qs=FAKE, qsf=None, kc=FAKE, ks=FAKE, ksf=None, vc=FAKE, vs=FAKE,
             vsf=None, o=FAKE, dtype=1, B=1, H=1, N=128, d=64, causal=0, sm=0.125)
    a.update(kw)
    return lib.sage_attn_fwd_quantized(a["mode"], a["qc"], a["qs"], a["qsf"], a["kc"], a["ks"],
                                       a["ksf"], a["vc"], a["vs"], a["vsf"], a["o"], a["dtype"],
                                       a["B"], a["H"], a["N"], a["d"], a["causal"],
                                       ctypes.c_float(a["sm"]), None)


@pytest.mark.parametrize("kw,status,text", [
    (dict(dtype=7), -1, "dtype"),
    (dict(mode=3), -1, "mode"),
    (dict(B=-1), -1, "negative"),
    (dict(d=96), -2, "head dim"),
    (dict(mode=1, d=64, qsf=FAKE, ksf=FAKE, vsf=FAKE), -2, "FP4"),
    (dict(B=1, H=1, N=2 ** 31 - 100), -2, "2^31"),     # rounded up past 2^31
    (dict(qc=None), -1, "q_codes is NULL"),
    (dict(o=FAKE + 4), -2, "aligned"),
    (dict(qsf=FAKE), -1, "must be NULL"),
    (dict(mode=1, d=128), -1, "q_sf is NULL"),
    (dict(sm=-1.0), -1, "sm_scale"),
    (dict(B=70000, H=1), -2, "65535"),
])
def test_attn_argument_errors(lib, kw, status, text):
    s = call_attn(lib, **kw)
    assert s == status
    assert text in lib.sage_status_string(s).decode()


def test_empty_is_a_noop(lib):
    for B, H, N in [(0, 4, 128), (2, 0, 128), (2, 4, 0)]:
        assert call_attn(lib, B=B, H=H, N=N) == 0
        assert lib.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, 1, B, H, N, 128, 0,
                                 ctypes.c_float(0.0), 0, None) == 0


def test_quant_argument_errors(lib):
    s = lib.sage_quant_qk(FAKE, FAKE, 1, 1, 1, 128, 64, 0, FAKE, FAKE, None, FAKE, FAKE, None,
                          None, None)
    assert s == -1 and "k_mean" in lib.sage_status_string(s).decode()
    s = lib.sage_quant_v(FAKE, 1, 1, 1, 128, 128, 1, FAKE, FAKE, None, None)
    assert s == -1 and "v_sf" in lib.sage_status_string(s).decode()
    assert lib.sage_quant_v(FAKE, 1, 0, 1, 128, 128, 0, FAKE, FAKE, None, None) == 0


def test_status_strings(lib):
    for s, t in [(0, "ok"), (-1, "invalid"), (-2, "unsupported"), (-3, "CUDA"), (-4, "timed out")]:
        assert t in lib.sage_status_string(s).decode()


def gqa(lib, B=2, H=8, Hkv=2, N=128, d=128, mode=0):
    lib.sage_attn_fwd_gqa.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] + \
        [ctypes.c_int64] * 5 + [ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
    return lib.sage_attn_fwd_gqa(FAKE, FAKE, FAKE, FAKE, 1, B, H, Hkv, N, d, 0,
                                 ctypes.c_float(0.0), mode, None)


@pytest.mark.parametrize("H,Hkv", [(8, 0), (8, 3), (8, 16), (8, -1), (0, 1)])
def test_gqa_head_count_errors(lib, H, Hkv):
    s = gqa(lib, H=H, Hkv=Hkv)
    assert s == -1 and "Hkv" in lib.sage_status_string(s).decode()


def test_gqa_empty_and_shape_errors(lib):
    assert gqa(lib, B=0) == 0
    assert gqa(lib, N=0) == 0
    assert gqa(lib, H=0, Hkv=0) == 0
    s = gqa(lib, B=1, H=8, Hkv=2, N=2 ** 28)
    assert s == -2 and "2^31" in lib.sage_status_string(s).decode()


def test_missing_library_fails_loudly(monkeypatch):
    # no CPU fallback: without libsage_b200.so every entry point raises
    import torch
    import quantized_attention_quant_b200 as sage
    monkeypatch.setattr(sage, "library_path", "/nonexistent/libsage_b200.so")
    monkeypatch.setattr(sage, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        sage.library()
    with pytest.raises(RuntimeError, match="no fallback"):
        sage.buffer_bytes("int8_fp8", "q_codes", 1, 1, 128, 64)
    # and host tensors are refused rather than computed on the CPU
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sage.sage_attn_fwd(q, q, q)


def test_smoothing_buffers_and_argument_errors(lib):
    # Q smoothing: buffer sizes, and every refusal comes before any device
    # call (required pointers; the FP4 scale-factor buffers; the mode flag)
    import quantized_attention_quant_b200 as q
    B, H, N, d = 2, 3, 200, 128
    nt, Np = 2, 256
    assert q.buffer_bytes("int8_fp8", "q_mean", B, H, N, d) == B * H * nt * d * 4
    assert q.buffer_bytes("fp8", "ds", B, H, N, d) == B * H * nt * Np * 4
    assert q.buffer_bytes("fp4", "q_mean", B, H, N, d) == B * H * nt * d * 4
    assert q.buffer_bytes("fp4", "ds", B, H, N, d) == B * H * nt * Np * 4
    s = lib.sage_quant_qk_smooth(FAKE, FAKE, 1, 1, 1, 128, 128, 1, FAKE, FAKE, None, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, FAKE, None)
    assert s == -1 and "q_sf is NULL" in lib.sage_status_string(s).decode()
    s = lib.sage_quant_qk_smooth(FAKE, FAKE, 1, 1, 1, 128, 128, 0, FAKE, FAKE, None, FAKE, FAKE,
                                 None, FAKE, None, FAKE, None)
    assert s == -1 and "q_mean is NULL" in lib.sage_status_string(s).decode()
    s = lib.sage_attn_fwd_quantized_smooth(0, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, FAKE,
                                           None, None, FAKE, 1, 1, 1, 128, 128, 0,
                                           ctypes.c_float(0.1), None)
    assert s == -1 and "ds is NULL" in lib.sage_status_string(s).decode()
    s = lib.sage_attn_fwd_quantized_smooth(0, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE,
                                           None, FAKE, FAKE, 1, 1, 1, 128, 128, 0,
                                           ctypes.c_float(0.1), None)
    assert s == -1 and "must be NULL" in lib.sage_status_string(s).decode()
    assert lib.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, 1, 0, 1, 128, 128, 0, ctypes.c_float(0.0),
                             q.SMOOTH_Q, None) == 0
    s = lib.sage_attn_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 128, 128, 0,
                                  ctypes.c_float(0.0), q.SMOOTH_Q, None)
    assert s == -1 and "mode" in lib.sage_status_string(s).decode()


def test_host_pass_argument_errors(lib):
    s = lib.sage_attn_fwd_host(FAKE, None, FAKE, FAKE, 1, 1, 1, 128, 128, 0, ctypes.c_float(0.0),
                               0, None)
    assert s == -1 and "NULL" in lib.sage_status_string(s).decode()
    assert lib.sage_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, 1, 0, 4, 128, 128, 0,
                                  ctypes.c_float(0.0), 0, None) == 0
    s = lib.sage_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 128, 96, 0, ctypes.c_float(0.0),
                               0, None)
    assert s == -2 and "head dim" in lib.sage_status_string(s).decode()
