"""GPU attention parity against the oracle (through the C ABI).

Bars (floating point):
  * |O_gpu - O_emulated| <= 2e-3 + half an ulp of the output dtype at
    |O_emulated| (the kernel's result is rounded to bf16/fp16 on output,
    which by itself moves a value by up to half an ulp) + the oracle's bound
    for P~ codes that lie within a relative 2^-15 of an e4m3 rounding
    midpoint (the kernel evaluates P~ in FP32, so either neighbouring code is
    a correct result there; see oracle.attention.fp8_p_ambiguity), and in
    FP4 mode of an e2m1 midpoint or of a UE4M3 group-scale midpoint
    (oracle.attention.fp4_p_ambiguity);
  * cosine(O_gpu, O_exact) >= 0.999 where the quantization scheme itself
    reaches it on the workload, and never more than 2e-4 below the
    emulated oracle's own cosine.
"""

import math

import numpy as np
import pytest
import torch

import quantized_attention_quant_b200 as sage
from oracle import attention as att
from oracle import encoders as enc
from quantized_attention_quant_b200.workloads import WORKLOADS, make_qkv, to_numpy32
from tests.test_gpu_prepass import rand_qkv

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
AMBIGUITY_EPS = 2.0 ** -15


def half_ulp(x, dtype):
    bits = 8 if dtype == "bf16" else 11
    a = np.maximum(np.abs(x), 2.0 ** -14)
    return np.ldexp(1.0, np.floor(np.log2(a)).astype(int) - bits)


def cosine(a, b):
    a = a.astype(np.float64).ravel()
    b = b.astype(np.float64).ravel()
    return float(a @ b / math.sqrt((a @ a) * (b @ b)))


def check_against_oracle(o_gpu, q, k, v, causal, sm_scale, mode, dtype, rows=None, cos_floor=None,
                         smooth_q=False):
    qs, ks, vs = (to_numpy32(t) for t in (q, k, v))
    emu, amb = att.emulated_sage_attention(qs, ks, vs, causal, sm_scale, mode=mode, rows=rows,
                                           ambiguity_eps=AMBIGUITY_EPS, smooth_q=smooth_q)
    ex = att.exact_attention(qs, ks, vs, causal, sm_scale, rows=rows)
    g = o_gpu.astype(np.float64)
    err = np.abs(g - emu)
    tol = MAX_ABS + half_ulp(emu, dtype) + amb
    bad = err > tol
    assert not bad.any(), (
        f"{bad.sum()} of {bad.size} outside tolerance; worst excess "
        f"{(err - tol).max():.3e} at {np.unravel_index((err - tol).argmax(), err.shape)}")
    c_gpu, c_emu = cosine(g, ex), cosine(emu, ex)
    assert c_gpu >= c_emu - 2e-4, (c_gpu, c_emu)
    if cos_floor is not None:
        assert c_gpu >= cos_floor, (c_gpu, c_emu)
    return err.max(), c_gpu, c_emu


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("N", [128, 512])
def test_int8_fp8_random(cuda_device, N, dtype, d, causal):
    q, k, v = rand_qkv(2, 2, N, d, dtype, seed=100 + N + d + causal)
    o = sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode="int8_fp8")
    torch.cuda.synchronize()
    check_against_oracle(to_numpy32(o), q, k, v, causal, 1 / math.sqrt(d), "int8_fp8", dtype)
    assert sage.device_status() == 0


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("N", [128, 512])
def test_fp4_random(cuda_device, N, dtype, causal):
    q, k, v = rand_qkv(2, 2, N, 128, dtype, seed=300 + N + causal)
    o = sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode="fp4")
    torch.cuda.synchronize()
    check_against_oracle(to_numpy32(o), q, k, v, causal, 1 / math.sqrt(128), "fp4", dtype)
    assert sage.device_status() == 0


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("N", [128, 512])
def test_fp8_qk_random(cuda_device, N, dtype, d, causal):
    q, k, v = rand_qkv(2, 2, N, d, dtype, seed=500 + N + d + causal)
    o = sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode="fp8")
    torch.cuda.synchronize()
    check_against_oracle(to_numpy32(o), q, k, v, causal, 1 / math.sqrt(d), "fp8", dtype)
    assert sage.device_status() == 0


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mode", ["int8_fp8", "fp8", "fp4"])
@pytest.mark.parametrize("N", [1, 77, 200, 1000])
def test_ragged_lengths(cuda_device, N, mode, causal):
    # N not a multiple of 128: the last tile is partial (keys past N masked,
    # rows past N not stored); d = 64 where the mode allows it
    d = 128 if mode == "fp4" else (64 if N % 2 else 128)
    q, k, v = rand_qkv(2, 2, N, d, "f16", seed=700 + N + causal)
    dev = torch.device("cuda")
    out = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, mode=mode)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    check_against_oracle(to_numpy32(out), q, k, v, causal, 1 / math.sqrt(d), mode, "f16")


def test_ragged_output_stays_in_bounds(cuda_device):
    # O of a ragged sequence is written for its N rows only: a buffer with a
    # sentinel tail right after O keeps the sentinel
    B, H, N, d = 1, 2, 200, 128
    q, k, v = rand_qkv(B, H, N, d, "bf16", seed=801)
    dev = torch.device("cuda")
    n = B * H * N * d
    buf = torch.full((n + 4096,), 3.0, dtype=torch.bfloat16, device=dev)
    o = buf[:n].view(B, H, N, d)
    sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev), out=o)
    torch.cuda.synchronize()
    assert torch.all(buf[n:] == 3.0)
    check_against_oracle(to_numpy32(o), q, k, v, False, 1 / math.sqrt(d), "int8_fp8", "bf16")


def test_fp4_zero_q_gives_mean_v(cuda_device):
    # Q = 0 -> every score 0 -> P~ = 1 -> s16 = 448, code e2m1(6) = 6, whose
    # value 6 * 448 / 2688 is exactly 1 -> O = mean of the FP4-dequantized V
    # (prefix means when causal).  Exercises the FP4 P~V path and its
    # scale factors in closed form.
    B, H, N, d = 1, 2, 512, 128
    _, k, v = rand_qkv(B, H, N, d, "bf16", seed=6)
    q = torch.zeros_like(k)
    from oracle import prepass as pp
    vc, vsf, vg = pp.quant_v_fp4(to_numpy32(v))
    # [B, H, d, N] values -> [B, H, N, d]
    tile_of = np.arange(N) // 128
    vd = (enc.e2m1_decode(vc) * np.repeat(enc.ue4m3_decode(vsf), 16, axis=-1)
          * vg[:, :, None, tile_of]).transpose(0, 1, 3, 2)
    for causal in (False, True):
        o = to_numpy32(sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode="fp4"))
        if causal:
            want = np.cumsum(vd, axis=2) / np.arange(1, N + 1)[None, None, :, None]
        else:
            want = np.broadcast_to(vd.mean(axis=2, keepdims=True), vd.shape)
        assert np.max(np.abs(o - want) - half_ulp(want, "bf16") - 1e-5) <= 0
    assert sage.device_status() == 0


def test_int8_fp8_zero_q_gives_mean_v(cuda_device):
    # Q = 0 -> every score 0 -> P~ = 1 (code 448) -> O = mean of dequantized V.
    B, H, N, d = 1, 2, 512, 128
    _, k, v = rand_qkv(B, H, N, d, "bf16", seed=5)
    q = torch.zeros_like(k)
    for causal in (False, True):
        o = to_numpy32(sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal))
        vs = to_numpy32(v)
        from oracle import prepass as pp
        vc, s = pp.quant_v_fp8(vs)
        vd = enc.e4m3_decode(vc).transpose(0, 1, 3, 2) * s[:, :, None, :]
        if causal:
            want = np.cumsum(vd, axis=2) / np.arange(1, N + 1)[None, None, :, None]
        else:
            want = np.broadcast_to(vd.mean(axis=2, keepdims=True), vd.shape)
        assert np.max(np.abs(o - want) - half_ulp(want, "bf16") - 1e-5) <= 0


def test_int8_fp8_onehot_selects_rows(cuda_device):
    # Query r points at key pi(r) only; the logit gap makes P~ one-hot, so
    # O[r] = dequantized V[pi(r)].  Exercises the Q K^T row/column mapping.
    B, H, N, d = 1, 1, 128, 128
    dev = torch.device("cuda")
    perm = np.random.default_rng(3).permutation(N)
    qc = np.zeros((N, d), np.int8)
    qc[np.arange(N), perm] = 127
    kc = np.zeros((N, d), np.int8)
    kc[np.arange(N), np.arange(N)] = 127
    v = torch.from_numpy(np.random.default_rng(4).standard_normal((B, H, N, d)).astype(np.float32)
                         ).to(torch.bfloat16)
    vq = sage.sage_quant_v(v.to(dev))
    qk = {"q_codes": torch.from_numpy(qc.view(np.uint8).ravel()).to(dev),
          # one Q scale per token, one K scale per 32 keys, all 1
          "q_scales": torch.ones(N, dtype=torch.float32, device=dev).view(torch.uint8),
          "q_sf": None,
          "k_codes": torch.from_numpy(kc.view(np.uint8).ravel()).to(dev),
          "k_scales": torch.ones(N // 32, dtype=torch.float32, device=dev).view(torch.uint8),
          "k_sf": None}
    o = to_numpy32(sage.sage_attn_fwd_quantized(qk, vq, (B, H, N, d), sm_scale=0.05))
    from oracle import prepass as pp
    vc, s = pp.quant_v_fp8(to_numpy32(v))
    vd = enc.e4m3_decode(vc).transpose(0, 1, 3, 2) * s[:, :, None, :]
    want = vd[0, 0, perm]
    assert np.max(np.abs(o[0, 0] - want) - half_ulp(want, "bf16")) <= 1e-6


def test_fwd_equals_prepass_plus_attention(cuda_device):
    q, k, v = rand_qkv(1, 4, 384, 128, "bf16", seed=9)
    dev = torch.device("cuda")
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    for mode in ["int8_fp8", "fp4", "fp8"]:
        a = sage.sage_attn_fwd(qg, kg, vg, causal=True, mode=mode)
        qk = sage.sage_quant_qk(qg, kg, mode)
        vq = sage.sage_quant_v(vg, mode)
        b = sage.sage_attn_fwd_quantized(qk, vq, tuple(q.shape), mode, causal=True,
                                         out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_side_stream(cuda_device):
    q, k, v = rand_qkv(1, 2, 256, 64, "bf16", seed=10)
    dev = torch.device("cuda")
    ref = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev))
    s.synchronize()
    assert torch.equal(ref, out)


# cosine floor against exact attention where the quantization scheme itself
# reaches 0.999 (per-token Q and per-32-key K scales); elsewhere the test holds
# the GPU to the emulated oracle's own cosine
FULL = [("tiny", 0.999), ("llm", None), ("video", 0.999), ("long", 0.999), ("long_causal", 0.999),
        ("fp4", None), ("long_fp8", None), ("llm_fp8", None), ("short", None),
        ("n16k", 0.999), ("n16k_fp8", None)]


@pytest.mark.parametrize("name,cos_floor", FULL)
def test_full_workloads(cuda_device, name, cos_floor):
    """Full-size launch (as timed by bench.py); sampled heads and rows."""
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    dev = torch.device("cuda")
    o = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=w.causal, mode=w.mode)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    rng = np.random.default_rng(0)
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    n_rows = w.N if w.N <= 512 else 256
    rows = np.sort(rng.choice(w.N, n_rows, replace=False))
    rows[-1] = w.N - 1                                   # always include the last row
    og = to_numpy32(o)
    for (b, h) in heads:
        sel = (slice(b, b + 1), slice(h, h + 1))
        check_against_oracle(og[sel][:, :, rows], q[sel], k[sel], v[sel], w.causal, w.sm_scale,
                             w.mode, w.dtype, rows=rows, cos_floor=cos_floor)


def test_bounded_wait_expires_and_context_survives(cuda_device):
    # a wait that nothing completes gives up after about a second, records
    # the timeout in the device status word, and leaves the context usable
    assert sage.device_status() == 0
    sage.selftest_bounded_wait()
    with pytest.raises(sage.SageError, match="timed out|bounded wait expired"):
        sage.device_status()
    assert sage.device_status() == 0          # read-and-clear
    q, k, v = rand_qkv(1, 2, 256, 128, "bf16", seed=77)
    o = sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    check_against_oracle(to_numpy32(o), q, k, v, True, 1 / math.sqrt(128), "int8_fp8", "bf16")
    assert sage.device_status() == 0


@pytest.mark.parametrize("mode", ["int8_fp8", "fp8"])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,d", [(512, 128), (300, 64), (1000, 128)])
def test_persistent_kernel_matches_one_item_per_cta(cuda_device, mode, causal, N, d):
    """Many short work items run on the persistent INT8/FP8 kernel (one CTA
    per SM working through a list of (query tile, head) items); a launch
    with few items runs one CTA per item.  Both compute the same arithmetic
    in the same order, so the heads they share must agree bit for bit; the
    large launch is also held to the oracle on sampled heads."""
    H = 80                                   # 80 heads x >= 3 tiles > 148 items
    q, k, v = rand_qkv(1, H, N, d, "bf16", seed=900 + N + d + causal)
    dev = torch.device("cuda")
    big = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, mode=mode)
    sub = [0, 37, 79]
    small = sage.sage_attn_fwd(q[:, sub].contiguous().to(dev), k[:, sub].contiguous().to(dev),
                               v[:, sub].contiguous().to(dev), causal=causal, mode=mode)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    assert torch.equal(big[:, sub], small)
    for h in (0, 79):
        sel = (slice(0, 1), slice(h, h + 1))
        check_against_oracle(to_numpy32(big[sel]), q[sel], k[sel], v[sel], causal,
                             1 / math.sqrt(d), mode, "bf16")


# N = 640: the cluster-fused pre-pass (one launch); N = 1280: the two
# pre-pass chains, the V chain forked onto the library's second stream
@pytest.mark.parametrize("N", [640, 1280])
def test_cuda_graph_capture_and_replay(cuda_device, N):
    # sage_attn_fwd inside a captured CUDA graph (with the chains, the
    # fork/join to the library's second stream is recorded too); replays
    # match eager runs
    B, H, d = 1, 4, 128
    q, k, v = rand_qkv(B, H, N, d, "bf16", seed=1300)
    dev = torch.device("cuda")
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty_like(qg)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        sage.sage_attn_fwd(qg, kg, vg, causal=True, out=out)   # warm-up: workspace, streams
    s.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sage.sage_attn_fwd(qg, kg, vg, causal=True, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    qg.copy_(rand_qkv(B, H, N, d, "bf16", seed=1301)[0].to(dev))
    g.replay()
    torch.cuda.synchronize()
    ref = sage.sage_attn_fwd(qg, kg, vg, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert sage.device_status() == 0


def test_workspace_allocation_failure_is_reported(cuda_device):
    """A failed workspace allocation (made to fail on the host, in place of
    the allocation call) comes back as SAGE_ERR_CUDA naming the failure;
    nothing is launched, and the next call allocates and computes."""
    lib = sage.library()
    # larger than anything the other tests run on a pooled stream, so the
    # stream's workspace has to grow
    B, H, N, d = 1, 8, 4096, 128
    q, k, v = rand_qkv(B, H, N, d, "bf16", seed=1700)
    dev = torch.device("cuda")
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    s = torch.cuda.Stream()
    out = torch.full_like(qg, 7.0)
    assert lib.sage_debug_fail_allocations(1) == 0
    with torch.cuda.stream(s):
        with pytest.raises(sage.SageError) as err:
            sage.sage_attn_fwd(qg, kg, vg, out=out)
    assert err.value.status == -3 and "injected failure" in str(err.value)
    s.synchronize()
    assert torch.all(out == 7.0)            # no kernel ran
    with torch.cuda.stream(s):
        sage.sage_attn_fwd(qg, kg, vg, out=out)
    s.synchronize()
    assert sage.device_status() == 0
    rows = np.r_[0:8, 1000, 2047, 4095]
    hs = [0, H - 1]
    check_against_oracle(to_numpy32(out)[:, hs][:, :, rows], q[:, hs], k[:, hs], v[:, hs], False,
                         1 / math.sqrt(d), "int8_fp8", "bf16", rows=rows)
    assert lib.sage_debug_fail_allocations(-1) == -1
    assert lib.sage_debug_fail_allocations(0) == 0
