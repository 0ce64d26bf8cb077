"""Q smoothing on the GPU (SageAttention2 abstract, "we propose a method to
smooth Q"; the oracle's pre-pass reading 2), through the C ABI.

The pre-pass outputs (codes, scales, the K mean, the per-block Q means and
the FP32 score bias) must equal the oracle's bit for bit; O must meet the
attention bar of tests/test_gpu_attention.py against the oracle's smoothed
emulation; the one-call path must equal the split calls bit for bit; and on
queries that carry a per-channel bias the smoothed pass must come closer to
exact attention than the unsmoothed one.
"""

import math

import numpy as np
import pytest
import torch

import quantized_attention_quant_b200 as sage
from oracle import attention as att
from oracle import prepass as pp
from quantized_attention_quant_b200.workloads import to_numpy32
from tests import layouts as L
from tests.test_gpu_attention import check_against_oracle, cosine

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def biased_qkv(B, H, N, d, dtype, seed, q_bias=3.0, k_bias=2.0, Hkv=None):
    """Q and K with per-channel biases (what the two smoothings remove)."""
    g = np.random.default_rng(seed)
    Hkv = Hkv or H
    q = g.standard_normal((B, H, N, d)) + q_bias * g.standard_normal((B, H, 1, d))
    k = g.standard_normal((B, Hkv, N, d)) + k_bias * g.standard_normal((B, Hkv, 1, d))
    v = g.standard_normal((B, Hkv, N, d))
    return [torch.from_numpy(x.astype(np.float32)).to(TDT[dtype]) for x in (q, k, v)]


@pytest.mark.parametrize("mode,N,d", [(m, N, d) for m in ("int8_fp8", "fp8")
                                      for (N, d) in [(128, 128), (300, 64), (1000, 128), (2048, 128)]]
                         + [("fp4", 128, 128), ("fp4", 300, 128), ("fp4", 2048, 128)])
def test_smoothed_prepass_matches_oracle(cuda_device, mode, N, d):
    B, H = 1, 2
    q, k, _ = biased_qkv(B, H, N, d, "bf16", seed=N + d)
    dev = torch.device("cuda")
    qk = sage.sage_quant_qk_smooth(q.to(dev), k.to(dev), mode)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    Np, nt = L.np_of(N), -(-N // 128)
    ds = L.f32(qk["ds"], B, H, nt * Np).reshape(B, H, nt, Np)
    assert not ds[..., N:].any()                       # keys past N hold 0
    got = dict(k_mean=L.f32(qk["k_mean"], B, H, d),
               q_mean=L.f32(qk["q_mean"], B, H, nt * d).reshape(B, H, nt, d),
               dS=ds[..., :N])
    if mode == "fp4":
        got.update(q_codes=L.unpack_fp4(qk["q_codes"], B, H, Np, d)[:, :, :N],
                   q_sf=L.qk_sf(qk["q_sf"], B, H, N, d), q_g=L.f32(qk["q_scales"], B, H, nt),
                   k_codes=L.unpack_fp4(qk["k_codes"], B, H, Np, d)[:, :, :N],
                   k_sf=L.qk_sf(qk["k_sf"], B, H, N, d), k_g=L.f32(qk["k_scales"], B, H, nt))
    else:
        codes = L.token_codes if mode == "fp8" else L.int8_codes
        got.update(q_codes=codes(qk["q_codes"], B, H, N, d),
                   q_scales=L.f32(qk["q_scales"], B, H, Np)[:, :, :N],
                   k_codes=codes(qk["k_codes"], B, H, N, d),
                   k_scales=L.f32(qk["k_scales"], B, H, Np // 32)[:, :, :-(-N // 32)])
    assert not L.padded_tokens(qk["q_codes"], B, H, N).any()
    qs, ks = to_numpy32(q), to_numpy32(k)
    fn = {"fp8": pp.quant_qk_fp8, "int8_fp8": pp.quant_qk_int8, "fp4": pp.quant_qk_fp4}[mode]
    want = fn(qs, ks, smooth=True)
    for name, arr in want.items():
        g = got[name]
        if arr.dtype == np.float32:
            assert np.array_equal(g.view(np.uint32), arr.view(np.uint32)), name
        else:
            assert np.array_equal(g.view(np.uint8), arr.view(np.uint8)), name


# N = 77 is one key tile; N >= 1100 (9 to 11 tiles, ragged) cycles the
# exp warpgroups' shared slots (2 for the partial maxima, 4 for alpha and
# the biases) more than twice
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mode,N,d", [("int8_fp8", 512, 128), ("int8_fp8", 300, 64),
                                      ("fp8", 640, 128), ("int8_fp8", 77, 128),
                                      ("fp4", 512, 128), ("fp4", 300, 128),
                                      ("int8_fp8", 1200, 128), ("fp8", 1300, 64),
                                      ("fp4", 1100, 128)])
def test_smoothed_attention_matches_oracle(cuda_device, mode, N, d, causal):
    B, H = 1, 2
    q, k, v = biased_qkv(B, H, N, d, "bf16", seed=10 + N + d + causal)
    dev = torch.device("cuda")
    o = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, mode=mode,
                           smooth_q=True)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    check_against_oracle(to_numpy32(o), q, k, v, causal, 1 / math.sqrt(d), mode, "bf16",
                         smooth_q=True)


@pytest.mark.parametrize("mode", ["int8_fp8", "fp8", "fp4"])
def test_smoothed_one_call_equals_split_calls(cuda_device, mode):
    B, H, N, d = 2, 3, 700, 128
    q, k, v = (t.cuda() for t in biased_qkv(B, H, N, d, "bf16", seed=41))
    one = sage.sage_attn_fwd(q, k, v, causal=True, mode=mode, smooth_q=True)
    qk = sage.sage_quant_qk_smooth(q, k, mode)
    vq = sage.sage_quant_v(v, mode)
    two = sage.sage_attn_fwd_quantized_smooth(qk, vq, (B, H, N, d), mode, causal=True)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    assert torch.equal(one, two)


@pytest.mark.parametrize("mode", ["int8_fp8", "fp8", "fp4"])
def test_smoothed_gqa_equals_repeated_heads(cuda_device, mode):
    # grouped-query attention with Q smoothing: the bias pairs each query
    # head's block means with its key/value head's smoothed keys, and the
    # exp warpgroups read the K scales of the key/value head
    B, H, Hkv, N, d = 1, 4, 2, 384, 128
    q, k, v = (t.cuda() for t in biased_qkv(B, H, N, d, "bf16", seed=43, Hkv=Hkv))
    o = sage.sage_attn_fwd_gqa(q, k, v, mode=mode, smooth_q=True)
    rep = H // Hkv
    o2 = sage.sage_attn_fwd(q, k.repeat_interleave(rep, 1).contiguous(),
                            v.repeat_interleave(rep, 1).contiguous(), mode=mode,
                            smooth_q=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)


@pytest.mark.parametrize("mode,gain,floor", [("int8_fp8", 0.0, 0.999), ("fp8", 5e-4, 0.999),
                                             ("fp4", 5e-3, 0.989)])
def test_smoothing_brings_biased_queries_closer_to_exact(cuda_device, mode, gain, floor):
    # queries with a per-channel bias (N(0, 3)): the smoothed pass is closer
    # to exact attention; sampled rows of 2 heads at N = 4096
    B, H, N, d = 1, 2, 4096, 128
    q, k, v = biased_qkv(B, H, N, d, "bf16", seed=47)
    dev = torch.device("cuda")
    o0 = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev), mode=mode)
    o1 = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev), mode=mode, smooth_q=True)
    torch.cuda.synchronize()
    rows = np.linspace(0, N - 1, 96).astype(int)
    ex = att.exact_attention(to_numpy32(q), to_numpy32(k), to_numpy32(v), rows=rows)
    c0 = cosine(to_numpy32(o0)[:, :, rows], ex)
    c1 = cosine(to_numpy32(o1)[:, :, rows], ex)
    assert c1 > c0 + gain, (c0, c1)
    assert c1 >= floor, c1
