"""Grouped-query and multi-query attention on the GPU (through the C ABI).

Query head h of a group of G = H / Hkv heads reads key/value head h // G.
K smoothing and the K/V quantization act per key/value head and per token
block, so the result must equal, bit for bit, the multi-head forward pass on
K and V repeated G times along the head axis; that pass is in turn held to
the oracle here (same bars as tests/test_gpu_attention.py).
"""

import math

import pytest
import torch

import quantized_attention_quant_b200 as sage
from quantized_attention_quant_b200.workloads import to_numpy32
from tests.test_gpu_attention import check_against_oracle
from tests.test_gpu_prepass import rand_qkv

pytestmark = pytest.mark.gpu


def gqa_inputs(B, H, Hkv, N, d, dtype, seed):
    q, _, _ = rand_qkv(B, H, N, d, dtype, seed)
    _, k, v = rand_qkv(B, Hkv, N, d, dtype, seed + 1)
    return q, k, v


def repeat_heads(x, G):
    return x.repeat_interleave(G, dim=1).contiguous()


CASES = [  # (B, H, Hkv, N, d)
    (2, 8, 2, 384, 128),
    (1, 4, 1, 256, 128),     # multi-query
    (2, 6, 3, 256, 64),
    (1, 2, 2, 128, 64),      # Hkv == H: plain multi-head attention
    (2, 4, 2, 333, 128),     # a ragged length
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mode", ["int8_fp8", "fp4", "fp8"])
@pytest.mark.parametrize("B,H,Hkv,N,d", CASES)
def test_gqa_matches_repeated_kv(cuda_device, B, H, Hkv, N, d, mode, causal):
    if mode == "fp4" and d != 128:
        pytest.skip("FP4 mode runs at d = 128")
    q, k, v = gqa_inputs(B, H, Hkv, N, d, "bf16", seed=300 + H * Hkv + N + d)
    dev = torch.device("cuda")
    G = H // Hkv
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    o = sage.sage_attn_fwd_gqa(qg, kg, vg, causal=causal, mode=mode)
    o_rep = sage.sage_attn_fwd(qg, repeat_heads(kg, G), repeat_heads(vg, G), causal=causal,
                               mode=mode)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    assert torch.equal(o, o_rep)
    check_against_oracle(to_numpy32(o), q, repeat_heads(k, G), repeat_heads(v, G), causal,
                         1 / math.sqrt(d), mode, "bf16")


def test_gqa_dispatch_from_sage_attn_fwd(cuda_device):
    q, k, v = gqa_inputs(1, 8, 2, 256, 128, "f16", seed=41)
    dev = torch.device("cuda")
    a = sage.sage_attn_fwd(q.to(dev), k.to(dev), v.to(dev))
    b = sage.sage_attn_fwd_gqa(q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("mode", ["int8_fp8", "fp4"])
def test_gqa_many_heads(cuda_device, mode):
    """An LLM-like head layout: 32 query heads over 8 key/value heads, two
    batches, several K/V tiles; bit-exact against repeated K/V."""
    B, H, Hkv, N, d = 2, 32, 8, 1024, 128
    q, k, v = gqa_inputs(B, H, Hkv, N, d, "bf16", seed=55)
    dev = torch.device("cuda")
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    for causal in (False, True):
        o = sage.sage_attn_fwd_gqa(qg, kg, vg, causal=causal, mode=mode)
        o_rep = sage.sage_attn_fwd(qg, repeat_heads(kg, 4), repeat_heads(vg, 4), causal=causal,
                                   mode=mode)
        torch.cuda.synchronize()
        assert torch.equal(o, o_rep)
    assert sage.device_status() == 0


def test_gqa_rejects_bad_head_counts(cuda_device):
    q, k, v = gqa_inputs(1, 6, 4, 128, 64, "bf16", seed=3)
    dev = torch.device("cuda")
    with pytest.raises(sage.SageError, match="Hkv"):
        sage.sage_attn_fwd_gqa(q.to(dev), k.to(dev), v.to(dev))


@pytest.mark.parametrize("causal", [True, False])
def test_gqa_persistent_kernel(cuda_device, causal):
    """Enough short items for the persistent INT8/FP8 kernel: GQA still
    equals the multi-head pass on repeated K/V bit for bit."""
    B, H, Hkv, N, d = 2, 48, 12, 384, 128
    q, k, v = gqa_inputs(B, H, Hkv, N, d, "bf16", seed=77 + causal)
    dev = torch.device("cuda")
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    o = sage.sage_attn_fwd_gqa(qg, kg, vg, causal=causal)
    o_rep = sage.sage_attn_fwd(qg, repeat_heads(kg, 4), repeat_heads(vg, 4), causal=causal)
    torch.cuda.synchronize()
    assert sage.device_status() == 0
    assert torch.equal(o, o_rep)
