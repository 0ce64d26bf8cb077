"""The no-allocation entry point (sage_attn_fwd_noalloc).

Callers that cannot allocate device memory while they run -- a memory pool
that admits no new allocations, an allocator that owns the whole device, a
caller that may not take the driver's allocation locks -- use this variant:
its scratch is a fixed array inside the library's device image.  These tests
check, through the C ABI, that it gives the same result as sage_attn_fwd on
two calls in a row (the second call reuses the array the first one left
behind), and that a shape too large for the array is refused.

The file is named so that pytest collects it last.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import quantized_attention_quant_b200 as sage
from quantized_attention_quant_b200 import build as qb

MAX_ABS = 2e-3


def within_tolerance(a, b, dtype_bits):
    """|a - b| <= 2e-3 + half an ulp of the output dtype (the parity bar)."""
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    half_ulp = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -14))).astype(int)
                        - dtype_bits)
    return float((np.abs(a - b) - MAX_ABS - half_ulp).max()) <= 0.0


def draw(shape, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(shape, generator=g)
    k = torch.randn(shape, generator=g) + 3.0 * torch.randn(shape[:2] + (1, shape[3]), generator=g)
    v = torch.randn(shape, generator=g)
    return [t.to(dtype).cuda() for t in (q, k, v)]


@pytest.mark.gpu
@pytest.mark.parametrize("d,causal,dtype", [(128, True, torch.bfloat16),
                                            (64, False, torch.float16)])
def test_noalloc_matches_sage_attn_fwd_twice(cuda_device, d, causal, dtype):
    bits = 8 if dtype == torch.bfloat16 else 11
    shape = (1, 4, 512, d)
    for call, seed in enumerate((11, 12)):           # two calls in a row
        q, k, v = draw(shape, seed + d, dtype)
        out = torch.empty_like(q)
        got = sage.sage_attn_fwd_noalloc(q, k, v, causal=causal, out=out)
        want = sage.sage_attn_fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert got.data_ptr() == out.data_ptr()
        assert within_tolerance(got, want, bits), f"call {call}"
    assert sage.device_status() == 0


def test_noalloc_rejects_oversized_shapes():
    # validation happens before any device call: fake, aligned pointers
    qb.build()
    lib = sage.library()
    fake = 0x10000
    B, H, N, d = 1, 64, 4096, 128                     # ~101 MB of scratch > 64 MiB
    s = lib.sage_attn_fwd_noalloc(fake, fake, fake, fake, 1, B, H, N, d, 0,
                                  ctypes.c_float(1 / math.sqrt(d)), 0, None)
    assert s == -2
    text = lib.sage_status_string(s).decode()
    assert "bytes of scratch" in text and str(64 << 20) in text
