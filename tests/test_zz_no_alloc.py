"""The no-allocation entry point (sage_attn_fwd_noalloc).

Callers that cannot allocate device memory while they run -- a memory pool
that admits no new allocations, an allocator that owns the whole device, a
caller that may not take the driver's allocation locks -- use this variant:
its scratch is a fixed array inside the library's device image.  These tests
check, through the C ABI, that it gives the same bits as sage_attn_fwd (both
run the same kernels on the same inputs, only the scratch differs) on two
calls in a row (the second call reuses the array the first one left
behind), that the result meets the oracle's parity bar, and that a shape too
large for the array is refused.  The shapes cover both pre-pass launch forms
(the cluster-fused one for short sequences of few heads, the two-launch
chains with their per-head counters otherwise), every mode, and a ragged N.

The file is named so that pytest collects it last.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import quantized_attention_quant_b200 as sage
from quantized_attention_quant_b200 import build as qb
from quantized_attention_quant_b200.workloads import to_numpy32
from tests.test_gpu_attention import check_against_oracle
from tests.test_gpu_prepass import rand_qkv

# (B, H, N, d, causal, dtype, mode); B*H <= 16 and N <= 1024 in an 8-bit mode
# take the cluster-fused pre-pass, the rest the two-launch chains
CASES = [
    (1, 4, 512, 128, True, "bf16", "int8_fp8"),     # fused pre-pass
    (1, 4, 512, 64, False, "f16", "int8_fp8"),      # fused pre-pass, d = 64
    (1, 32, 2048, 128, False, "bf16", "int8_fp8"),  # chains
    (1, 32, 2048, 128, True, "bf16", "fp8"),        # chains, FP8 Q/K
    (1, 32, 2048, 128, False, "bf16", "fp4"),       # FP4 (always chained)
    (1, 17, 1000, 128, False, "f16", "int8_fp8"),   # chains, ragged N, 17 heads
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal,dtype,mode", CASES)
def test_noalloc_equals_sage_attn_fwd_twice(cuda_device, B, H, N, d, causal, dtype, mode):
    rows = np.unique(np.r_[0, 1, 127, 128, N // 2, N - 1,
                           np.random.default_rng(N + H).integers(0, N, 10)])
    for call, seed in enumerate((11, 12)):                 # two calls in a row
        q, k, v = rand_qkv(B, H, N, d, dtype, seed=seed * 1000 + N + H + d)
        dq, dk, dv = (t.cuda() for t in (q, k, v))
        out = torch.empty_like(dq)
        got = sage.sage_attn_fwd_noalloc(dq, dk, dv, causal=causal, mode=mode, out=out)
        want = sage.sage_attn_fwd(dq, dk, dv, causal=causal, mode=mode)
        torch.cuda.synchronize()
        assert sage.device_status() == 0
        assert got.data_ptr() == out.data_ptr()
        assert torch.equal(got, want), f"call {call}: differs from sage_attn_fwd"
        # and the shared result meets the parity bar on sampled rows of two heads
        hs = [0, H - 1]
        check_against_oracle(to_numpy32(got)[:, hs][:, :, rows], q[:, hs], k[:, hs], v[:, hs],
                             causal, 1 / math.sqrt(d), mode, dtype, rows=rows)


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
