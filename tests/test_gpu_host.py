"""The host-buffer forward pass (sage_attn_fwd_host): heads cut into chunks
whose copies in and out overlap the compute of their neighbours.  Heads are
independent, so the result must equal sage_attn_fwd's bit for bit, whatever
the chunking (one chunk, several, a short last one), the mode, the mask, a
ragged N, Q smoothing, and pinned or pageable host memory."""

import numpy as np
import pytest
import torch

import quantized_attention_quant_b200 as sage
from tests.test_gpu_prepass import rand_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d,mode,causal,smooth", [
    (2, 3, 1000, 128, "int8_fp8", True, False),      # one chunk
    (1, 40, 4096, 128, "int8_fp8", False, False),    # four chunks of 10 heads
    (1, 45, 4000, 128, "fp8", True, False),          # ragged N, a short last chunk
    (1, 45, 4096, 128, "fp4", False, False),
    (1, 24, 4096, 64, "int8_fp8", True, True),       # d = 64, Q smoothing
    (1, 40, 4096, 128, "fp4", False, True),
])
def test_host_pass_equals_device_pass(cuda_device, B, H, N, d, mode, causal, smooth):
    q, k, v = rand_qkv(B, H, N, d, "bf16", seed=1000 + H + N)
    want = sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode=mode,
                              smooth_q=smooth).cpu()
    for pinned in (True, False):
        qh, kh, vh = ((t.pin_memory() if pinned else t.clone()) for t in (q, k, v))
        got = sage.sage_attn_fwd_host(qh, kh, vh, causal=causal, mode=mode, smooth_q=smooth)
        assert sage.device_status() == 0
        assert torch.equal(got, want), (pinned, (got.float() - want.float()).abs().max())


def test_host_pass_twice_and_after_other_work(cuda_device):
    # consecutive calls reuse the copy streams and their events; a device pass
    # in between on the same stream uses the same workspace
    q, k, v = (t.pin_memory() for t in rand_qkv(1, 40, 4096, 128, "bf16", seed=7))
    a = sage.sage_attn_fwd_host(q, k, v)
    d = sage.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda()).cpu()
    b = sage.sage_attn_fwd_host(q, k, v)
    assert torch.equal(a, d) and torch.equal(b, d)
