"""Seeded synthetic workloads (shapes, value distributions, seeds).

This module only draws random numbers and casts them to the input dtype; it
holds none of the attention method's arithmetic, so the CUDA path, the tests
and the CPU oracle can all take their inputs from it.

Each (b, h) head is drawn from its own PCG64 stream seeded by
SeedSequence([seed, b, h]), so any subset of heads can be regenerated alone
(used to check large workloads against the oracle on sampled heads).

Distributions (normal laws written N(0, sigma); the K bias is one value per
(b, h, channel) added to every token of K):

  tiny   Q, V ~ N(0,1); K ~ N(0,1) + bias, bias ~ N(0,3)
  llm    Q, K ~ N(0,1) with 4 random channels per head scaled by 20 in both
         Q and K (the same channel set for Q and K of a head);
         bias ~ N(0,2); V ~ N(0,1)
  short  as llm (a batch of 1024-token sequences)
  video  Q, K, V ~ N(0,1); bias ~ N(0,4)
  long   Q, K, V ~ Student-t(nu=4) / sqrt(2) (unit variance); bias ~ N(0,2)
  fp4    Q, K ~ N(0,1); bias ~ N(0,3); V ~ N(0,1)
  n16k   the fp4 laws and shape in the 8-bit modes
"""

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dtype: str          # "bf16" or "f16"
    mode: str           # "int8_fp8" or "fp4"
    seed: int
    dist: str           # "normal", "llm_outliers", "student_t"
    k_bias_sigma: float

    @property
    def sm_scale(self):
        return 1.0 / float(np.sqrt(self.d))

    @property
    def ops(self):
        """Effective operation count 4*B*H*N^2*d (the throughput numerator)."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, False, "f16", "int8_fp8", 0, "normal", 3.0),
    "llm": Workload("llm", 1, 32, 4096, 128, True, "bf16", "int8_fp8", 1, "llm_outliers", 2.0),
    "video": Workload("video", 2, 24, 16384, 64, False, "bf16", "int8_fp8", 2, "normal", 4.0),
    "long": Workload("long", 1, 16, 32768, 128, False, "bf16", "int8_fp8", 3, "student_t", 2.0),
    "long_causal": Workload("long_causal", 1, 16, 32768, 128, True, "bf16", "int8_fp8", 3,
                            "student_t", 2.0),
    "fp4": Workload("fp4", 2, 32, 16384, 128, False, "bf16", "fp4", 4, "normal", 3.0),
    # the long-context inputs through the FP8 Q/K mode
    "long_fp8": Workload("long_fp8", 1, 16, 32768, 128, False, "bf16", "fp8", 3, "student_t",
                         2.0),
    "llm_fp8": Workload("llm_fp8", 1, 32, 4096, 128, True, "bf16", "fp8", 1, "llm_outliers", 2.0),
    # a batch of short LLM prefills (the llm value laws), 200 MB of inputs
    "short": Workload("short", 8, 32, 1024, 128, True, "bf16", "int8_fp8", 5, "llm_outliers", 2.0),
    # the fp4 shape and value laws (16k tokens, d = 128, non-causal) through
    # the 8-bit modes: INT8 Q/K (and FP8 Q/K) with FP8 P~ and V
    "n16k": Workload("n16k", 2, 32, 16384, 128, False, "bf16", "int8_fp8", 6, "normal", 3.0),
    "n16k_fp8": Workload("n16k_fp8", 2, 32, 16384, 128, False, "bf16", "fp8", 6, "normal", 3.0),
}


def head_rng(seed, b, h):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, b, h])))


def draw_head(w: Workload, b: int, h: int):
    """float32 (q, k, v) [N, d] for head (b, h), before the dtype cast."""
    rng = head_rng(w.seed, b, h)
    shape = (w.N, w.d)
    if w.dist == "student_t":
        q = rng.standard_t(4.0, size=shape) / np.sqrt(2.0)
        k = rng.standard_t(4.0, size=shape) / np.sqrt(2.0)
        v = rng.standard_t(4.0, size=shape) / np.sqrt(2.0)
    else:
        q = rng.standard_normal(shape, dtype=np.float32)
        k = rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
    bias = rng.standard_normal(w.d, dtype=np.float32) * np.float32(w.k_bias_sigma)
    if w.dist == "llm_outliers":
        ch = rng.choice(w.d, size=4, replace=False)
        q[:, ch] *= 20.0
        k[:, ch] *= 20.0
    k = k + bias[None, :]
    return (np.asarray(q, np.float32), np.asarray(k, np.float32), np.asarray(v, np.float32))


def _cast(x, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float16)


def make_qkv(w: Workload, heads=None):
    """CPU torch tensors (q, k, v) of shape [B, H, N, d] in the workload dtype.

    heads: optional list of (b, h) pairs; then the tensors have shape
    [len(heads), 1, N, d] (one sampled head per row, same values as in the
    full tensor).
    """
    import torch
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        out_shape = (w.B, w.H, w.N, w.d)
    else:
        out_shape = (len(heads), 1, w.N, w.d)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    q = torch.empty((len(heads), w.N, w.d), dtype=dt)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for i, (b, h) in enumerate(heads):
        qh, kh, vh = draw_head(w, b, h)
        q[i] = _cast(qh, w.dtype)
        k[i] = _cast(kh, w.dtype)
        v[i] = _cast(vh, w.dtype)
    return q.view(out_shape), k.view(out_shape), v.view(out_shape)


def to_numpy32(t):
    """float32 NumPy copy of a CPU/GPU torch tensor (exact for bf16/f16)."""
    return t.detach().float().cpu().numpy()
