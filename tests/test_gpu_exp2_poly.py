"""The FMA-pipe exponential of the attention kernels (exp2_poly.cuh: a rint
split, a degree-4 Remez polynomial on [-1/2, 1/2], the integer part added to
the exponent field) evaluated on the GPU and held to its stated relative
error, 2^-18.5, against FP64 exp2 over the whole argument range the kernels
use, including the integer points and the half-integer split points."""

import ctypes

import numpy as np
import pytest

from quantized_attention_quant_b200 import build as qb

pytestmark = pytest.mark.gpu


def test_exp2_poly_relative_error(cuda_device):
    qb.build()
    ub = ctypes.CDLL(qb.UBENCH_LIB)
    ub.sage_ubench_exp2_poly.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    rng = np.random.default_rng(3)
    t = np.concatenate([
        rng.uniform(-125.0, 9.0, 1 << 20),                    # the range of t - m + log2 448
        np.arange(-125, 10, dtype=np.float64),                # integers
        np.arange(-125, 10, dtype=np.float64) + 0.5,          # split points of rint
        np.arange(-124, 10, dtype=np.float64) - 0.5,
        np.nextafter(np.arange(-124, 10, dtype=np.float32) + np.float32(0.5), np.float32(-1e9)),
    ]).astype(np.float32)
    assert t.min() >= -125.0                                  # below, the clamp (checked last)
    out = np.empty_like(t)
    assert ub.sage_ubench_exp2_poly(t.ctypes.data, out.ctypes.data, t.size) == 0
    exact = np.exp2(t.astype(np.float64))
    rel = np.abs(out.astype(np.float64) - exact) / exact
    assert rel.max() <= 2.0 ** -18.5, (rel.max(), t[rel.argmax()])
    # arguments below -125 take the clamp: 2^-125 exactly up to the same bound
    low = np.array([-126.0, -200.0, -1e30], np.float32)
    out_low = np.empty_like(low)
    assert ub.sage_ubench_exp2_poly(low.ctypes.data, out_low.ctypes.data, low.size) == 0
    assert np.all(np.abs(out_low / 2.0 ** -125 - 1.0) <= 2.0 ** -18.5)
