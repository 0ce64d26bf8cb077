"""Pins of the oracle's number-format encoders (CPU only).

Each arithmetic encoder is checked exhaustively over every finite fp16 and
bf16 input against an independent brute-force nearest-grid encoder, against
points that the format definitions fix, and (in range) against torch's own
float8_e4m3fn cast.
"""

import numpy as np
import pytest
import torch

from oracle import encoders as enc


def all_f16():
    x = np.arange(1 << 16, dtype=np.uint16).view(np.float16).astype(np.float32)
    return x[np.isfinite(x)]


def all_bf16():
    u = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    return u[np.isfinite(u)]


@pytest.mark.parametrize("gen", [all_f16, all_bf16])
def test_e4m3_matches_bruteforce_exhaustive(gen):
    x = gen()
    a = enc.e4m3_encode(x)
    b = enc.e4m3_encode_bruteforce(x)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("gen", [all_f16, all_bf16])
def test_e2m1_matches_bruteforce_exhaustive(gen):
    x = gen()
    assert np.array_equal(enc.e2m1_encode(x), enc.e2m1_encode_bruteforce(x))


def test_e4m3_in_range_matches_torch_cast():
    # torch's float8_e4m3fn cast rounds to nearest-even; beyond 448 it does not
    # saturate, so compare only inside the finite range.
    x = all_f16()
    x = x[np.abs(x) <= 448.0]
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(enc.e4m3_encode(x), t)


def test_e4m3_fixed_points():
    assert enc.e4m3_decode(0x7E) == 448.0
    assert enc.e4m3_decode(0x01) == 2.0 ** -9
    assert enc.e4m3_decode(0x08) == 2.0 ** -6
    assert enc.e4m3_encode(np.float32(1e6)) == 0x7E          # saturates
    assert enc.e4m3_encode(np.float32(-1e6)) == 0xFE
    assert enc.e4m3_encode(np.float32(464.0)) == 0x7E        # tie above max
    assert enc.e4m3_encode(np.float32(2.0 ** -10)) == 0x00   # tie -> even (0)
    assert enc.e4m3_encode(np.float32(3 * 2.0 ** -10)) == 0x02  # tie -> even (2^-8)
    assert enc.e4m3_encode(np.float32(-2.0 ** -12)) == 0x80  # keeps the sign
    assert enc.e4m3_round(np.float32(1.0625)) == 1.0         # tie -> even mantissa
    assert enc.e4m3_round(np.float32(1.1875)) == 1.25


def test_e4m3_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = enc.e4m3_decode(codes)
    assert np.array_equal(enc.e4m3_encode(vals), codes)


def test_e4m3_relative_error_bound():
    x = all_f16()
    x = x[(np.abs(x) >= 2.0 ** -6) & (np.abs(x) <= 448.0)]
    r = enc.e4m3_round(x)
    assert np.all(np.abs(r - x) <= np.abs(x) * 2.0 ** -4)


def test_e2m1_fixed_points():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for i, g in enumerate(grid):
        assert enc.e2m1_encode(np.float32(g)) == i
        assert enc.e2m1_encode(np.float32(-g)) == i | 8
    for x, want in [(2.5, 2.0), (5.0, 4.0), (0.25, 0.0), (0.75, 1.0), (1.25, 1.0),
                    (1.75, 2.0), (3.5, 4.0), (100.0, 6.0), (-7.0, -6.0)]:
        assert enc.e2m1_decode(enc.e2m1_encode(np.float32(x))) == want, x


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(enc.e2m1_encode(enc.e2m1_decode(codes)), codes)


def test_e2m1_half_step_bound():
    x = all_f16()
    x = x[np.abs(x) <= 6.0]
    r = enc.e2m1_round(x)
    step = np.where(np.abs(x) < 2, 0.5, np.where(np.abs(x) < 4, 1.0, 2.0))
    assert np.all(np.abs(r - x) <= step / 2)


def test_ue4m3_rejects_negative():
    with pytest.raises(ValueError):
        enc.ue4m3_encode(np.float32(-1.0))
    assert enc.ue4m3_encode(np.float32(-0.0)) == 0


def test_int8_quantize_bounds_and_ties():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * 3).astype(np.float32)
    s = np.float32(np.abs(x).max() / np.float32(127))
    q = enc.int8_quantize(x, s)
    assert q.min() >= -127 and q.max() <= 127
    # |x - q s| <= s/2 up to the FP32 rounding of x/s
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * float(s))
    assert np.all(err <= float(s) * (0.5 + 1e-6))
    assert np.abs(q).max() == 127
    # ties to even
    assert enc.int8_quantize(np.float32(2.5), np.float32(1)) == 2
    assert enc.int8_quantize(np.float32(-3.5), np.float32(1)) == -4
    assert enc.int8_quantize(np.float32(5.0), np.float32(0)) == 0


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(200000) * 10 ** rng.uniform(-5, 5, 200000)).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(enc.bf16_round(x), t)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_round_to_dtype_single_rounding(dtype):
    # Reference: round the FP64 value directly to the 16-bit format's number of
    # significant bits (rint on the exactly scaled significand), i.e. one
    # rounding, no float32 step.
    rng = np.random.default_rng(2)
    x = rng.standard_normal(20000) * 4
    base = enc.round_to_dtype(x, dtype).astype(np.float64)
    bits = 8 if dtype == "bf16" else 11
    ulp = np.ldexp(1.0, np.frexp(base)[1] - bits)
    # values just off 16-bit ties, where a double rounding through float32 fails
    y = np.concatenate([x, base + ulp * (0.5 + 2.0 ** -30), base - ulp * (0.5 + 2.0 ** -30),
                        base + ulp * 0.5, base - ulp * 0.5])
    r = enc.round_to_dtype(y, dtype).astype(np.float64)
    m, e = np.frexp(y)
    want = np.ldexp(np.rint(np.ldexp(m, bits)), e - bits)
    assert np.array_equal(r, want)
