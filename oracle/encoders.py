"""Scalar number-format encoders for the oracle (TEST INFRASTRUCTURE ONLY).

Formats (none is defined on the method pages beyond its name; the bit
layouts are the standard ones the names refer to):

* INT8, symmetric: code = clamp(rne(x / s), -127, 127).  SageAttention
  abstract ("8-bit attention") and the kernel-comparison blog, section "How
  SageAttention uses quantization for more throughput" (Q/K to INT8).
* E4M3 ("fn" variant: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
  no infinities, max finite 448, smallest subnormal 2^-9).  SageAttention2
  abstract: P~ and V to FP8.
* E2M1 (1 sign, 2 exponent bits with bias 1, 1 mantissa bit; grid
  0, .5, 1, 1.5, 2, 3, 4, 6).  SageAttention3 abstract: FP4.
* UE4M3: E4M3 restricted to non-negative values, used for the FP4 block
  scale factors.

Reading taken: every cast rounds to nearest with ties to even and
saturates to the largest finite value (no NaN/Inf is produced; non-finite
inputs are not supported and rejected).  A result that rounds to zero keeps
the sign of its input (so -tiny encodes as the negative-zero code).

Each format has two independent encoders: an arithmetic one (binade +
quantum, used by the oracle) and a brute-force nearest-grid-point one
(used only by the pins in ``tests/``).
"""

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0
INT8_MAX = 127


def _finite64(x):
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input is not supported by the encoders")
    return x


def _binade(a):
    """floor(log2(a)) for a > 0, exactly (via frexp); 0 where a == 0."""
    _, ex = np.frexp(a)
    return np.where(a > 0, ex - 1, 0).astype(np.int64)


# --------------------------------------------------------------------------
# E4M3 (fn)
# --------------------------------------------------------------------------

def e4m3_round(x):
    """Round to the nearest E4M3 value (ties to even), saturating at +-448.

    Arithmetic encoder: the binade exponent is clamped at -6 (the subnormal
    binade shares the quantum 2^-9 with the first normal binade), the value
    is divided by the binade's quantum 2^(E-3), rounded half-to-even to an
    integer and scaled back.  All steps are exact in FP64.
    """
    x = _finite64(x)
    a = np.abs(x)
    e = np.maximum(_binade(a), -6)
    quantum = np.ldexp(1.0, e - 3)
    r = np.rint(a / quantum) * quantum
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(x):
    """E4M3 code byte (uint8) of rne_sat(x); sign bit copied from x."""
    x = _finite64(x)
    r = np.abs(e4m3_round(x))
    e = _binade(r)
    normal = r >= 2.0 ** -6
    exp_field = np.where(normal, e + 7, 0)
    mant = np.where(normal,
                    (r / np.ldexp(1.0, np.where(normal, e, 0)) - 1.0) * 8.0,
                    r / 2.0 ** -9)
    code = (exp_field.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    code = code | (np.signbit(x).astype(np.int64) << 7)
    return code.astype(np.uint8)


def e4m3_decode(code):
    """Value of an E4M3 code byte (float64).  0x7F / 0xFF (NaN) raise."""
    c = np.asarray(code, dtype=np.int64)
    if np.any((c & 0x7F) == 0x7F):
        raise ValueError("NaN code")
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(ef == 0, m * 2.0 ** -9,
                   np.ldexp(1.0 + m / 8.0, ef - 7))
    return sign * val


def e4m3_grid():
    """(codes, values) of all non-negative finite E4M3 codes 0x00..0x7E."""
    codes = np.arange(0x7F, dtype=np.int64)
    return codes, e4m3_decode(codes)


def e4m3_encode_bruteforce(x):
    """Independent encoder: nearest finite grid point, ties to the even code.

    Searches all 127 non-negative finite codes for the one nearest to |x|;
    between two equally near codes the one with an even mantissa LSB wins.
    The largest finite value is also the nearest finite value to anything
    above it, so saturation needs no special case.
    """
    x = _finite64(x)
    codes, vals = e4m3_grid()
    # beyond twice the largest value the nearest point is the largest value;
    # clipping there keeps every distance exact in FP64
    a = np.minimum(np.abs(x), 2 * E4M3_MAX).reshape(-1, 1)
    dist = np.abs(a - vals.reshape(1, -1))
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # prefer an even code among the (at most two) nearest ones
    even = cand & ((codes.reshape(1, -1) & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    code = codes[pick] | (np.signbit(x).reshape(-1).astype(np.int64) << 7)
    return code.astype(np.uint8).reshape(np.shape(x))


# --------------------------------------------------------------------------
# E2M1
# --------------------------------------------------------------------------

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_round(x):
    """Round to the nearest E2M1 value (ties to even), saturating at +-6."""
    x = _finite64(x)
    a = np.abs(x)
    e = np.maximum(_binade(a), 0)
    quantum = np.ldexp(1.0, e - 1)
    r = np.rint(a / quantum) * quantum
    r = np.minimum(r, E2M1_MAX)
    return np.copysign(r, x)


def e2m1_encode(x):
    """4-bit E2M1 code (uint8 in 0..15) of rne_sat(x); sign bit = bit 3."""
    x = _finite64(x)
    r = np.abs(e2m1_round(x))
    e = _binade(r)
    normal = r >= 1.0
    exp_field = np.where(normal, e + 1, 0)
    mant = np.where(normal, (r / np.ldexp(1.0, np.where(normal, e, 0)) - 1.0) * 2.0,
                    r * 2.0)
    code = (exp_field.astype(np.int64) << 1) | np.rint(mant).astype(np.int64)
    code = code | (np.signbit(x).astype(np.int64) << 3)
    return code.astype(np.uint8)


def e2m1_decode(code):
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x8, -1.0, 1.0)
    return sign * E2M1_VALUES[c & 0x7]


def e2m1_encode_bruteforce(x):
    """Independent encoder: nearest of the 8 grid values, ties to even code."""
    x = _finite64(x)
    codes = np.arange(8, dtype=np.int64)
    a = np.minimum(np.abs(x), 2 * E2M1_MAX).reshape(-1, 1)
    dist = np.abs(a - E2M1_VALUES.reshape(1, -1))
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & ((codes.reshape(1, -1) & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    code = codes[pick] | (np.signbit(x).reshape(-1).astype(np.int64) << 3)
    return code.astype(np.uint8).reshape(np.shape(x))


# --------------------------------------------------------------------------
# UE4M3 (block scale factors): E4M3 on non-negative values
# --------------------------------------------------------------------------

def ue4m3_encode(x):
    x = _finite64(x)
    if np.any(x < 0):
        raise ValueError("UE4M3 takes non-negative values")
    return e4m3_encode(np.abs(x))  # abs() drops a -0.0 sign


def ue4m3_decode(code):
    return e4m3_decode(np.asarray(code, dtype=np.int64) & 0x7F)


# --------------------------------------------------------------------------
# INT8 symmetric
# --------------------------------------------------------------------------

def int8_quantize(x, s):
    """clamp(rne(fp32(x / s)), -127, 127) with an IEEE FP32 division.

    ``x`` and ``s`` are float32 (broadcastable); where s == 0 the code is 0.
    """
    x = np.asarray(x, dtype=np.float32)
    s = np.asarray(s, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(s != 0, x / np.where(s != 0, s, np.float32(1)), np.float32(0))
    t = t.astype(np.float32)
    return np.clip(np.rint(t), -INT8_MAX, INT8_MAX).astype(np.int8)


# --------------------------------------------------------------------------
# 16-bit input formats
# --------------------------------------------------------------------------

def bf16_round(x):
    """Round float32 values to bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def f16_round(x):
    """Round to IEEE binary16 (ties to even); returns float32."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def round_to_dtype(x, dtype):
    """Round FP64/FP32 values to 'bf16' or 'f16' with ties to even.

    Goes through float32 only when that step is exact for the final result:
    the FP64 value is first rounded to float32 with round-to-odd so that the
    second rounding to 16 bits cannot double-round.
    """
    x64 = np.asarray(x, dtype=np.float64)
    x32 = x64.astype(np.float32)
    # round-to-odd correction: if the float32 rounding was inexact, force the
    # last float32 mantissa bit to 1 (sticky) toward the true value.
    back = x32.astype(np.float64)
    inexact = back != x64
    u = np.ascontiguousarray(x32).view(np.uint32).copy()
    toward_zero = np.abs(back) > np.abs(x64)
    # step toward zero by one ulp where float32 rounding went away from zero
    u = np.where(inexact & toward_zero & (u & 1 == 0), u - 1, u)
    u = np.where(inexact & ~toward_zero & (u & 1 == 0), u + 1, u)
    x32 = u.astype(np.uint32).view(np.float32)
    if dtype == "bf16":
        return bf16_round(x32)
    if dtype == "f16":
        return f16_round(x32)
    raise ValueError(dtype)
