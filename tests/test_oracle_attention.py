"""Pins of the oracle's pre-pass and attention (CPU only).

Exact attention is pinned against a pure-Python triple loop, closed forms
and invariants; the emulated path is pinned by reducing to exact attention
with identity quantizers, by closed forms whose every quantizer step is
exact, and by exact scaling laws.
"""

import math

import numpy as np
import pytest

from oracle import attention as att
from oracle import encoders as enc
from oracle import prepass as pp


def rnd(shape, seed, scale=1.0, dtype="bf16"):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * np.float32(scale)
    return enc.bf16_round(x) if dtype == "bf16" else enc.f16_round(x)


def brute_attention(q, k, v, causal, sm_scale):
    """softmax(q k^T sm_scale) v with Python scalars, one (b, h)."""
    N, d = len(q), len(q[0])
    out = []
    for i in range(N):
        keys = [j for j in range(N) if (j <= i or not causal)]
        s = [sum(float(q[i][c]) * float(k[j][c]) for c in range(d)) * sm_scale for j in keys]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        z = math.fsum(w)
        out.append([math.fsum(w[t] * float(v[j][c]) for t, j in enumerate(keys)) / z
                    for c in range(d)])
    return np.array(out)


# ---------------------------------------------------------------- exact ----

@pytest.mark.parametrize("causal", [False, True])
def test_exact_matches_bruteforce(causal):
    q, k, v = rnd((1, 2, 13, 5), 1), rnd((1, 2, 13, 5), 2), rnd((1, 2, 13, 5), 3)
    o = att.exact_attention(q, k, v, causal, 0.37)
    for h in range(2):
        ref = brute_attention(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), causal, 0.37)
        assert np.max(np.abs(o[0, h] - ref)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_exact_rows_sum_to_one(causal):
    q, k = rnd((2, 1, 300, 16), 4, 3.0), rnd((2, 1, 300, 16), 5, 3.0)
    o = att.exact_attention(q, k, np.ones((2, 1, 300, 16)), causal, 0.25, row_chunk=97)
    assert np.max(np.abs(o - 1.0)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_exact_zero_q_gives_visible_mean(causal):
    v = rnd((1, 1, 50, 8), 6)
    o = att.exact_attention(np.zeros((1, 1, 50, 8)), rnd((1, 1, 50, 8), 7), v, causal, 1.0)
    v64 = v[0, 0].astype(np.float64)
    if causal:
        want = np.cumsum(v64, axis=0) / np.arange(1, 51)[:, None]
    else:
        want = np.broadcast_to(v64.mean(axis=0), (50, 8))
    assert np.max(np.abs(o[0, 0] - want)) <= 1e-12


def test_exact_dominant_key_selects_its_value():
    N, d = 40, 8
    k = rnd((1, 1, N, d), 8, 0.01)
    q = np.zeros((1, 1, N, d), np.float32)
    q[..., 0] = 1.0
    k[0, 0, 17, 0] = 1000.0
    v = rnd((1, 1, N, d), 9)
    o = att.exact_attention(q, k, v, False, 1.0)
    assert np.max(np.abs(o[0, 0] - v[0, 0, 17][None, :].astype(np.float64))) <= 1e-12


def test_exact_key_permutation_equivariance():
    q, k, v = rnd((1, 2, 64, 16), 10), rnd((1, 2, 64, 16), 11), rnd((1, 2, 64, 16), 12)
    perm = np.random.default_rng(0).permutation(64)
    a = att.exact_attention(q, k, v, False, 0.25)
    b = att.exact_attention(q, k[:, :, perm], v[:, :, perm], False, 0.25)
    assert np.max(np.abs(a - b)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_exact_k_shift_invariance(causal):
    # the smoothing invariant: K + 1 c^T leaves O unchanged
    q, k, v = rnd((1, 1, 96, 16), 13), rnd((1, 1, 96, 16), 14), rnd((1, 1, 96, 16), 15)
    c = np.random.default_rng(1).standard_normal(16) * 5
    a = att.exact_attention(q, k, v, causal, 0.25)
    b = att.exact_attention(q, k.astype(np.float64) + c, v, causal, 0.25)
    assert np.max(np.abs(a - b)) <= 1e-12


# ------------------------------------------------------------- pre-pass ----

def test_k_mean_is_the_mean():
    k = rnd((2, 3, 300, 32), 16, 4.0)
    mu = pp.k_channel_mean(k)
    for b in range(2):
        for h in range(3):
            for c in range(0, 32, 7):
                exact = math.fsum(float(x) for x in k[b, h, :, c]) / 300
                assert abs(float(mu[b, h, c]) - exact) <= abs(exact) * 2.0 ** -24 + 1e-30


def test_k_mean_chunk_order():
    # the FP64 sum is taken per 128-token chunk in token order, then over
    # chunks; a set of values whose sum depends on the order pins that order
    N = 256
    k = np.zeros((1, 1, N, 1), np.float64)
    k[0, 0, 0, 0] = 2.0 ** 60
    k[0, 0, 1, 0] = 1.0
    k[0, 0, 128, 0] = -(2.0 ** 60)
    # in token order over all N the 1.0 is absorbed; chunk-wise it is too
    # (2^60 + 1 rounds to 2^60 inside chunk 0), so the mean is 0
    assert pp.k_channel_mean(k)[0, 0, 0] == 0.0
    k[0, 0, 1, 0] = 0.0
    k[0, 0, 129, 0] = 1.0
    # chunk 1 sums to -2^60 exactly (+1 absorbed), total 0
    assert pp.k_channel_mean(k)[0, 0, 0] == 0.0
    k[0, 0, 129, 0] = 0.0
    k[0, 0, 130, 0] = 2.0 ** 60
    k[0, 0, 131, 0] = 3.0
    # chunk 1: -2^60 + 2^60 + 3 = 3 exactly; chunk 0: 2^60; total 2^60 + 3 -> 2^60
    assert pp.k_channel_mean(k)[0, 0, 0] == np.float32(2.0 ** 60 / N)


def test_int8_blocks_properties():
    x = rnd((1, 2, 300, 64), 17, 2.0)
    x[0, 1, 128:256] = 0.0                               # an all-zero block
    codes, scales = pp.quant_int8_blocks(x)
    assert scales.shape == (1, 2, 3)
    assert scales[0, 1, 1] == 0 and np.all(codes[0, 1, 128:256] == 0)
    for h in range(2):
        for i, (s, e) in enumerate([(0, 128), (128, 256), (256, 300)]):
            blk = x[0, h, s:e].astype(np.float64)
            sc = float(scales[0, h, i])
            if sc == 0:
                continue
            assert np.abs(codes[0, h, s:e]).max() == 127
            assert np.all(np.abs(blk - codes[0, h, s:e] * sc) <= sc * (0.5 + 1e-6))
            assert scales[0, h, i] == np.float32(np.float32(np.abs(blk).max()) / np.float32(127))


@pytest.mark.parametrize("tokens", [1, 32])
def test_int8_blocks_small_groups(tokens):
    # the block rule holds for any group size: one scale per `tokens` tokens
    # (the last group of a ragged head shorter), amax / 127, codes within
    # half a step, the group max on +-127
    x = rnd((1, 2, 77, 64), 117 + tokens, 2.0)
    x[0, 1, 32:64] = 0.0                                 # zero groups
    codes, scales = pp.quant_int8_blocks(x, tokens)
    assert scales.shape == (1, 2, -(-77 // tokens))
    for h in range(2):
        for i in range(scales.shape[2]):
            s, e = i * tokens, min((i + 1) * tokens, 77)
            blk = x[0, h, s:e].astype(np.float64)
            sc = float(scales[0, h, i])
            if np.abs(blk).max() == 0:
                assert sc == 0 and np.all(codes[0, h, s:e] == 0)
                continue
            assert np.abs(codes[0, h, s:e]).max() == 127
            # the code is decided on the FP32 quotient, which may sit up to
            # 127 * 2^-24 past a half step
            assert np.all(np.abs(blk - codes[0, h, s:e] * sc) <= sc * (0.5 + 128 * 2.0 ** -24))


def test_int8_qk_scales_pinned():
    """Q takes one scale per token, smoothed K one per 32 tokens: planted
    values make every scale and code a closed form.  Token t of Q has amax
    127 * 2^e_t.  K is planted in (+x, -x) token pairs of one channel, so
    every channel mean is exactly 0 and smoothing changes nothing; its
    32-token block b has amax 127 * 2^f_b and its other values are
    +-60 * 2^f_b.  A 128-token Q block, a 128-token or per-token K block, or
    a 126 divisor each break the closed form."""
    N, d = 128, 16
    q = np.zeros((1, 1, N, d), np.float32)
    k = np.zeros((1, 1, N, d), np.float32)
    eq = (np.arange(N) % 7) - 3                          # per-token exponents -3..3
    ek = np.array([-2, 1, 0, 3])                         # per-32-token-block exponents
    want_qc = np.zeros((N, d), np.int8)
    want_kc = np.zeros((N, d), np.int8)
    for t in range(N):
        c = t % d
        q[0, 0, t, c] = 127.0 * 2.0 ** eq[t]
        q[0, 0, t, (c + 5) % d] = -45.0 * 2.0 ** eq[t]
        want_qc[t, c], want_qc[t, (c + 5) % d] = 127, -45
        ck = (t // 2) % d
        mag = 127 if t % 32 in (4, 5) else 60
        sgn = 1 if t % 2 == 0 else -1
        k[0, 0, t, ck] = sgn * mag * 2.0 ** ek[t // 32]
        want_kc[t, ck] = sgn * mag
    r = pp.quant_qk_int8(q, k)
    assert np.all(r["k_mean"] == 0)
    assert r["q_scales"].shape == (1, 1, N) and r["k_scales"].shape == (1, 1, 4)
    np.testing.assert_array_equal(r["q_scales"][0, 0], (2.0 ** eq).astype(np.float32))
    np.testing.assert_array_equal(r["q_codes"][0, 0], want_qc)
    np.testing.assert_array_equal(r["k_scales"][0, 0], (2.0 ** ek).astype(np.float32))
    np.testing.assert_array_equal(r["k_codes"][0, 0], want_kc)


def test_quant_qk_smooths_k_only():
    q, k = rnd((1, 1, 256, 32), 18), rnd((1, 1, 256, 32), 19) + np.float32(10)
    r = pp.quant_qk_int8(q, k)
    c2, s2 = pp.quant_int8_blocks(q, 1)
    assert np.array_equal(r["q_codes"], c2) and np.array_equal(r["q_scales"], s2)
    kc, ks = pp.quant_int8_blocks(k.astype(np.float32) - r["k_mean"][:, :, None, :], 32)
    assert np.array_equal(r["k_codes"], kc) and np.array_equal(r["k_scales"], ks)
    assert np.all(np.abs(r["k_mean"] - 10) < 0.5)
    assert r["q_scales"].shape == (1, 1, 256) and r["k_scales"].shape == (1, 1, 8)


def test_query_rows_quantized_independently():
    # one scale per query token: a huge value planted in one query row
    # changes no other row's codes or output (bit for bit)
    q, k, v = rnd((1, 1, 256, 32), 30), rnd((1, 1, 256, 32), 31), rnd((1, 1, 256, 32), 32)
    o = att.emulated_sage_attention(q, k, v, True, 0.2)
    q2 = q.copy()
    q2[0, 0, 100, 3] = np.float32(1000.0)
    o2 = att.emulated_sage_attention(q2, k, v, True, 0.2)
    rows = np.arange(256) != 100
    assert np.array_equal(o[0, 0, rows], o2[0, 0, rows])
    assert not np.array_equal(o[0, 0, 100], o2[0, 0, 100])


def test_fp8_v_properties():
    v = rnd((1, 2, 256, 32), 20, 3.0)
    v[0, 0, :, 5] = 0.0
    codes, s = pp.quant_v_fp8(v)
    assert codes.shape == (1, 2, 32, 256) and s.shape == (1, 2, 32)
    assert s[0, 0, 5] == 0 and np.all(codes[0, 0, 5] == 0)
    vt = v.transpose(0, 1, 3, 2).astype(np.float64)
    deq = enc.e4m3_decode(codes) * s[..., None]
    for h in range(2):
        for c in range(32):
            if s[0, h, c] == 0:
                continue
            row = np.abs(vt[0, h, c])
            j = row.argmax()
            assert codes[0, h, c, j] & 0x7F == 0x7E          # the channel max hits 448
            big = row >= float(s[0, h, c]) * 2.0 ** -6
            err = np.abs(deq[0, h, c] - vt[0, h, c])
            assert np.all(err[big] <= row[big] * 2.0 ** -4 * (1 + 1e-6))


def test_fp8_v_scale_pinned():
    """s_V of a channel is amax over ALL N tokens of the head, over 448, and
    the codes follow from it: planted values make every expected scale and
    code a closed form.  Channel c's largest |V| is 448 * 2^e_c and sits in
    the second 128-token block, whose maximum differs from the first
    block's; the other planted values are 2^e_c times exact e4m3 grid
    points.  A 447 divisor, a per-block amax, or a max over the channel axis
    instead of the token axis each break the closed form."""
    N, d = 256, 8
    grid = np.array([96.0, -40.0, 13.0, 0.5, -2.0 ** -6, 2.0 ** -9], np.float64)  # e4m3 values
    codes_of = {96.0: 0x6C, -40.0: 0xE2, 13.0: 0x55, 0.5: 0x30, -2.0 ** -6: 0x88,
                2.0 ** -9: 0x01}
    for val, code in codes_of.items():                    # the grid points, decoded
        assert float(enc.e4m3_decode(np.array([code], np.uint8))[0]) == val
    v = np.zeros((1, 2, N, d), np.float32)
    expect_s = np.zeros((1, 2, d), np.float32)
    expect_codes = np.zeros((1, 2, d, N), np.uint8)
    for h in range(2):
        for c in range(d):
            e = c - 4 + 3 * h                                # scales 2^-4 .. 2^6
            s_c = 2.0 ** e
            expect_s[0, h, c] = s_c
            t_max = 128 + (37 * c + 11 * h) % 128            # in the second block
            v[0, h, t_max, c] = -448.0 * s_c if c % 2 else 448.0 * s_c
            expect_codes[0, h, c, t_max] = 0xFE if c % 2 else 0x7E
            for i, g in enumerate(grid):                     # first block: max 96 * s_c
                t = (5 * c + 3 * i) % 128
                v[0, h, t, c] = g * s_c
                expect_codes[0, h, c, t] = codes_of[g]
    # the per-channel scale is 2^e exactly, so every planted code is exact
    codes, s = pp.quant_v_fp8(v)
    assert s.dtype == np.float32
    np.testing.assert_array_equal(s.view(np.uint32), expect_s.view(np.uint32))
    np.testing.assert_array_equal(codes, expect_codes)
    # a value that is not a power of two times 448: s = fp32(amax / 448), the
    # correctly rounded quotient, checked against exact rational arithmetic
    from fractions import Fraction
    w = np.zeros((1, 1, N, 1), np.float32)
    w[0, 0, 200, 0] = np.float32(1000.0)
    w[0, 0, 10, 0] = np.float32(-3.0)
    _, s2 = pp.quant_v_fp8(w)
    q = Fraction(1000) / 448
    cand = [np.nextafter(s2[0, 0, 0], np.float32(-np.inf)), s2[0, 0, 0],
            np.nextafter(s2[0, 0, 0], np.float32(np.inf))]
    dist = [abs(Fraction(float(x)) - q) for x in cand]
    assert dist[1] < dist[0] and dist[1] < dist[2]


def test_fp4_tokens_properties():
    x = rnd((1, 1, 256, 64), 21, 2.0)
    codes, sf, g = pp.quant_fp4_tokens(x)
    assert codes.shape == (1, 1, 256, 64) and sf.shape == (1, 1, 256, 4) and g.shape == (1, 1, 2)
    for t in range(2):
        blk = x[0, 0, t * 128:(t + 1) * 128].astype(np.float64)
        r, c = np.unravel_index(np.abs(blk).argmax(), blk.shape)
        assert codes[0, 0, t * 128 + r, c] & 7 == 7                   # the tile max -> 6
        assert sf[0, 0, t * 128 + r, c // 16] == 0x7E                 # with scale 448
        assert g[0, 0, t] == np.float32(np.float32(np.abs(blk).max()) / np.float32(2688))
        den = (enc.ue4m3_decode(sf[0, 0, t * 128:(t + 1) * 128]).astype(np.float32)
               * g[0, 0, t]).astype(np.float32).astype(np.float64)
        den = np.repeat(den, 16, axis=1)
        deq = enc.e2m1_decode(codes[0, 0, t * 128:(t + 1) * 128]) * den
        sat = np.maximum(np.abs(blk) - 6 * den, 0)
        assert np.all(np.abs(deq - blk) <= den * (1 + 1e-6) + sat)


def test_fp4_v_layout_and_zero_channel():
    v = rnd((1, 1, 256, 32), 22)
    v[0, 0, :, 3] = 0.0
    codes, sf, g = pp.quant_v_fp4(v)
    assert codes.shape == (1, 1, 32, 256) and sf.shape == (1, 1, 32, 16)
    assert np.all(codes[0, 0, 3] == 0) and np.all(sf[0, 0, 3] == 0)
    # encoding V^T with the token routine on the transposed tile gives the same
    c2, s2, g2 = pp.quant_fp4_tokens(np.ascontiguousarray(v.transpose(0, 1, 3, 2))[:, :, :, :128]
                                     .transpose(0, 1, 3, 2).copy())
    assert g2[0, 0, 0] == g[0, 0, 0]


def test_integer_qk_is_exact():
    q = np.random.default_rng(3).integers(-127, 128, (128, 128))
    k = np.random.default_rng(4).integers(-127, 128, (128, 128))
    assert np.array_equal((q.astype(np.float64) @ k.T.astype(np.float64)).astype(np.int64),
                          q.astype(np.int64) @ k.T.astype(np.int64))


# ------------------------------------------------------------- emulated ----

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 384])
def test_emulated_identity_equals_exact(causal, N):
    q, k, v = rnd((1, 2, N, 16), 30, 2.0), rnd((1, 2, N, 16), 31, 2.0), rnd((1, 2, N, 16), 32)
    a = att.emulated_sage_attention(q, k, v, causal, 0.3, quantizers="identity")
    b = att.exact_attention(q, k, v, causal, 0.3)
    assert np.max(np.abs(a - b)) <= 1e-12


@pytest.mark.parametrize("N", [256, 200])
@pytest.mark.parametrize("mode", ["int8_fp8", "fp4"])
@pytest.mark.parametrize("causal", [False, True])
def test_emulated_constant_k_gives_visible_mean(mode, causal, N):
    # K rows all equal -> smoothed K = 0 -> all scores 0 -> P~ = 1 exactly;
    # V on the format grid with an exact scale -> O is the visible mean of V.
    # N = 200 ends in a partial tile (and, in FP4 mode, a partial 16-group).
    d = 32
    rng = np.random.default_rng(5)
    q = rnd((1, 1, N, d), 33)
    k = np.broadcast_to(rnd((1, 1, 1, d), 34), (1, 1, N, d)).copy()
    if mode == "int8_fp8":
        grid = enc.e4m3_decode(np.arange(0x7F))
        v = rng.choice(grid, (1, 1, N, d)) * rng.choice([-1, 1], (1, 1, N, d))
        v[0, 0, 0, :] = 448.0                        # channel max 448 -> s_V = 1
        tol = 1e-12
    else:
        grid = enc.E2M1_VALUES
        v = rng.choice(grid, (1, 1, N, d)) * rng.choice([-1, 1], (1, 1, N, d))
        v[0, 0, ::16, :] = 6.0                        # every 16-block holds 6
        tol = 1e-6                                    # g = 6/2688 is inexact in fp32
    v = v.astype(np.float32)
    o = att.emulated_sage_attention(q, k, v, causal, 0.2, mode=mode)
    v64 = v[0, 0].astype(np.float64)
    want = (np.cumsum(v64, axis=0) / np.arange(1, N + 1)[:, None]) if causal \
        else np.broadcast_to(v64.mean(axis=0), (N, d))
    assert np.max(np.abs(o[0, 0] - want)) <= tol * max(1.0, np.abs(want).max())


def test_emulated_two_key_closed_form():
    # One query direction, keys arranged so that exactly two keys matter with
    # P~ = 1 and 1/1.1; every quantizer step except P~ is exact, and P~ = 1/1.1
    # encodes as 448/1.1 = 407.27 -> 416.  l sums the unquantized P~.
    N, d = 128, 16
    q = np.zeros((1, 1, N, d), np.float32)
    q[..., 0] = 127.0                                   # s_Q = 1, codes 127
    k = np.zeros((1, 1, N, d), np.float32)
    kc = np.full(N, -2.0)
    kc[0], kc[1], kc[2] = 127.0, 126.0, -3.0            # channel sum 0 -> mean 0
    k[0, 0, :, 0] = kc
    sm_scale = math.log(1.1) / 127.0                    # S0 - S1 = ln 1.1
    rng = np.random.default_rng(6)
    grid = enc.e4m3_decode(np.arange(0x7F))
    v = (rng.choice(grid, (1, 1, N, d)) * rng.choice([-1, 1], (1, 1, N, d))).astype(np.float32)
    v[0, 0, 5, :] = 448.0                               # s_V = 1
    o = att.emulated_sage_attention(q, k, v, False, sm_scale)
    v0, v1 = v[0, 0, 0].astype(np.float64), v[0, 0, 1].astype(np.float64)
    p1 = math.exp(-math.log(1.1))
    others = sum(math.exp(127 * (x - 127.0) * sm_scale) for x in kc[2:])
    assert enc.e4m3_decode(enc.e4m3_encode(448 * p1)) == 416.0
    want = (v0 + (416.0 / 448.0) * v1) / (1.0 + p1 + others)
    # the other keys' P~ (< 1e-4) quantize to small nonzero codes; bound them
    rest = (np.abs(v[0, 0, 2:]).max() * others * 1.1)
    assert np.max(np.abs(o[0, 0] - want[None, :])) <= rest + 1e-12


def test_emulated_v_scaling_is_exact():
    q, k, v = rnd((1, 1, 256, 32), 40), rnd((1, 1, 256, 32), 41), rnd((1, 1, 256, 32), 42)
    for mode in ["int8_fp8", "fp4"]:
        a = att.emulated_sage_attention(q, k, v, False, 0.2, mode=mode)
        b = att.emulated_sage_attention(q, k, v * np.float32(8), False, 0.2, mode=mode)
        assert np.array_equal(8 * a, b)


def test_emulated_k_and_sm_scale_trade_exactly():
    q, k, v = rnd((1, 1, 256, 32), 43), rnd((1, 1, 256, 32), 44), rnd((1, 1, 256, 32), 45)
    for mode in ["int8_fp8", "fp4"]:
        a = att.emulated_sage_attention(q, k, v, True, 0.25, mode=mode)
        b = att.emulated_sage_attention(q, k * np.float32(4), v, True, 0.0625, mode=mode)
        assert np.array_equal(a, b)


@pytest.mark.parametrize("mode,tol", [("int8_fp8", 0.999), ("fp4", 0.97)])
def test_emulated_close_to_exact(mode, tol):
    q, k = rnd((1, 2, 512, 64), 50), rnd((1, 2, 512, 64), 51) + np.float32(2.0)
    v = rnd((1, 2, 512, 64), 52)
    a = att.emulated_sage_attention(q, k, v, False, 0.125, mode=mode)
    b = att.exact_attention(q, k, v, False, 0.125)
    cos = np.sum(a * b) / np.sqrt(np.sum(a * a) * np.sum(b * b))
    assert cos >= tol


def test_output_rounding_matches_dtype():
    o = np.random.default_rng(7).standard_normal((4, 4))
    r = enc.round_to_dtype(o, "bf16")
    assert np.array_equal(r, enc.bf16_round(r))
    assert np.max(np.abs(r - o)) <= np.abs(o).max() * 2.0 ** -8


@pytest.mark.parametrize("N", [384, 300])
@pytest.mark.parametrize("mode", ["int8_fp8", "fp4", "fp8"])
@pytest.mark.parametrize("causal", [False, True])
def test_row_subset_matches_full(mode, causal, N):
    # computing a subset of query rows gives exactly those rows of the full run
    q, k, v = rnd((1, 2, N, 32), 60), rnd((1, 2, N, 32), 61), rnd((1, 2, N, 32), 62)
    rows = np.array([0, 5, 127, 128, 200, N - 1])
    full = att.emulated_sage_attention(q, k, v, causal, 0.2, mode=mode)
    sub = att.emulated_sage_attention(q, k, v, causal, 0.2, mode=mode, rows=rows)
    assert np.array_equal(full[:, :, rows], sub)
    fe = att.exact_attention(q, k, v, causal, 0.2)
    se = att.exact_attention(q, k, v, causal, 0.2, rows=rows)
    assert np.max(np.abs(fe[:, :, rows] - se)) <= 1e-15


def test_fp8_p_ambiguity_marks_midpoints():
    # 448 P~ exactly at / near the midpoint of two e4m3 values is ambiguous;
    # far from any midpoint it is not
    mids = np.array([432.0, 17.0, 1.0625, 2.0 ** -9 * 1.5]) / 448.0     # 416|448, 16|18, 1|1.125
    amb = att.fp8_p_ambiguity(mids, 1e-6)
    assert np.array_equal(amb, np.array([32.0, 2.0, 0.125, 2.0 ** -9]))
    far = np.array([440.0, 16.1, 1.01]) / 448.0
    assert np.all(att.fp8_p_ambiguity(far, 1e-6) == 0)


def test_ambiguity_bound_covers_flipped_codes():
    # Perturbing P~ by a relative 1e-4 before quantization (a stand-in for a
    # kernel's FP32 evaluation) moves O by no more than the bound for 1e-4,
    # and does move it (some codes flip).
    q, k, v = rnd((1, 1, 256, 32), 70, 2.0), rnd((1, 1, 256, 32), 71, 2.0), rnd((1, 1, 256, 32), 72)
    o, bnd = att.emulated_sage_attention(q, k, v, True, 0.3, ambiguity_eps=1e-4)
    base = att.quant_p_fp8
    moved = 0
    try:
        for sgn in (+1, -1):
            att.quant_p_fp8 = lambda pt, s=sgn: base(pt * (1 + s * 1e-4))
            # the tile loop receives the perturbed quantizer through the module
            o2 = att.emulated_sage_attention(q, k, v, True, 0.3)
            assert np.all(np.abs(o2 - o) <= bnd + 1e-12)
            moved += int(np.any(o2 != o))
    finally:
        att.quant_p_fp8 = base
    assert moved == 2
    assert np.array_equal(att.emulated_sage_attention(q, k, v, True, 0.3), o)


def test_fp4_p_ambiguity_marks_midpoints():
    # one row of two 16-key groups:
    #   group 0: amax = 1 (s16 = 448, a grid value, unambiguous); 6 P~ = 2.5 is
    #            an e2m1 midpoint (2|3), so that value may move by 1 * s16;
    #            6 P~ = 0.6 and 6 P~ = 4.2 are far from any midpoint
    #   group 1: 448 amax = 17 lies between e4m3 16 and 18: the scale itself is
    #            ambiguous, and the bound covers the group re-quantized
    row = np.zeros((1, 32))
    row[0, 0], row[0, 1], row[0, 2], row[0, 3] = 1.0, 2.5 / 6, 0.1, 0.7
    row[0, 16], row[0, 17] = 17.0 / 448, 5.0 / 448
    b = att.fp4_p_ambiguity(row, 1e-6)
    assert b[0, 1] == 448.0
    assert np.all(b[0, [0, 2, 3]] == 0) and np.all(b[0, 4:16] == 0)
    # group 1 with s16 = 16 or 18 (g = 1/2688): the element at 17/448 codes to
    # 6 * 17/16 -> 6 (sat) * 16 = 96 or 6 * 17/18 -> 6 * 18 = 108
    base = att.quant_p_fp4(row)
    assert base[0, 16] in (96.0, 108.0)
    assert b[0, 16] >= 12.0
    assert np.all(b[0, 18:] == 0)


def test_fp4_ambiguity_bound_covers_flipped_codes():
    # FP4 mode: a relative 1e-4 perturbation of P~ before quantization moves O
    # by no more than the bound, and does move it.
    q, k, v = rnd((1, 1, 256, 32), 80, 2.0), rnd((1, 1, 256, 32), 81, 2.0), rnd((1, 1, 256, 32), 82)
    o, bnd = att.emulated_sage_attention(q, k, v, True, 0.3, mode="fp4", ambiguity_eps=1e-4)
    base = att.quant_p_fp4
    moved = 0
    try:
        for sgn in (+1, -1):
            att.quant_p_fp4 = lambda pt, s=sgn: base(pt * (1 + s * 1e-4))
            o2 = att.emulated_sage_attention(q, k, v, True, 0.3, mode="fp4")
            assert np.all(np.abs(o2 - o) <= bnd + 1e-12)
            moved += int(np.any(o2 != o))
    finally:
        att.quant_p_fp4 = base
    assert moved == 2
    assert np.array_equal(att.emulated_sage_attention(q, k, v, True, 0.3, mode="fp4"), o)


# ------------------------------------------------------------ FP8 Q/K ----

def test_fp8_blocks_properties():
    x = rnd((1, 2, 300, 64), 90, 3.0)
    x[0, 1, 128:256] = 0.0                               # an all-zero block
    codes, scales = pp.quant_fp8_blocks(x)
    assert codes.dtype == np.uint8 and scales.shape == (1, 2, 3)
    assert scales[0, 1, 1] == 0 and np.all(codes[0, 1, 128:256] == 0)
    for h in range(2):
        for i, (s, e) in enumerate([(0, 128), (128, 256), (256, 300)]):
            blk = x[0, h, s:e].astype(np.float64)
            sc = float(scales[0, h, i])
            if sc == 0:
                continue
            assert scales[0, h, i] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448))
            dec = enc.e4m3_decode(codes[0, h, s:e]) * sc
            # the block maximum lands on the top of the grid
            assert np.abs(enc.e4m3_decode(codes[0, h, s:e])).max() == 448.0
            # e4m3 relative error 2^-4 in the normal range, half the
            # subnormal step (2^-10 s) below it
            err = np.abs(dec - blk)
            assert np.all(err <= np.maximum(np.abs(blk) * 2.0 ** -4, sc * 2.0 ** -10) * (1 + 1e-6))
            # codes: the independent brute-force nearest-grid encoder on the
            # FP32 quotients
            t = (x[0, h, s:e] / np.float32(sc)).astype(np.float32)
            assert np.array_equal(codes[0, h, s:e], enc.e4m3_encode_bruteforce(t))


def test_quant_qk_fp8_smooths_k_only():
    q, k = rnd((1, 1, 256, 32), 91), rnd((1, 1, 256, 32), 92) + np.float32(10)
    r = pp.quant_qk_fp8(q, k)
    c2, s2 = pp.quant_fp8_blocks(q, 1)
    assert np.array_equal(r["q_codes"], c2) and np.array_equal(r["q_scales"], s2)
    kc, ks = pp.quant_fp8_blocks(k.astype(np.float32) - r["k_mean"][:, :, None, :], 32)
    assert np.array_equal(r["k_codes"], kc) and np.array_equal(r["k_scales"], ks)
    assert r["q_scales"].shape == (1, 1, 256) and r["k_scales"].shape == (1, 1, 8)


@pytest.mark.parametrize("N", [256, 139])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_constant_k_gives_visible_mean(causal, N):
    # K rows all equal -> smoothed K = 0 -> s_K = 0, codes 0 -> P~ = 1 -> O is
    # the visible mean of V (V on the e4m3 grid with s_V = 1: exact)
    d = 32
    rng = np.random.default_rng(93)
    q = rnd((1, 1, N, d), 94)
    k = np.broadcast_to(rnd((1, 1, 1, d), 95), (1, 1, N, d)).copy()
    grid = enc.e4m3_decode(np.arange(0x7F))
    v = (rng.choice(grid, (1, 1, N, d)) * rng.choice([-1, 1], (1, 1, N, d))).astype(np.float32)
    v[0, 0, 0, :] = 448.0
    o = att.emulated_sage_attention(q, k, v, causal, 0.2, mode="fp8")
    v64 = v[0, 0].astype(np.float64)
    want = (np.cumsum(v64, axis=0) / np.arange(1, N + 1)[:, None]) if causal \
        else np.broadcast_to(v64.mean(axis=0), (N, d))
    assert np.max(np.abs(o[0, 0] - want)) <= 1e-12 * max(1.0, np.abs(want).max())


def test_fp8_two_key_closed_form():
    # Q and K on the e4m3 grid with block maxima 448 (scales exactly 1): the
    # emulated scores are the exact q . k; the top two keys have P~ = 1 and
    # 1/1.1, the latter encoding as 448/1.1 -> 416 (as in INT8 mode).
    N, d = 128, 16
    q = np.zeros((1, 1, N, d), np.float32)
    q[..., 0] = 448.0
    k = np.zeros((1, 1, N, d), np.float32)
    kc = np.full(N, -7.0)
    kc[0], kc[1], kc[2] = 448.0, 416.0, 0.0
    kc[3] = -(kc[:3].sum() + kc[4:].sum())               # = 4: channel sum 0 -> mean 0
    assert enc.e4m3_decode(enc.e4m3_encode(np.float32(kc[3]))) == kc[3]
    k[0, 0, :, 0] = kc
    sm_scale = math.log(1.1) / (448.0 * 32.0)            # S0 - S1 = ln 1.1
    rng = np.random.default_rng(96)
    grid = enc.e4m3_decode(np.arange(0x7F))
    v = (rng.choice(grid, (1, 1, N, d)) * rng.choice([-1, 1], (1, 1, N, d))).astype(np.float32)
    v[0, 0, 5, :] = 448.0
    o = att.emulated_sage_attention(q, k, v, False, sm_scale, mode="fp8")
    S = 448.0 * kc * sm_scale
    p = np.exp(S - S.max())
    codes = enc.e4m3_decode(enc.e4m3_encode(448.0 * p)) / 448.0
    assert codes[1] == 416.0 / 448.0
    want = (codes[:, None] * v[0, 0].astype(np.float64)).sum(axis=0) / p.sum()
    assert np.max(np.abs(o[0, 0] - want[None, :])) <= 1e-12


def test_fp8_scaling_laws_and_subsets():
    q, k, v = rnd((1, 1, 256, 32), 97), rnd((1, 1, 256, 32), 98), rnd((1, 1, 256, 32), 99)
    a = att.emulated_sage_attention(q, k, v, True, 0.25, mode="fp8")
    assert np.array_equal(att.emulated_sage_attention(q, k * np.float32(4), v, True, 0.0625,
                                                      mode="fp8"), a)
    assert np.array_equal(att.emulated_sage_attention(q, k, v * np.float32(8), True, 0.25,
                                                      mode="fp8"), 8 * a)
    rows = np.array([0, 77, 128, 255])
    assert np.array_equal(att.emulated_sage_attention(q, k, v, True, 0.25, mode="fp8",
                                                      rows=rows), a[:, :, rows])


def test_fp8_close_to_exact():
    q, k = rnd((1, 2, 512, 64), 100), rnd((1, 2, 512, 64), 101) + np.float32(2.0)
    v = rnd((1, 2, 512, 64), 102)
    a = att.emulated_sage_attention(q, k, v, False, 0.125, mode="fp8")
    b = att.exact_attention(q, k, v, False, 0.125)
    assert np.sum(a * b) / np.sqrt(np.sum(a * a) * np.sum(b * b)) >= 0.998


def _fp32_dot_orders(a, b):
    """Sums of the (exact FP32) products a_c b_c in FP32 in several orders."""
    t = (a.astype(np.float32) * b.astype(np.float32)).astype(np.float32)
    outs = []
    for order in (t, t[::-1], np.random.default_rng(0).permutation(t)):
        acc = np.float32(0)
        for x in order:
            acc = np.float32(acc + x)
        outs.append(float(acc))
    w = t.copy()                                   # pairwise (tree) order
    while len(w) > 1:
        w = (w[0::2] + w[1::2]).astype(np.float32)
    outs.append(float(w[0]))
    return outs


def test_fp8_accumulation_bound_covers_fp32_sums():
    # the bound the FP8 mode grants the kernel's Q K^T holds for FP32
    # accumulation in any of several orders, including adversarial terms
    rng = np.random.default_rng(103)
    grid = enc.e4m3_decode(np.arange(0x7F))
    cases = [(rng.choice(grid, 128) * rng.choice([-1, 1], 128),
              rng.choice(grid, 128) * rng.choice([-1, 1], 128)) for _ in range(200)]
    big = np.full(128, 2.0 ** -9)
    big[0] = 448.0
    cases.append((big, big.copy()))                # one huge product, 127 tiny ones
    alt = np.where(np.arange(128) % 2 == 0, 448.0, -448.0) * 1.0
    alt[-1] = 2.0 ** -9
    cases.append((alt, np.abs(alt)))               # cancellation down to a tiny remainder
    for a, b in cases:
        exact = float(np.dot(a, b))                # exact in FP64 (e4m3 products)
        bound = att.FP8_QK_ACC_REL * float(np.dot(np.abs(a), np.abs(b)))
        for s in _fp32_dot_orders(a, b):
            assert abs(s - exact) <= bound


def test_fp8_ambiguity_bound_covers_fp32_accumulation():
    # The kernel's Q K^T in FP32 (here: sequential FP32 sums, forward or
    # backward over the channels) moves O by no more than the bound the FP8
    # mode returns, and does move it.
    q, k, v = rnd((1, 1, 256, 64), 104, 2.0), rnd((1, 1, 256, 64), 105, 2.0), rnd((1, 1, 256, 64), 106)
    o, bnd = att.emulated_sage_attention(q, k, v, True, 0.3, mode="fp8", ambiguity_eps=2.0 ** -15)
    base = att.qk_product

    def fp32_seq(qd, kd, rev):
        qf, kf = qd.astype(np.float32), kd.astype(np.float32)
        acc = np.zeros((len(qd), len(kd)), np.float32)
        chans = range(qd.shape[1] - 1, -1, -1) if rev else range(qd.shape[1])
        for c in chans:
            acc = (acc + (qf[:, c, None] * kf[None, :, c]).astype(np.float32)).astype(np.float32)
        return acc.astype(np.float64)

    moved = 0
    try:
        for rev in (False, True):
            att.qk_product = lambda qd, kd, r=rev: fp32_seq(qd, kd, r)
            o2 = att.emulated_sage_attention(q, k, v, True, 0.3, mode="fp8")
            assert np.all(np.abs(o2 - o) <= bnd + 1e-12)
            moved += int(np.any(o2 != o))
    finally:
        att.qk_product = base
    assert moved >= 1
    assert np.array_equal(att.emulated_sage_attention(q, k, v, True, 0.3, mode="fp8"), o)


# ----------------------------------------------------------- ragged N ----

def test_fp4_v_ragged_counts_missing_tokens_as_zeros():
    # N = 200: the last 16-token group (tokens 192..199) is partial; its scale
    # and codes equal those of V padded with zero tokens to 208
    v = rnd((1, 2, 200, 32), 110, 2.0)
    c, f, g = pp.quant_v_fp4(v)
    assert c.shape == (1, 2, 32, 200) and f.shape == (1, 2, 32, 13) and g.shape == (1, 2, 2)
    vp = np.concatenate([v, np.zeros((1, 2, 8, 32), np.float32)], axis=2)
    cp, fp_, gp = pp.quant_v_fp4(vp)
    assert np.array_equal(c, cp[..., :200]) and np.array_equal(f, fp_) and np.array_equal(g, gp)
    assert np.all(cp[..., 200:] == 0)


def test_fp4_p_partial_group():
    # a 40-key row: groups 0..15, 16..31 and the partial 32..39
    pt = np.random.default_rng(111).random((3, 40))
    full = att.quant_p_fp4(np.concatenate([pt, np.zeros((3, 8))], axis=1))
    assert np.array_equal(att.quant_p_fp4(pt), full[:, :40])
    assert att.fp4_p_ambiguity(pt, 1e-6).shape == (3, 40)


@pytest.mark.parametrize("mode", ["int8_fp8", "fp8", "fp4"])
def test_ragged_identity_and_close_to_exact(mode):
    # a ragged length through every mode stays as close to exact attention as
    # the same data at a full-tile length does
    d = 64 if mode != "fp4" else 32
    q, k, v = rnd((1, 1, 300, d), 112), rnd((1, 1, 300, d), 113) + np.float32(1.0), \
        rnd((1, 1, 300, d), 114)
    for causal in (False, True):
        a = att.emulated_sage_attention(q, k, v, causal, 0.125, mode=mode)
        b = att.exact_attention(q, k, v, causal, 0.125)
        cos = np.sum(a * b) / np.sqrt(np.sum(a * a) * np.sum(b * b))
        assert cos >= (0.97 if mode == "fp4" else 0.995)


# ------------------------------------------------------ FP4 P~ encoder ----
# Pins of quant_p_fp4 itself (SageAttention3 abstract: FP4 values with one FP8
# scale per 16 elements; the P~ reading is s16 = ue4m3(448 amax16) with the
# static tile scale 1/2688).  The restatement below writes both grids out
# and takes the nearest value (ties to the even code, saturating), sharing
# nothing with oracle/encoders.py.

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
# UE4M3 codes 0..0x7E: eight subnormals k 2^-9, then (1 + m/8) 2^(e-7)
UE4M3_GRID = np.array([k * 2.0 ** -9 for k in range(8)] +
                      [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)][:-1])


def nearest_even(grid, x):
    x = np.minimum(np.asarray(x, np.float64), grid[-1])
    dist = np.abs(x[..., None] - grid)
    cand = dist == dist.min(axis=-1, keepdims=True)
    even = cand & (np.arange(len(grid)) % 2 == 0)
    pick = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1))
    return grid[pick]


def brute_quant_p_fp4(pt):
    R, C = pt.shape
    out = np.zeros((R, C))
    for r in range(R):
        for g0 in range(0, C, 16):
            blk = pt[r, g0:g0 + 16]
            s16 = nearest_even(UE4M3_GRID, blk.max() * 448.0)
            den = s16 / 2688.0
            if den > 0:
                out[r, g0:g0 + 16] = nearest_even(E2M1_GRID, blk / den) * s16
    return out


def test_fp4_p_encoder_matches_grid_restatement():
    g = np.random.default_rng(90)
    pt = np.exp(-np.abs(g.standard_normal((6, 128))) * 3.0)
    pt[0, 5] = 1.0                                   # a row max
    pt[1, 16:32] = 0.0                               # an all-zero group
    pt[2, 32:48] *= 2.0 ** -20                       # a group with a subnormal scale
    # values planted at e2m1 midpoints of their group (both ends must round
    # to the even code)
    den = nearest_even(UE4M3_GRID, pt[3, 64:80].max() * 448.0) / 2688.0
    for j, mid in enumerate([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]):
        if mid * den < pt[3, 64:80].max():
            pt[3, 65 + j] = mid * den
    assert np.array_equal(att.quant_p_fp4(pt), brute_quant_p_fp4(pt))


def test_fp4_p_encoder_closed_forms():
    # the row max P~ = 1: s16 = ue4m3(448) = 448, t = 6 P~ -> code 6, and the
    # value 6 * 448 times the tile scale 1/2688 is exactly 1
    pt = np.full((1, 32), 0.3)
    pt[0, 7] = 1.0
    v = att.quant_p_fp4(pt)
    assert v[0, 7] * att.P_FP4_G == 1.0
    # an all-zero group stays zero; other groups do not see it
    pt2 = pt.copy()
    pt2[0, 16:] = 0.0
    v2 = att.quant_p_fp4(pt2)
    assert np.all(v2[0, 16:] == 0.0)
    assert np.array_equal(v2[0, :16], v[0, :16])


def test_fp4_p_encoder_power_of_two_scaling():
    # both grids are the same in every normal binade: scaling a group by 2^-k
    # (scale still normal: 448 amax 2^-k >= 2^-6) scales its values by 2^-k
    g = np.random.default_rng(91)
    pt = np.exp(-np.abs(g.standard_normal((4, 64))) * 2.0)
    pt[:, 0] = 1.0
    base = att.quant_p_fp4(pt)
    for k in range(1, 9):
        assert np.array_equal(att.quant_p_fp4(pt * 2.0 ** -k), base * 2.0 ** -k)


def test_fp8_p_encoder_matches_grid_restatement():
    # quant_p_fp8 is the e4m3 value of 448 P~ (the non-negative e4m3 grid is
    # the UE4M3 grid above): the row max P~ = 1 is 448, and every value is the
    # nearest grid point, ties to the even code (planted midpoints included)
    g = np.random.default_rng(92)
    pt = np.exp(-np.abs(g.standard_normal((4, 128))) * 4.0)
    pt[0, 0] = 1.0
    mids = 0.5 * (UE4M3_GRID[1:] + UE4M3_GRID[:-1])
    mids = mids[(mids / 448.0) * 448.0 == mids] / 448.0   # 448 P~ lands on the midpoint
    assert len(mids) > 60
    pt[1, :len(mids[::2])] = mids[::2]
    pt[2, :len(mids[1::2])] = mids[1::2]
    got = att.quant_p_fp8(pt)
    assert got[0, 0] == 448.0
    assert np.array_equal(got, nearest_even(UE4M3_GRID, pt * 448.0))


# ------------------------------------------------ FP4 Q/K/V pre-pass encoders ----
# The FP32 formula of the FP4 encodings restated step by step on the grids
# above (SageAttention3 abstract; the reading of the scale chain:
# g = fp32(amax_tile / 2688), s16 = ue4m3(fp32(amax16 / fp32(6 g))),
# code = e2m1(fp32(x / fp32(s16 g)))); values compared, not code bits.

def brute_fp4_tile(blk):
    """blk float32 [L, W], 16-groups along W: (values [L, W], scales [L, W/16], g)."""
    f32 = np.float32
    g = f32(f32(np.abs(blk).max()) / f32(2688))
    six_g = f32(f32(6) * g)
    L, W = blk.shape
    vals = np.zeros((L, W))
    scales = np.zeros((L, W // 16))
    for l in range(L):
        for m in range(W // 16):
            grp = blk[l, 16 * m:16 * m + 16]
            r = f32(f32(np.abs(grp).max()) / six_g) if six_g != 0 else f32(0)
            s = nearest_even(UE4M3_GRID, float(r))
            scales[l, m] = s
            den = f32(f32(s) * g)
            if den != 0:
                t = (grp / den).astype(np.float32).astype(np.float64)
                vals[l, 16 * m:16 * m + 16] = np.sign(t) * nearest_even(E2M1_GRID, np.abs(t))
    return vals, scales, g


def e2m1_value(codes):
    c = codes.astype(np.int64)
    return np.where(c & 8, -1.0, 1.0) * E2M1_GRID[c & 7]


def test_fp4_token_encoder_matches_grid_restatement():
    x = rnd((1, 1, 256, 64), 23, 2.0)
    x[0, 0, 5, 16:32] = 0.0                          # an all-zero group
    x[0, 0, 9, 0:16] *= np.float32(2.0 ** -12)       # a group far below the tile max
    # exact e2m1 ties, x / fp32(s16 g) on a midpoint, planted under the
    # group max of a few groups of the first tile (each takes the even code;
    # a scale chain rounded differently breaks them the other way)
    f32 = np.float32
    tile_g = f32(f32(np.abs(x[0, 0, :128]).max()) / f32(2688))
    planted = 0
    for r in (20, 33, 77):
        for m in range(4):
            grp = x[0, 0, r, 16 * m:16 * m + 16]
            s = nearest_even(UE4M3_GRID, float(f32(f32(np.abs(grp).max()) / f32(f32(6) * tile_g))))
            den = f32(f32(s) * tile_g)
            for j, mid in enumerate([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]):
                xv = f32(f32(mid) * den)
                if abs(xv) < np.abs(grp).max() and f32(xv / den) == f32(mid):
                    x[0, 0, r, 16 * m + 1 + j] = -xv if j % 2 else xv
                    planted += 1
    assert planted > 40
    codes, sf, g = pp.quant_fp4_tokens(x)
    for t in range(2):
        blk = x[0, 0, 128 * t:128 * (t + 1)].astype(np.float32)
        vals, scales, gt = brute_fp4_tile(blk)
        assert g[0, 0, t] == gt
        assert np.array_equal(UE4M3_GRID[sf[0, 0, 128 * t:128 * (t + 1)]], scales)
        assert np.array_equal(e2m1_value(codes[0, 0, 128 * t:128 * (t + 1)]), vals)


def test_fp4_v_encoder_matches_grid_restatement():
    # V: 16-groups over tokens, written transposed; tile = 128 tokens x d
    v = rnd((1, 1, 256, 32), 24)
    v[0, 0, 40:56, 7] = 0.0                          # an all-zero token group of one channel
    codes, sf, g = pp.quant_v_fp4(v)
    vt = v[0, 0].T.astype(np.float32)                # [d, N]
    for t in range(2):
        blk = vt[:, 128 * t:128 * (t + 1)]
        vals, scales, gt = brute_fp4_tile(blk)
        assert g[0, 0, t] == gt
        assert np.array_equal(UE4M3_GRID[sf[0, 0, :, 8 * t:8 * (t + 1)]], scales)
        assert np.array_equal(e2m1_value(codes[0, 0, :, 128 * t:128 * (t + 1)]), vals)
