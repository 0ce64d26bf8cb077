"""Pins of the oracle's Q smoothing (CPU only).

Q smoothing (SageAttention2 abstract, "we propose a method to smooth Q";
the oracle's pre-pass reading 2) takes each 128-token query block's mean
out of Q before quantization and adds it back as a score bias
dS = qbar . k'.  The pins: the block mean against closed forms (a wrong axis
or a wrong block fails them); dS against exact rational arithmetic on the
smoothed keys (dS taken from the unsmoothed keys, a wrong index or a dropped
channel fails it); with identity quantizers the smoothed path must give
exact attention (a dropped or mis-signed bias, or one applied to the wrong
query block, fails it); a block whose mean is zero must change nothing.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import attention as att
from oracle import encoders as enc
from oracle import prepass as pp


def rnd(shape, seed, scale=1.0):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * np.float32(scale)
    return enc.bf16_round(x)


def biased_qk(B, H, N, d, seed):
    """Q and K with per-channel biases (what Q smoothing removes) as bf16."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N, d)) + 3.0 * rng.standard_normal((B, H, 1, d))
    k = rng.standard_normal((B, H, N, d)) + 2.0 * rng.standard_normal((B, H, 1, d))
    v = rng.standard_normal((B, H, N, d))
    return (enc.bf16_round(q.astype(np.float32)), enc.bf16_round(k.astype(np.float32)),
            enc.bf16_round(v.astype(np.float32)))


def test_block_mean_closed_form():
    # token t of channel c holds t + 1000 c (exact in FP32): the mean of a
    # block of tokens s .. e-1 is (s + e - 1) / 2 + 1000 c; the ragged last
    # block (N = 300: tokens 256 .. 299) averages its 44 tokens only
    N, d = 300, 8
    t = np.arange(N, dtype=np.float32)[:, None]
    c = np.arange(d, dtype=np.float32)[None, :]
    q = np.broadcast_to(t + 1000 * c, (1, 1, N, d)).astype(np.float32)
    m = pp.q_block_mean(q)
    assert m.shape == (1, 1, 3, d)
    for i, (s, e) in enumerate([(0, 128), (128, 256), (256, 300)]):
        np.testing.assert_array_equal(m[0, 0, i], (s + e - 1) / 2.0 + 1000 * np.arange(d))


def test_block_mean_of_cancelling_pairs_is_zero_and_smoothing_changes_nothing():
    # tokens 2i and 2i+1 are x and -x: every block mean is exactly 0, so the
    # smoothed Q is Q, the bias is 0, and the whole emulated pass is unchanged
    B, H, N, d = 1, 2, 256, 64
    half = rnd((B, H, N // 2, d), 1)
    q = np.empty((B, H, N, d), np.float32)
    q[:, :, 0::2], q[:, :, 1::2] = half, -half
    k, v = rnd((B, H, N, d), 2), rnd((B, H, N, d), 3)
    qm = pp.q_block_mean(q)
    assert not qm.any()
    for mode in ("int8_fp8", "fp8", "fp4"):
        fn = {"int8_fp8": pp.quant_qk_int8, "fp8": pp.quant_qk_fp8, "fp4": pp.quant_qk_fp4}[mode]
        a, b = fn(q, k), fn(q, k, smooth=True)
        assert not b["dS"].any()
        for key in a:
            np.testing.assert_array_equal(a[key], b[key])
        o0 = att.emulated_sage_attention(q, k, v, mode=mode)
        o1 = att.emulated_sage_attention(q, k, v, mode=mode, smooth_q=True)
        np.testing.assert_array_equal(o0, o1)


def test_smoothing_bias_against_exact_rationals():
    # dS[blk, j] = qbar[blk] . (fp32(K_j) - mean_K), checked with Fractions
    # on every entry; K has a per-channel mean, so the unsmoothed K gives
    # different values
    B, H, N, d = 1, 1, 160, 16
    q, k, _ = biased_qk(B, H, N, d, 7)
    qm = pp.q_block_mean(q)
    mean = pp.k_channel_mean(k)
    ks = pp.smooth_k(k, mean)
    ds = pp.smoothing_bias(qm, ks)
    assert ds.shape == (B, H, 2, N) and ds.dtype == np.float32
    for blk in range(2):
        for j in range(N):
            exact = sum(Fraction(float(qm[0, 0, blk, c])) * Fraction(float(ks[0, 0, j, c]))
                        for c in range(d))
            # the FP64 channel-order sum of exact products, rounded to FP32,
            # is within one FP32 rounding of the exact value
            assert abs(float(ds[0, 0, blk, j]) - float(exact)) <= \
                2.0 ** -23 * abs(float(exact)) + 2.0 ** -40
    raw = pp.smoothing_bias(qm, np.asarray(k, np.float32))
    assert np.abs(raw - ds).max() > 1e-2


@pytest.mark.parametrize("causal", [False, True])
def test_identity_quantizers_with_smoothing_give_exact_attention(causal):
    # Q' + qbar = Q and K' = K - mean (a per-row constant under softmax): with
    # every quantizer the identity the smoothed pass is exact attention up to
    # the FP32 roundings of Q', K' and dS.  N = 300 spans three query blocks,
    # the last one ragged.
    B, H, N, d = 1, 2, 300, 64
    q, k, v = biased_qk(B, H, N, d, 11)
    ex = att.exact_attention(q, k, v, causal=causal)
    o = att.emulated_sage_attention(q, k, v, causal=causal, quantizers="identity", smooth_q=True)
    assert np.abs(o - ex).max() < 5e-6
    # the bias of the wrong query block, or none, is far off
    qm = pp.q_block_mean(q)
    ks = pp.smooth_k(k, pp.k_channel_mean(k))
    qi = pp.smooth_q(q, qm)
    ds = pp.smoothing_bias(qm, ks)
    ones = np.ones(N)
    for bias in (None, ds[0, 0, ::-1].copy(), -ds[0, 0]):
        o_bad = att._tile_loop(qi[0, 0].astype(np.float64), ks[0, 0].astype(np.float64),
                               v[0, 0].astype(np.float64), ones, ones, np.ones((3, d)),
                               lambda x: x, causal, 1.0 / np.sqrt(d), s_bias=bias)
        assert np.abs(o_bad - ex[0, 0]).max() > 1e-2


def test_constant_query_block_quantizes_to_zero_and_keeps_its_scores_in_the_bias():
    # a block whose tokens are all q0: Q' = 0, so codes and scales are 0 and
    # every score of the block comes from dS = q0 . k'
    B, H, N, d = 1, 1, 128, 32
    rng = np.random.default_rng(5)
    q0 = enc.bf16_round(rng.standard_normal(d).astype(np.float32))
    q = np.broadcast_to(q0, (B, H, N, d)).astype(np.float32)
    k = rnd((B, H, N, d), 6)
    r = pp.quant_qk_int8(q, k, smooth=True)
    assert not r["q_codes"].any() and not r["q_scales"].any()
    ks = pp.smooth_k(k, r["k_mean"])
    np.testing.assert_allclose(r["dS"][0, 0, 0], ks[0, 0].astype(np.float64) @ q0.astype(np.float64),
                               rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("mode,floor", [("int8_fp8", 0.0), ("fp8", 1e-3), ("fp4", 1e-2)])
def test_smoothing_helps_when_queries_carry_a_channel_bias(mode, floor):
    # the purpose of the method: on queries with a per-channel bias, the
    # smoothed pass is closer to exact attention (by at least `floor` in
    # cosine for the coarser formats)
    B, H, N, d = 1, 2, 384, 64
    q, k, v = biased_qk(B, H, N, d, 21)
    ex = att.exact_attention(q, k, v).ravel()

    def cos(o):
        o = o.ravel()
        return float(o @ ex / np.sqrt((o @ o) * (ex @ ex)))

    c0 = cos(att.emulated_sage_attention(q, k, v, mode=mode))
    c1 = cos(att.emulated_sage_attention(q, k, v, mode=mode, smooth_q=True))
    assert c1 > c0 + floor
