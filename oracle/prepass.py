"""Quantization pre-pass of the oracle (TEST INFRASTRUCTURE ONLY).

Inputs are NumPy arrays of shape [B, H, N, d] holding bf16/fp16 values (as
float32 or float64; every bf16/fp16 value is exact in both).  Token blocks
are 128 tokens; the last block of a head may be shorter (ragged N).

Readings of the pages (they give the method only at abstract level):

1. K smoothing (SageAttention abstract, "accurate 8-bit attention"; the
   kernel-comparison blog's "precision-aware scaling"): K loses its
   per-channel mean over all N tokens of its (b, h) before quantization.
   Every score of a query row then moves by the same constant q . mean, so
   softmax -- and O -- is unchanged.  The mean is accumulated in FP64 in a
   fixed order: per 128-token chunk a partial sum in token order, then the
   chunk partials in chunk order; mean = fp32(total / N).
2. Q smoothing (SageAttention2 abstract: "we propose a method to smooth
   Q"), optional (smooth_q): per (b, h) and per 128-token block of queries
   (the query tile), qbar = fp32(mean of the block's tokens), accumulated in
   FP64 in token order; Q' = fp32(Q) - qbar (one FP32 subtraction) is what
   gets quantized.  What qbar removes comes back as a bias on every score of
   the block: dS[blk, j] = qbar[blk] . k'_j with k'_j = fp32(K_j) - mean_K
   the smoothed key (reading 1) before quantization, evaluated in FP64 with
   the d products added in channel order (each product of two FP32 values
   is exact in FP64, so one rounding per addition) and rounded once to
   FP32.  Without it Q is quantized as it is.
3. INT8 Q/K: one FP32 scale per block of tokens of one (b, h), covering all
   d channels: s = fp32(amax / 127); code = clamp(rne(fp32(x / s)), +-127);
   an all-zero block gets s = 0 and codes 0.  For K, x = fp32(K) - mean is a
   single FP32 subtraction.  Block sizes (the SageAttention2 abstract's
   "hardware-friendly thread-level granularity", read for a kernel in which
   one thread owns one query row and dequantizes 32 keys at a time): Q one
   token (Q_GROUP), K 32 tokens (K_GROUP).
4. FP8 V (SageAttention2 abstract): per channel over all N tokens of a
   (b, h): s_V = fp32(amax / 448); code = e4m3(fp32(V / s_V)).  Written
   transposed, [B, H, d, N], so that the P~V contraction (over tokens) reads
   it token-contiguous.
5. FP4 (SageAttention3 abstract; one FP8 scale per 16 elements):
   NVFP4-style two-level scaling.  Q and smoothed K: per 128-token tile
   g = fp32(amax_tile / 2688) (2688 = 448 * 6); per 16 contiguous channels
   s16 = ue4m3(fp32(amax16 / fp32(6 * g))); code = e2m1(fp32(x / fp32(s16 *
   g))); a zero g or s16 gives code 0.  V: the same, with the 16-element
   blocks running over tokens (per channel) inside each 128-token tile.
6. FP8 Q/K (the kernel-comparison blog, "How SageAttention uses
   quantization for more throughput": queries and keys go to INT8 or FP8):
   the INT8 scheme of reading 3 with the e4m3 grid in place of the
   integers, with the same blocks (Q per token, K per 32 tokens):
   s = fp32(amax / 448); code = e4m3(fp32(x / s)) (round to nearest even,
   saturating); an all-zero block gets s = 0 and codes 0.  K is smoothed
   first, as in reading 1.
7. Ragged sequences (N not a multiple of 128): the last block (of 32 K
   tokens, or 128 tokens in FP4 mode) may be shorter and its scale covers
   its tokens only; the K mean and the V
   scales divide by / range over the N real tokens; in FP4 mode a partial
   16-element group (V over tokens, P~ over keys) counts its missing
   elements as zeros, which change neither its maximum nor any code.
"""

import numpy as np

from .encoders import (e4m3_encode, e2m1_encode, ue4m3_encode, ue4m3_decode,
                       int8_quantize)

BLOCK = 128      # tokens per tile (FP4 tile scales, K-mean chunks, V tiles)
Q_GROUP = 1      # tokens per Q scale in the 8-bit modes (one query row)
K_GROUP = 32     # tokens per K scale in the 8-bit modes (32 keys)
FP4_VEC = 16     # elements per FP4 micro-block
FP4_G_DIV = np.float32(2688.0)   # 448 * 6
FP8_DIV = np.float32(448.0)
INT8_DIV = np.float32(127.0)


def _blocks(n, size=BLOCK):
    return [(s, min(s + size, n)) for s in range(0, n, size)]


def k_channel_mean(k):
    """Per-(b, h, channel) mean of K over all tokens, reading 1 above.

    Returns float32 [B, H, d].
    """
    k = np.asarray(k, dtype=np.float64)
    B, H, N, d = k.shape
    if N == 0:
        return np.zeros((B, H, d), np.float32)
    total = np.zeros((B, H, d), np.float64)
    for s, e in _blocks(N):
        part = np.zeros((B, H, d), np.float64)
        for t in range(s, e):          # token order inside the chunk
            part += k[:, :, t, :]
        total += part                  # chunk order
    return (total / np.float64(N)).astype(np.float32)


def smooth_k(k, mean):
    """fp32(K) - mean, one FP32 subtraction per element."""
    return (np.asarray(k, np.float32) - np.asarray(mean, np.float32)[:, :, None, :]).astype(np.float32)


def q_block_mean(q):
    """Per-(b, h, 128-token block, channel) mean of Q, reading 2.

    FP64 sum in token order over the block's tokens (a ragged last block:
    its tokens only), divided by their count, rounded to FP32.  Returns
    float32 [B, H, ceil(N/128), d].
    """
    q = np.asarray(q, np.float64)
    B, H, N, d = q.shape
    out = np.zeros((B, H, -(-N // BLOCK), d), np.float32)
    for i, (s, e) in enumerate(_blocks(N)):
        part = np.zeros((B, H, d), np.float64)
        for t in range(s, e):
            part += q[:, :, t, :]
        out[:, :, i, :] = (part / np.float64(e - s)).astype(np.float32)
    return out


def smooth_q(q, qmean):
    """fp32(Q) - qbar of the token's block, one FP32 subtraction per element."""
    q = np.asarray(q, np.float32)
    N = q.shape[2]
    return (q - np.asarray(qmean, np.float32)[:, :, np.arange(N) // BLOCK, :]).astype(np.float32)


def smoothing_bias(qmean, k_smoothed):
    """dS[b, h, blk, j] = qbar[b, h, blk] . k'[b, h, j] (reading 2).

    qmean float32 [B, H, nb, d]; k_smoothed float32 [B, H, N, d].  FP64
    accumulation in channel order c = 0 .. d-1 (every product of two FP32
    values is exact in FP64), rounded once to FP32.  Returns float32
    [B, H, nb, N].
    """
    qm = np.asarray(qmean, np.float32).astype(np.float64)
    kk = np.asarray(k_smoothed, np.float32).astype(np.float64)
    B, H, nb, d = qm.shape
    N = kk.shape[2]
    acc = np.zeros((B, H, nb, N), np.float64)
    for c in range(d):                 # channel order
        acc += qm[:, :, :, c, None] * kk[:, :, None, :, c]
    return acc.astype(np.float32)


def quant_int8_blocks(x, tokens=BLOCK):
    """Symmetric INT8 with one scale per block of `tokens` tokens (reading 3).

    x: float32 [B, H, N, d].  Returns (codes int8 [B,H,N,d],
    scales float32 [B,H,ceil(N/tokens)]).
    """
    x = np.asarray(x, np.float32)
    B, H, N, d = x.shape
    nb = -(-N // tokens)
    codes = np.zeros((B, H, N, d), np.int8)
    scales = np.zeros((B, H, nb), np.float32)
    for i, (s, e) in enumerate(_blocks(N, tokens)):
        blk = x[:, :, s:e, :]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        sc = (amax / INT8_DIV).astype(np.float32)
        scales[:, :, i] = sc
        codes[:, :, s:e, :] = int8_quantize(blk, sc[:, :, None, None])
    return codes, scales


def quant_fp8_blocks(x, tokens=BLOCK):
    """FP8 e4m3 with one scale per block of `tokens` tokens (reading 6).

    x: float32 [B, H, N, d].  Returns (codes uint8 e4m3 [B,H,N,d],
    scales float32 [B,H,ceil(N/tokens)]).
    """
    x = np.asarray(x, np.float32)
    B, H, N, d = x.shape
    nb = -(-N // tokens)
    codes = np.zeros((B, H, N, d), np.uint8)
    scales = np.zeros((B, H, nb), np.float32)
    for i, (s, e) in enumerate(_blocks(N, tokens)):
        blk = x[:, :, s:e, :]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        sc = (amax / FP8_DIV).astype(np.float32)
        scales[:, :, i] = sc
        den = np.where(sc != 0, sc, np.float32(1))[:, :, None, None]
        t = np.where(sc[:, :, None, None] != 0, blk / den, np.float32(0)).astype(np.float32)
        codes[:, :, s:e, :] = e4m3_encode(t)
    return codes, scales


def _q_for_quant(q, k_smoothed, smooth):
    """Q as it enters its quantizer, plus the smoothing outputs (reading 2)."""
    if not smooth:
        return np.asarray(q, np.float32), {}
    qm = q_block_mean(q)
    return smooth_q(q, qm), dict(q_mean=qm, dS=smoothing_bias(qm, k_smoothed))


def quant_qk_fp8(q, k, smooth=False):
    """FP8 Q/K mode pre-pass (reading 6; K smoothed as in reading 1; Q
    smoothed as in reading 2 when `smooth`).

    Returns dict with q_codes, q_scales [B,H,N] (one per token), k_codes,
    k_scales [B,H,ceil(N/32)], k_mean; with `smooth` also q_mean
    [B,H,ceil(N/128),d] and dS [B,H,ceil(N/128),N].
    """
    mean = k_channel_mean(k)
    ks_in = smooth_k(k, mean)
    q_in, extra = _q_for_quant(q, ks_in, smooth)
    qc, qs = quant_fp8_blocks(q_in, Q_GROUP)
    kc, ks = quant_fp8_blocks(ks_in, K_GROUP)
    return dict(q_codes=qc, q_scales=qs, k_codes=kc, k_scales=ks, k_mean=mean, **extra)


def quant_qk_int8(q, k, smooth=False):
    """INT8 mode pre-pass for Q and K (readings 1 and 3; Q smoothed as in
    reading 2 when `smooth`).

    Returns dict with q_codes, q_scales [B,H,N] (one per token), k_codes,
    k_scales [B,H,ceil(N/32)], k_mean; with `smooth` also q_mean
    [B,H,ceil(N/128),d] and dS [B,H,ceil(N/128),N].
    """
    mean = k_channel_mean(k)
    ks_in = smooth_k(k, mean)
    q_in, extra = _q_for_quant(q, ks_in, smooth)
    qc, qs = quant_int8_blocks(q_in, Q_GROUP)
    kc, ks = quant_int8_blocks(ks_in, K_GROUP)
    return dict(q_codes=qc, q_scales=qs, k_codes=kc, k_scales=ks, k_mean=mean, **extra)


def quant_v_fp8(v):
    """FP8 V (reading 4).  Returns (codes uint8 [B,H,d,N], scales f32 [B,H,d])."""
    v = np.asarray(v, np.float32)
    amax = np.abs(v).max(axis=2) if v.shape[2] else np.zeros(v.shape[:2] + v.shape[3:], np.float32)
    s = (amax.astype(np.float32) / FP8_DIV).astype(np.float32)     # [B,H,d]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(s[:, :, None, :] != 0,
                     v / np.where(s != 0, s, np.float32(1))[:, :, None, :],
                     np.float32(0)).astype(np.float32)
    codes = e4m3_encode(t)                                          # [B,H,N,d]
    return np.ascontiguousarray(codes.transpose(0, 1, 3, 2)), s


def _fp4_encode_tile(x, g):
    """Encode one tile with tile scale g (float32 scalar array, broadcast).

    x: float32 [..., L, 16*m] with the 16-element blocks along the last axis.
    g: float32 broadcastable to x[..., 0, 0].
    Returns (codes uint8 [..., L, 16*m], sf uint8 [..., L, m]).
    """
    *lead, L, W = x.shape
    m = W // FP4_VEC
    xb = x.reshape(*lead, L, m, FP4_VEC)
    a16 = np.abs(xb).max(axis=-1).astype(np.float32)                 # [..., L, m]
    g = np.asarray(g, np.float32)[..., None, None]
    six_g = (np.float32(6.0) * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(six_g != 0, a16 / np.where(six_g != 0, six_g, np.float32(1)),
                     np.float32(0)).astype(np.float32)
    sf = ue4m3_encode(r)                                             # [..., L, m]
    s_dec = ue4m3_decode(sf).astype(np.float32)
    den = (s_dec * g).astype(np.float32)                             # fp32(s16 * g)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(den[..., None] != 0,
                     xb / np.where(den != 0, den, np.float32(1))[..., None],
                     np.float32(0)).astype(np.float32)
    codes = e2m1_encode(t)
    # a zero scale gives code 0 (positive zero) whatever the sign of x
    codes = np.where(den[..., None] != 0, codes, 0).astype(np.uint8)
    return codes.reshape(*lead, L, W), sf


def quant_fp4_tokens(x):
    """FP4 encoding of Q or smoothed K (reading 5), 16-blocks over channels.

    x: float32 [B,H,N,d], d % 16 == 0.  Returns (codes uint8 0..15
    [B,H,N,d], sf ue4m3 codes [B,H,N,d/16], g float32 [B,H,ceil(N/128)]).
    """
    x = np.asarray(x, np.float32)
    B, H, N, d = x.shape
    nb = -(-N // BLOCK)
    codes = np.zeros((B, H, N, d), np.uint8)
    sf = np.zeros((B, H, N, d // FP4_VEC), np.uint8)
    g = np.zeros((B, H, nb), np.float32)
    for i, (s, e) in enumerate(_blocks(N)):
        blk = x[:, :, s:e, :]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        gi = (amax / FP4_G_DIV).astype(np.float32)
        g[:, :, i] = gi
        c, f = _fp4_encode_tile(blk, gi)
        codes[:, :, s:e, :] = c
        sf[:, :, s:e, :] = f
    return codes, sf, g


def quant_qk_fp4(q, k, smooth=False):
    """FP4 mode pre-pass for Q and K (readings 1 and 5; Q smoothed as in
    reading 2 when `smooth`)."""
    mean = k_channel_mean(k)
    ks_in = smooth_k(k, mean)
    q_in, extra = _q_for_quant(q, ks_in, smooth)
    qc, qsf, qg = quant_fp4_tokens(q_in)
    kc, ksf, kg = quant_fp4_tokens(ks_in)
    return dict(q_codes=qc, q_sf=qsf, q_g=qg, k_codes=kc, k_sf=ksf, k_g=kg, k_mean=mean, **extra)


def quant_v_fp4(v):
    """FP4 V (reading 5): transposed [B,H,d,N], 16-blocks over tokens.

    A ragged sequence (N % 16 != 0) ends in a partial 16-token group whose
    missing tokens count as zeros (reading 7).  Returns (codes uint8
    [B,H,d,N], sf [B,H,d,ceil(N/16)], g float32 [B,H,ceil(N/128)]).
    """
    v = np.asarray(v, np.float32)
    B, H, N, d = v.shape
    N16 = -(-N // FP4_VEC) * FP4_VEC
    vt = np.zeros((B, H, d, N16), np.float32)                          # [B,H,d,N16]
    vt[..., :N] = v.transpose(0, 1, 3, 2)
    nb = -(-N // BLOCK)
    codes = np.zeros((B, H, d, N16), np.uint8)
    sf = np.zeros((B, H, d, N16 // FP4_VEC), np.uint8)
    g = np.zeros((B, H, nb), np.float32)
    for i, (s, e) in enumerate(_blocks(N16)):
        blk = vt[:, :, :, s:e]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        gi = (amax / FP4_G_DIV).astype(np.float32)
        g[:, :, i] = gi
        c, f = _fp4_encode_tile(blk, gi)
        codes[:, :, :, s:e] = c
        sf[:, :, :, s // FP4_VEC:e // FP4_VEC] = f
    return np.ascontiguousarray(codes[..., :N]), sf, g
