"""Exact and emulated-quantized attention (TEST INFRASTRUCTURE ONLY).

Shapes: Q, K, V are [B, H, N, d] arrays holding bf16/fp16 values.

``exact_attention`` is the definition O = softmax(Q K^T * sm_scale + mask) V
evaluated in FP64.

``emulated_sage_attention`` follows the quantized forward pass step by step
(SageAttention / SageAttention2 / SageAttention3 abstracts on the dblp author
page; the kernel-comparison blog's "How FlashAttention reduces memory
traffic" for the tiled online softmax):

  for each query row, over key tiles j = 0, 1, ... of 128 keys, in order
  (causal: only keys t_k <= t_q):
    A      = q_codes . k_codes^T                (exact integer / exact FP64;
                                                 FP8 Q/K mode: e4m3 codes)
    S      = A * s_Q * s_K * sm_scale           (s_Q of the query's token,
                                                 s_K of the key's 32-token
                                                 block; FP4: A * g_Q * g_K *
                                                 sm_scale, block scales
                                                 inside A)
             (+ dS[query block, key] * sm_scale with Q smoothing: the
              SageAttention2 abstract's smoothed Q, prepass reading 2)
    m_new  = max(m, rowmax S)
    alpha  = exp(m - m_new)
    P~     = exp(S - m_new)                     (<= 1)
    p      = quantize(P~)                       (FP8: e4m3(448 P~);
                                                 FP4: per-16-key UE4M3 scale
                                                 with static tile scale 1/2688)
    partial= p . v_codes                        (level 1: fresh per tile, exact)
    O      = alpha O + partial * dequant        (level 2: running accumulator)
    l      = alpha l + rowsum(P~)               (unquantized P~, reading below)
  O / l

Readings (pages silent): the exponential may be taken in any base inside a
kernel (exp2 with log2(e) folded in is the same function); one key tile of
128 keys per level-1 partial; l sums the unquantized P~; the running max is
exact (no lazy rescaling); the causal mask is top-left aligned with
N_q == N_k so no row is ever fully masked.
"""

import numpy as np

from . import prepass as pp
from .encoders import (e4m3_encode, e4m3_decode, e2m1_encode, e2m1_decode,
                       ue4m3_encode, ue4m3_decode, round_to_dtype)

BLOCK = pp.BLOCK
P_FP8_SCALE = 448.0
P_FP4_G = 1.0 / 2688.0
# FP8 Q/K mode: a product of two e4m3 values is exact in FP32, but their sum
# over the d channels is accumulated in FP32 by the tensor core, in an order
# the oracle does not know.  Any order of n FP32 additions errs by at most
# (n - 1) u sum|terms| (u = 2^-24, first order); n <= 128 gives this bound.
FP8_QK_ACC_REL = 2.0 ** -17


def exact_attention(q, k, v, causal=False, sm_scale=None, row_chunk=1024, rows=None):
    """softmax(Q K^T sm_scale + mask) V in FP64, rows in chunks of row_chunk.

    rows: optional query-row indices; then O is [B, H, len(rows), d].
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, N, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((B, H, len(rows), d), np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, len(rows), row_chunk):
                rr = rows[r0:r0 + row_chunk]
                s = (q[b, h, rr] @ k[b, h].T) * sm_scale
                if causal:
                    s = np.where(np.arange(N)[None, :] <= rr[:, None], s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                p = np.exp(s - m)
                out[b, h, r0:r0 + len(rr)] = (p @ v[b, h]) / p.sum(axis=1, keepdims=True)
    return out


# --------------------------------------------------------------------------
# P~ quantizers (per key tile, rows x 128 keys, values in [0, 1])
# --------------------------------------------------------------------------

def quant_p_fp8(pt):
    """p = e4m3(P~ * 448); returns the dequantized-without-scale codes' values.

    The value returned is the E4M3 value of the code (i.e. 448 P~ rounded);
    the caller multiplies by 1/448 at the fold.
    """
    return e4m3_decode(e4m3_encode(pt * P_FP8_SCALE))


def fp8_p_ambiguity(pt, eps):
    """Size of the possible e4m3 code change of 448 P~ under a relative
    perturbation of at most eps (0 where the code is unambiguous).

    A kernel that evaluates P~ in FP32 can land on the other side of a
    rounding midpoint when 448 P~ lies within eps of it; both codes are then
    correct.  Returns |neighbour - code| for such elements.
    """
    x = pt * P_FP8_SCALE
    code = e4m3_encode(x).astype(np.int64) & 0x7F
    r = e4m3_decode(code)
    up = e4m3_decode(np.minimum(code + 1, 0x7E))
    dn = e4m3_decode(np.maximum(code - 1, 0))
    tol = eps * np.maximum(x, 2.0 ** -10)
    near_up = (code < 0x7E) & (np.abs(x - 0.5 * (r + up)) <= tol)
    near_dn = (code > 0) & (np.abs(x - 0.5 * (r + dn)) <= tol)
    return np.where(near_up, up - r, 0.0) + np.where(near_dn, r - dn, 0.0)


def _pad16(pt):
    """P~ with the key axis padded by zeros to a multiple of 16: the last tile
    of a ragged sequence has a partial 16-key group, whose missing keys have
    P~ = 0 (they change neither the group max nor any code)."""
    R, C = pt.shape
    Cp = -(-C // 16) * 16
    if Cp == C:
        return pt
    return np.concatenate([pt, np.zeros((R, Cp - C))], axis=1)


def quant_p_fp4(pt):
    """FP4 P~ with the static tile scale g = 1/2688 and per-16-key UE4M3 scales.

    s16 = ue4m3(amax16 * 448); code = e2m1(P~ / (s16 * g)).  Returns the
    value code * s16 (the caller multiplies by g at the fold).  A partial
    16-key group (ragged last tile) counts its missing keys as P~ = 0.
    """
    C = pt.shape[1]
    pt = _pad16(pt)
    R, Cp = pt.shape
    blk = pt.reshape(R, Cp // 16, 16)
    a16 = blk.max(axis=-1)
    s16 = ue4m3_decode(ue4m3_encode(a16 * P_FP8_SCALE))
    den = s16 * P_FP4_G
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(den[..., None] > 0, blk / np.where(den > 0, den, 1.0)[..., None], 0.0)
    codes = e2m1_decode(e2m1_encode(t))
    return (codes * s16[..., None]).reshape(R, Cp)[:, :C]


def _e2m1_flip(t, eps):
    """|neighbour - value| for the e2m1 code of t >= 0 where t lies within a
    relative eps of a rounding midpoint (either code is then correct); 0
    elsewhere."""
    code = e2m1_encode(t).astype(np.int64) & 0x7
    r = e2m1_decode(code)
    up = e2m1_decode(np.minimum(code + 1, 7))
    dn = e2m1_decode(np.maximum(code - 1, 0))
    tol = eps * np.maximum(t, 2.0 ** -30)
    near_up = (code < 7) & (np.abs(t - 0.5 * (r + up)) <= tol)
    near_dn = (code > 0) & (np.abs(t - 0.5 * (r + dn)) <= tol)
    return np.where(near_up, up - r, 0.0) + np.where(near_dn, r - dn, 0.0)


def fp4_p_ambiguity(pt, eps):
    """Bound on the change of the FP4 P~ values (in the units quant_p_fp4
    returns: code * s16) when P~ is perturbed by a relative eps at most.

    Two decisions can go either way near a midpoint: the UE4M3 group scale
    s16 = ue4m3(448 amax16), which moves every value of the 16-key group,
    and each e2m1 code.  Where the scale is ambiguous the bound covers the
    whole group re-quantized with the neighbouring scale.  eps is a scalar;
    a partial 16-key group is padded as in quant_p_fp4.
    """
    C = pt.shape[1]
    pt = _pad16(pt)
    R, Cp = pt.shape
    blk = pt.reshape(R, Cp // 16, 16)
    x = blk.max(axis=-1) * P_FP8_SCALE
    code = ue4m3_encode(x).astype(np.int64)
    s = ue4m3_decode(code)
    up = ue4m3_decode(np.minimum(code + 1, 0x7E))
    dn = ue4m3_decode(np.maximum(code - 1, 0))
    tol = eps * np.maximum(x, 2.0 ** -30)
    near_up = (code < 0x7E) & (np.abs(x - 0.5 * (s + up)) <= tol)
    near_dn = (code > 0) & (np.abs(x - 0.5 * (s + dn)) <= tol)

    def values(scale):
        den = scale * P_FP4_G
        with np.errstate(divide="ignore", invalid="ignore"):
            t = np.where(den[..., None] > 0, blk / np.where(den > 0, den, 1.0)[..., None], 0.0)
        return e2m1_decode(e2m1_encode(t)) * scale[..., None], _e2m1_flip(t, eps) * scale[..., None]

    base, bound = values(s)
    for near, alt in ((near_up, up), (near_dn, dn)):
        if np.any(near):
            v_alt, b_alt = values(np.where(near, alt, s))
            bound = bound + np.where(near[..., None], np.abs(v_alt - base) + b_alt, 0.0)
    return bound.reshape(R, Cp)[:, :C]


# --------------------------------------------------------------------------
# The tile loop
# --------------------------------------------------------------------------

def _tile_loop(qd, kd, vd, s_row, s_key, v_fold, p_quant, causal, sm_scale, rows=None,
               p_ambiguity=None, qk_acc_rel=0.0, s_bias=None):
    """Online softmax + two-level P~V accumulation for one (b, h).

    qd [N, d], kd [N, d]: decoded code values (exact FP64).
    vd [N, d]: decoded V code values (exact FP64).
    s_row [N]: per-row dequant factor of A (s_Q of the row's block).
    s_key [N]: per-key dequant factor of A (s_K of the key's block).
    v_fold [ntiles, d]: factor applied to a tile's level-1 partial at the fold.
    p_quant: P~ -> quantized P~ values (scaled as the partial expects).
    rows: query rows to compute (default all); each row's arithmetic does not
    depend on which other rows are computed.
    p_ambiguity: optional (P~, extra relative perturbation) -> size of a
    possible code change (see fp8_p_ambiguity); then a second array bounds,
    per output element, how far O can move when every ambiguous code takes
    its other valid value.
    qk_acc_rel: relative accumulation error of the kernel's Q K^T (0 when it
    is exact, as in INT8 mode).  With the bound requested, each score may
    then be off by dS = qk_acc_rel |q| . |k| (dequantized), the running max by
    the largest dS so far (Dm), so each P~ by a factor within exp(+-(dS +
    Dm)): the code decisions get that much extra room, and the row sum (thus
    O / l) a relative deviation of at most expm1(2 Dm).
    s_bias: optional [ceil(N/128), N] score bias of Q smoothing (dS, in the
    units of A * s_Q * s_K): row r's scores gain s_bias[r // 128] * sm_scale.
    Returns O [len(rows), d] in FP64 (before the output rounding), and the
    bound when p_ambiguity is given.
    """
    N, d = qd.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    R = len(rows)
    O = np.zeros((R, d))
    Bd = np.zeros((R, d)) if p_ambiguity is not None else None
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    Dm = np.zeros(R)
    for j, (ks, ke) in enumerate(pp._blocks(N)):
        act = np.nonzero(rows >= ks)[0] if causal else np.arange(R)   # rows that see tile j
        if act.size == 0:
            continue
        r_act = rows[act]
        A = qk_product(qd[r_act], kd[ks:ke])       # exact
        S = A * s_row[r_act, None] * s_key[None, ks:ke] * sm_scale
        if s_bias is not None:
            S = S + s_bias[r_act // BLOCK, ks:ke].astype(np.float64) * sm_scale
        if causal:
            S = np.where(np.arange(ks, ke)[None, :] <= r_act[:, None], S, -np.inf)
        m_new = np.maximum(m[act], S.max(axis=1))
        alpha = np.exp(m[act] - m_new)            # exp(-inf) = 0 on the first tile
        Pt = np.exp(S - m_new[:, None])
        p = p_quant(Pt)
        partial = p @ vd[ks:ke]                   # level 1: exact
        O[act] = alpha[:, None] * O[act] + partial * v_fold[j][None, :]
        if Bd is not None:
            extra = 0.0
            if qk_acc_rel:
                dS = qk_acc_rel * (np.abs(qd[r_act]) @ np.abs(kd[ks:ke]).T) * \
                    s_row[r_act, None] * s_key[None, ks:ke] * sm_scale
                if causal:
                    dS = np.where(np.arange(ks, ke)[None, :] <= r_act[:, None], dS, 0.0)
                Dm[act] = np.maximum(Dm[act], dS.max(axis=1))
                extra = np.expm1(dS + Dm[act][:, None])
            Bd[act] = alpha[:, None] * Bd[act] + \
                (p_ambiguity(Pt, extra) @ np.abs(vd[ks:ke])) * np.abs(v_fold[j])[None, :]
        l[act] = alpha * l[act] + Pt.sum(axis=1)
        m[act] = m_new
    if Bd is not None:
        grow = np.exp(2.0 * Dm)[:, None]
        return O / l[:, None], Bd / l[:, None] * grow + np.abs(O / l[:, None]) * (grow - 1.0)
    return O / l[:, None]


def qk_product(qd, kd):
    """A = qd . kd^T for decoded code values in FP64.  Exact for INT8 codes
    (integer sums below 2^53) and for e4m3 codes (products of 8 significant
    bits spanning 2^-18 .. 2^17.6: 8 + 36 + 7 bits for 128 terms < 53).  FP4
    values times their UE4M3 group scales can span a wider range, where FP64
    errs by at most 128 * 2^-53 of sum|terms| (far below any tolerance)."""
    return qd @ kd.T


def _identity(x):
    return x


def emulated_sage_attention(q, k, v, causal=False, sm_scale=None, mode="int8_fp8",
                            quantizers="faithful", rows=None, ambiguity_eps=None,
                            smooth_q=False):
    """Step-by-step emulation of the quantized forward pass, FP64 O [B,H,N,d].

    mode: "int8_fp8" (INT8 Q/K, FP8 P~ and V), "fp8" (FP8 Q/K, P~ and V) or
    "fp4" (FP4 Q/K/P~/V).
    quantizers="identity" replaces every quantizer by the identity (codes =
    the values, scales = 1, P~ unrounded); the result must then equal
    ``exact_attention`` up to FP64 rounding.
    rows: optional query-row indices; then O is [B, H, len(rows), d] and only
    those rows are computed (the pre-pass still sees every token).
    ambiguity_eps: when given, also return a per-element bound on how far O
    moves if every P~ decision lying within this relative distance of a
    rounding midpoint takes its other (equally valid) value: the e4m3 codes in
    INT8/FP8 and FP8 mode; the UE4M3 group scales and e2m1 codes in FP4 mode.
    In FP8 mode the bound also covers the FP32 accumulation of Q K^T
    (FP8_QK_ACC_REL).
    smooth_q: Q smoothing (prepass reading 2): Q loses its per-block mean
    before quantization and every score of the block gains dS * sm_scale.
    With quantizers="identity" the smoothed Q' and the smoothed K' enter
    unrounded beside the FP32 dS, so the result is exact attention up to the
    FP32 roundings of Q', K' and dS.
    """
    q = np.asarray(q, np.float32)
    k = np.asarray(k, np.float32)
    v = np.asarray(v, np.float32)
    B, H, N, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    nrows = N if rows is None else len(rows)
    out = np.zeros((B, H, nrows, d))
    ntiles = -(-N // BLOCK)
    tile_of = np.arange(N) // BLOCK

    if quantizers == "identity":
        qi, ki, bias = q, k, None
        if smooth_q:
            ki = pp.smooth_k(k, pp.k_channel_mean(k))
            qm = pp.q_block_mean(q)
            qi, bias = pp.smooth_q(q, qm), pp.smoothing_bias(qm, ki)
        for b in range(B):
            for h in range(H):
                ones_n = np.ones(N)
                out[b, h] = _tile_loop(qi[b, h].astype(np.float64), ki[b, h].astype(np.float64),
                                       v[b, h].astype(np.float64), ones_n, ones_n,
                                       np.ones((ntiles, d)), _identity, causal, sm_scale, rows,
                                       s_bias=None if bias is None else bias[b, h])
        return out
    if quantizers != "faithful":
        raise ValueError(quantizers)

    if mode in ("int8_fp8", "fp8"):
        fp8_qk = mode == "fp8"
        bound = np.zeros_like(out) if ambiguity_eps is not None else None
        amb = ((lambda pt, extra: fp8_p_ambiguity(pt, ambiguity_eps + extra))
               if bound is not None else None)
        qk = pp.quant_qk_fp8(q, k, smooth_q) if fp8_qk else pp.quant_qk_int8(q, k, smooth_q)
        vc, vs = pp.quant_v_fp8(v)
        for b in range(B):
            for h in range(H):
                if fp8_qk:
                    qd = e4m3_decode(qk["q_codes"][b, h])
                    kd = e4m3_decode(qk["k_codes"][b, h])
                else:
                    qd = qk["q_codes"][b, h].astype(np.float64)
                    kd = qk["k_codes"][b, h].astype(np.float64)
                vd = e4m3_decode(vc[b, h]).T                      # [N, d]
                s_row = qk["q_scales"][b, h].astype(np.float64)[np.arange(N) // pp.Q_GROUP]
                s_key = qk["k_scales"][b, h].astype(np.float64)[np.arange(N) // pp.K_GROUP]
                v_fold = np.broadcast_to(vs[b, h].astype(np.float64) / P_FP8_SCALE, (ntiles, d))
                res = _tile_loop(qd, kd, vd, s_row, s_key, v_fold, quant_p_fp8,
                                 causal, sm_scale, rows, amb,
                                 FP8_QK_ACC_REL if fp8_qk else 0.0,
                                 qk["dS"][b, h] if smooth_q else None)
                if bound is None:
                    out[b, h] = res
                else:
                    out[b, h], bound[b, h] = res
        return out if bound is None else (out, bound)

    if mode == "fp4":
        bound = np.zeros_like(out) if ambiguity_eps is not None else None
        amb = ((lambda pt, extra: fp4_p_ambiguity(pt, ambiguity_eps + extra))
               if bound is not None else None)
        qk = pp.quant_qk_fp4(q, k, smooth_q)
        vc, vsf, vg = pp.quant_v_fp4(v)
        for b in range(B):
            for h in range(H):
                qd = e2m1_decode(qk["q_codes"][b, h]) * np.repeat(
                    ue4m3_decode(qk["q_sf"][b, h]), 16, axis=1)
                kd = e2m1_decode(qk["k_codes"][b, h]) * np.repeat(
                    ue4m3_decode(qk["k_sf"][b, h]), 16, axis=1)
                vdt = e2m1_decode(vc[b, h]) * np.repeat(ue4m3_decode(vsf[b, h]), 16,
                                                         axis=1)[:, :N]
                s_row = qk["q_g"][b, h].astype(np.float64)[tile_of]
                s_key = qk["k_g"][b, h].astype(np.float64)[tile_of]
                v_fold = (vg[b, h].astype(np.float64) * P_FP4_G)[:, None] * np.ones((1, d))
                res = _tile_loop(qd, kd, vdt.T, s_row, s_key, v_fold, quant_p_fp4,
                                 causal, sm_scale, rows, amb,
                                 s_bias=qk["dS"][b, h] if smooth_q else None)
                if bound is None:
                    out[b, h] = res
                else:
                    out[b, h], bound[b, h] = res
        return out if bound is None else (out, bound)
    raise ValueError(mode)


def sage_attention_output(q, k, v, causal=False, sm_scale=None, mode="int8_fp8", dtype="bf16",
                          smooth_q=False):
    """Emulated O rounded to the input dtype ('bf16' or 'f16'), as float32."""
    return round_to_dtype(emulated_sage_attention(q, k, v, causal, sm_scale, mode,
                                                  smooth_q=smooth_q), dtype)
