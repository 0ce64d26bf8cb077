"""Decoding of the library's buffer layouts into the oracle's array shapes.

Pure indexing (no arithmetic of the method): turns the raw byte buffers that
the C ABI fills into the arrays the oracle returns, so that the two can be
compared element by element.  Code buffers hold Np = N rounded up to a
multiple of 128 tokens per head; the decoders return the first N (padded()
gives the padding itself, which must be zero).
"""

import numpy as np


def _np(t):
    return t.detach().cpu().numpy()


def np_of(N):
    return -(-N // 128) * 128


def int8_codes(buf, B, H, N, d):
    return _np(buf).view(np.int8).reshape(B, H, np_of(N), d)[:, :, :N]


def token_codes(buf, B, H, N, d):
    """Q/K 8-bit codes [B, H, N, d] (padding dropped)."""
    return _np(buf).reshape(B, H, np_of(N), d)[:, :, :N]


def vt_codes(buf, B, H, d, N):
    """V^T 8-bit codes [B, H, d, N] (padding dropped)."""
    return _np(buf).reshape(B, H, d, np_of(N))[..., :N]


def padded_tokens(buf, B, H, N):
    """The padding of a token-major code buffer: tokens N .. Np-1 of every
    head (all bytes of those rows)."""
    return _np(buf).reshape(B, H, np_of(N), -1)[:, :, N:]


def f32(buf, *shape):
    return _np(buf).view(np.float32).reshape(*shape)


def u8(buf, *shape):
    return _np(buf).reshape(*shape)


def unpack_fp4(buf, *shape):
    """Packed e2m1x2 bytes (low nibble = even element) -> codes 0..15."""
    b = _np(buf)
    out = np.empty(b.size * 2, np.uint8)
    out[0::2] = b & 0xF
    out[1::2] = b >> 4
    return out.reshape(*shape)


def sf_rows(buf, BH, ntiles, nchunk, rows_used):
    """Tensor-core scale layout -> [BH, ntiles, rows_used, nchunk*4].

    Byte 16*l + 4*j + s of the 512-byte block (tile t, chunk c) holds row
    32*j + l, 16-group 4*c + s.
    """
    b = _np(buf).reshape(BH, ntiles, nchunk, 32, 4, 4)          # [.., l, j, s]
    b = b.transpose(0, 1, 4, 3, 2, 5)                           # [BH, t, j, l, c, s]
    b = b.reshape(BH, ntiles, 128, nchunk * 4)
    return b[:, :, :rows_used, :]


def qk_sf(buf, B, H, N, d):
    """Q/K FP4 scales -> [B, H, N, d/16] (the oracle's layout)."""
    nt = -(-N // 128)
    r = sf_rows(buf, B * H, nt, d // 64, 128)                   # [BH, t, 128, d/16]
    return r.reshape(B, H, nt * 128, d // 16)[:, :, :N]


def v_sf(buf, B, H, N, d):
    """V FP4 scales -> [B, H, d, ceil(N/16)] (the oracle's layout)."""
    nt = -(-N // 128)
    r = sf_rows(buf, B * H, nt, 2, d)                           # [BH, t, d, 8]
    return r.transpose(0, 2, 1, 3).reshape(B, H, d, nt * 8)[..., :-(-N // 16)]
