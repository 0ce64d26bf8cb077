"""GPU pre-pass parity: codes and scales bit-identical to the oracle.

Calls the CUDA path through the C ABI (Python binding) and the CPU oracle on
the same seeded inputs.
"""

import numpy as np
import pytest
import torch

import quantized_attention_quant_b200 as sage
from oracle import encoders as enc
from oracle import prepass as pp
from quantized_attention_quant_b200.workloads import WORKLOADS, make_qkv, to_numpy32
from tests import layouts as L

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def rand_qkv(B, H, N, d, dtype, seed, k_bias=3.0):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, H, N, d)).astype(np.float32)
    k = g.standard_normal((B, H, N, d)).astype(np.float32) + \
        g.standard_normal((B, H, 1, d)).astype(np.float32) * k_bias
    v = g.standard_normal((B, H, N, d)).astype(np.float32)
    return [torch.from_numpy(x).to(TDT[dtype]) for x in (q, k, v)]


def check_int8(q, k, v, heads=None, mode="int8_fp8", fused=False):
    """Run the INT8/FP8 (or FP8 Q/K) pre-pass on the GPU; compare (sampled)
    heads.  fused: through sage_quant_qkv (one call for Q, K and V, the
    cluster-fused kernel where the sequence fits in it), else through the
    separate Q/K and V calls (two launches each)."""
    B, H, N, d = q.shape
    dev = torch.device("cuda")
    if fused:
        qk, vq = sage.sage_quant_qkv(q.to(dev), k.to(dev), v.to(dev), mode)
    else:
        qk = sage.sage_quant_qk(q.to(dev), k.to(dev), mode)
        vq = sage.sage_quant_v(v.to(dev), mode)
    torch.cuda.synchronize()
    Np = L.np_of(N)
    nk = -(-N // 32)
    codes = L.token_codes if mode == "fp8" else L.int8_codes
    qsc = L.f32(qk["q_scales"], B, H, Np)          # one per token
    ksc = L.f32(qk["k_scales"], B, H, Np // 32)    # one per 32 tokens
    # padding tokens (and K blocks of padding only) have scale 0
    assert not qsc[:, :, N:].any() and not ksc[:, :, nk:].any()
    g = dict(q_codes=codes(qk["q_codes"], B, H, N, d),
             q_scales=qsc[:, :, :N],
             k_codes=codes(qk["k_codes"], B, H, N, d),
             k_scales=ksc[:, :, :nk],
             k_mean=L.f32(qk["k_mean"], B, H, d),
             v_codes=L.vt_codes(vq["v_codes"], B, H, d, N),
             v_scales=L.f32(vq["v_scales"], B, H, d))
    # the padding of a ragged sequence holds zero codes
    assert not L.padded_tokens(qk["q_codes"], B, H, N).any()
    assert not L.padded_tokens(qk["k_codes"], B, H, N).any()
    assert not L._np(vq["v_codes"]).reshape(B, H, d, Np)[..., N:].any()
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in heads:
        qs, ks, vs = (to_numpy32(t[b:b + 1, h:h + 1]) for t in (q, k, v))
        want = pp.quant_qk_fp8(qs, ks) if mode == "fp8" else pp.quant_qk_int8(qs, ks)
        vc, vsc = pp.quant_v_fp8(vs)
        want.update(v_codes=vc, v_scales=vsc)
        for name, arr in want.items():
            got = g[name][b:b + 1, h:h + 1]
            assert np.array_equal(got.view(np.uint8) if got.dtype != np.float32 else got.view(np.uint32),
                                  arr.view(np.uint8) if arr.dtype != np.float32 else arr.view(np.uint32)), \
                (name, b, h)


def check_fp4(q, k, v, heads=None):
    B, H, N, d = q.shape
    dev = torch.device("cuda")
    qk = sage.sage_quant_qk(q.to(dev), k.to(dev), "fp4")
    vq = sage.sage_quant_v(v.to(dev), "fp4")
    torch.cuda.synchronize()
    nt = -(-N // 128)
    Np = L.np_of(N)
    g = dict(q_codes=L.unpack_fp4(qk["q_codes"], B, H, Np, d)[:, :, :N],
             q_sf=L.qk_sf(qk["q_sf"], B, H, N, d),
             q_g=L.f32(qk["q_scales"], B, H, nt),
             k_codes=L.unpack_fp4(qk["k_codes"], B, H, Np, d)[:, :, :N],
             k_sf=L.qk_sf(qk["k_sf"], B, H, N, d),
             k_g=L.f32(qk["k_scales"], B, H, nt),
             k_mean=L.f32(qk["k_mean"], B, H, d),
             v_codes=L.unpack_fp4(vq["v_codes"], B, H, d, Np)[..., :N],
             v_sf=L.v_sf(vq["v_sf"], B, H, N, d),
             v_g=L.f32(vq["v_scales"], B, H, nt))
    # the padding of a ragged sequence holds zero codes
    assert not L.padded_tokens(qk["q_codes"], B, H, N).any()
    assert not L.padded_tokens(qk["k_codes"], B, H, N).any()
    assert not L.unpack_fp4(vq["v_codes"], B, H, d, Np)[..., N:].any()
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in heads:
        qs, ks, vs = (to_numpy32(t[b:b + 1, h:h + 1]) for t in (q, k, v))
        want = pp.quant_qk_fp4(qs, ks)
        vc, vsf, vg = pp.quant_v_fp4(vs)
        want.update(v_codes=vc, v_sf=vsf, v_g=vg)
        for name, arr in want.items():
            got = g[name][b:b + 1, h:h + 1]
            if arr.dtype == np.float32:
                assert np.array_equal(got.view(np.uint32), arr.view(np.uint32)), (name, b, h)
            else:
                assert np.array_equal(got, arr), (name, b, h)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [128, 384])
def test_int8_prepass_random(cuda_device, dtype, d, N):
    q, k, v = rand_qkv(2, 2, N, d, dtype, seed=N + d)
    check_int8(q, k, v)


def test_int8_prepass_edge_values(cuda_device):
    B, H, N, d = 1, 3, 384, 128
    q, k, v = rand_qkv(B, H, N, d, "bf16", seed=7)
    q[0, 0, 128:256] = 0                      # an all-zero Q block -> s = 0, codes 0
    k[0, 1] = 5.0                             # constant K -> smoothed K = 0
    v[0, 2, :, 3] = 0                         # a zero V channel -> s_V = 0
    q[0, 2, 5, 7] = 3.0e38                    # near the bf16 max
    v[0, 0, 9, 1] = -1.0e-38                  # bf16 subnormal range
    check_int8(q, k, v)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("d", [64, 128])
def test_fp8_qk_prepass_random(cuda_device, dtype, d):
    q, k, v = rand_qkv(2, 2, 384, d, dtype, seed=3 * d + 1)
    check_int8(q, k, v, mode="fp8")


def test_fp8_qk_prepass_edge_values(cuda_device):
    B, H, N, d = 1, 3, 384, 128
    q, k, v = rand_qkv(B, H, N, d, "bf16", seed=8)
    q[0, 0, 128:256] = 0                      # an all-zero Q block -> s = 0, codes 0
    k[0, 1] = -7.0                            # constant K -> smoothed K = 0
    q[0, 2, 5, 7] = 3.0e38                    # near the bf16 max: the rest of its block
                                              # lands in the e4m3 subnormals or at 0
    q[0, 1, 300, 0] = 1.0e-37                 # tiny values next to normal ones
    check_int8(q, k, v, mode="fp8")


def test_fp8_qk_encoder_exhaustive(cuda_device):
    # every finite fp16 value of magnitude <= 448 as Q, with a 448 in channel
    # 0 of every token (Q has one scale per token, so s = 1 and the code is
    # exactly e4m3(x))
    x = np.arange(1 << 16, dtype=np.uint16).view(np.float16).astype(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448)]
    per = 63                                  # values per token (channel 0 keeps the 448)
    ntok = -(-x.size // per)
    ntok = -(-ntok // 128) * 128
    rows = np.zeros((ntok, 64), np.float32)
    flat = np.zeros(ntok * per, np.float32)
    flat[:x.size] = x
    rows[:, 1:] = flat.reshape(ntok, per)
    rows[:, 0] = 448.0
    q = torch.from_numpy(rows.reshape(1, 1, ntok, 64)).to(torch.float16)
    qk = sage.sage_quant_qk(q.cuda(), q.cuda(), "fp8")
    torch.cuda.synchronize()
    assert np.all(L.f32(qk["q_scales"], 1, 1, ntok) == 1.0)
    codes = L.u8(qk["q_codes"], 1, 1, ntok, 64)[0, 0]
    assert np.array_equal(codes[:, 1:].reshape(-1)[:x.size], enc.e4m3_encode(x))


@pytest.mark.parametrize("mode", ["int8_fp8", "fp8", "fp4"])
@pytest.mark.parametrize("N", [1, 77, 200, 300])
def test_prepass_ragged(cuda_device, mode, N):
    d = 128 if mode == "fp4" else 64
    q, k, v = rand_qkv(2, 3, N, d, "bf16", seed=600 + N)
    if mode == "fp4":
        check_fp4(q, k, v)
    else:
        check_int8(q, k, v, mode=mode)


def test_fp8_v_encoder_exhaustive(cuda_device):
    # every finite fp16 value of magnitude <= 448, plus a 448 in each channel
    # (so s_V = 1 and the V code is exactly e4m3(x))
    x = np.arange(1 << 16, dtype=np.uint16).view(np.float16).astype(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448)]
    N = ((x.size + 1 + 127) // 128) * 128
    col = np.zeros(N, np.float32)
    col[0] = 448.0
    col[1:1 + x.size] = x
    v = torch.from_numpy(np.repeat(col[None, None, :, None], 64, axis=3)).to(torch.float16)
    vq = sage.sage_quant_v(v.cuda(), "int8_fp8")
    torch.cuda.synchronize()
    codes = L.u8(vq["v_codes"], 1, 1, 64, N)[0, 0, 0]
    assert np.all(L.f32(vq["v_scales"], 1, 1, 64) == 1.0)
    assert np.array_equal(codes[1:1 + x.size], enc.e4m3_encode(x))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("N", [128, 384])
def test_fp4_prepass_random(cuda_device, dtype, N):
    q, k, v = rand_qkv(2, 2, N, 128, dtype, seed=11 + N)
    check_fp4(q, k, v)


def test_fp4_prepass_edge_values(cuda_device):
    B, H, N, d = 1, 2, 256, 128
    q, k, v = rand_qkv(B, H, N, d, "bf16", seed=12)
    q[0, 0, 0:128] = 0
    k[0, 1] = -2.5
    v[0, 1, 128:256] = 0
    q[0, 1, 3, 0:16] = 1e-30                  # tiny 16-group -> scale rounds to 0
    v[0, 0, 0:16, 5] = -1e-30
    check_fp4(q, k, v)


@pytest.mark.parametrize("name", ["tiny", "llm", "video", "long", "fp4", "short", "n16k"])
@pytest.mark.parametrize("fused", [False, True])
def test_prepass_full_workloads(cuda_device, name, fused):
    """The pre-pass over the full workload tensors, checked on sampled heads;
    fused: through sage_quant_qkv (the launch bench.py times)."""
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    if w.mode == "fp4":
        if fused:
            pytest.skip("FP4 has no sage_quant_qkv-only path")
        check_fp4(q, k, v, heads)
    else:
        check_int8(q, k, v, heads, fused=fused)


# (N, d): through the cluster-fused kernel (8 CTAs, one tile each): one
# token (seven CTAs without a tile), a partial tile, a partial eighth tile,
# eight whole tiles; past it (two-launch chains on two streams): one token
# more, and the llm length
FUSED_SIZES = [(1, 64), (77, 128), (1000, 64), (1024, 128), (1025, 64), (4096, 128)]


@pytest.mark.parametrize("mode", ["int8_fp8", "fp8"])
@pytest.mark.parametrize("N,d", FUSED_SIZES)
def test_quant_qkv_matches_oracle(cuda_device, mode, N, d):
    """sage_quant_qkv (the path sage_attn_fwd takes) is bit-identical to the
    oracle on every head."""
    q, k, v = rand_qkv(1, 3, N, d, "bf16" if d == 128 else "f16", seed=1400 + N + d)
    check_int8(q, k, v, mode=mode, fused=True)


# (B, H): 16 heads (the most the fused kernel takes), 17 (the chains)
@pytest.mark.parametrize("B,H", [(2, 8), (1, 17)])
def test_quant_qkv_head_limit(cuda_device, B, H):
    q, k, v = rand_qkv(B, H, 200, 128, "bf16", seed=1500 + H)
    check_int8(q, k, v, fused=True)


@pytest.mark.parametrize("mode,N,d", [("int8_fp8", 384, 128), ("fp8", 300, 64), ("fp4", 200, 128),
                                      ("int8_fp8", 1024, 128), ("fp8", 1000, 64),
                                      ("int8_fp8", 1025, 128)])
def test_quant_qkv_equals_separate_calls(cuda_device, mode, N, d):
    # sage_quant_qkv (the cluster-fused kernel, or past its size the V chain
    # forked onto the library's second stream) gives the same bytes as the
    # two separate calls
    q, k, v = rand_qkv(2, 3, N, d, "bf16", seed=1200 + N)
    dev = torch.device("cuda")
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    qk1, vq1 = sage.sage_quant_qkv(qg, kg, vg, mode)
    qk2 = sage.sage_quant_qk(qg, kg, mode)
    vq2 = sage.sage_quant_v(vg, mode)
    torch.cuda.synchronize()
    for a, b in list(zip(qk1.values(), qk2.values())) + list(zip(vq1.values(), vq2.values())):
        assert (a is None and b is None) or torch.equal(a, b)
