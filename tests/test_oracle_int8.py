"""Pins for the oracle's int8 KV-cache reading (no GPU).

The quantised cache ("FlashAttention技术深度解析：重塑LLM推理性能的新范式"
§发展趋势 / 量化技术融合 names an INT8/INT4 quantised KV cache without a
format) is read as symmetric per-(token, kv head) rows: scale = max|x| / 127,
code = round-half-even(x / scale), both in float32. These tests pin the
quantiser with hand-computed rows and pin the int8 decode step by reducing it
to the (separately pinned) 16-bit decode on data the int8 format represents
exactly.
"""

import numpy as np
import pytest

from oracle import dequantize_int8, kvcache_decode, kvcache_decode_int8, quantize_int8


def rng(seed):
    return np.random.default_rng(seed)


def test_quantize_hand_rows():
    # max |x| = 63.5 -> scale 0.5; every element is a multiple of 0.5
    codes, scale = quantize_int8(np.array([[63.5, -32.0, 0.0, 0.5, -63.5]]))
    assert scale.dtype == np.float32 and scale[0] == np.float32(0.5)
    np.testing.assert_array_equal(codes[0], [127, -64, 0, 1, -127])
    assert codes.dtype == np.int8
    # max |x| = 127 -> scale 1; x / scale = 2.5, 3.5, -2.5 round half to even
    codes, scale = quantize_int8(np.array([[127.0, 2.5, 3.5, -2.5, 0.4999]]))
    assert scale[0] == 1.0
    np.testing.assert_array_equal(codes[0], [127, 2, 4, -2, 0])


def test_quantize_zero_row_and_shapes():
    x = np.zeros((2, 3, 4))
    x[1, 2] = [0.0, -1.0, 0.25, 0.0]
    codes, scale = quantize_int8(x)
    assert codes.shape == (2, 3, 4) and scale.shape == (2, 3)
    np.testing.assert_array_equal(codes[0], 0)
    np.testing.assert_array_equal(scale[0], 0.0)
    assert scale[1, 2] == np.float32(1.0) / np.float32(127.0)
    np.testing.assert_array_equal(codes[1, 2], [0, -127, 32, 0])  # 0.25 * 127 = 31.75 -> 32


def test_quantize_error_bound_and_range():
    r = rng(3)
    x = (r.standard_normal((64, 128)) * r.uniform(0.01, 30.0, (64, 1))).astype(np.float32)
    codes, scale = quantize_int8(x)
    assert np.all(np.abs(codes.astype(np.int32)) <= 127)
    # the largest element of every row maps to +-127
    np.testing.assert_array_equal(np.max(np.abs(codes.astype(np.int32)), axis=1), 127)
    err = np.abs(dequantize_int8(codes, scale) - x.astype(np.float64))
    bound = scale.astype(np.float64)[:, None] * (0.5 + 127 * 2.0 ** -22)
    assert np.all(err <= bound)


def representable(r, shape, exp_lo=-6, exp_hi=0):
    """Rows of code * 2^e with |code| <= 127 and one +-127 per row: the int8
    format holds them exactly (scale = 2^e exactly), and so do bf16 and fp16."""
    codes = r.integers(-127, 128, shape)
    idx = r.integers(0, shape[-1], shape[:-1])
    np.put_along_axis(codes, idx[..., None], 127 * r.choice([-1, 1], shape[:-1])[..., None], -1)
    e = r.integers(exp_lo, exp_hi + 1, shape[:-1])
    return codes * np.exp2(e)[..., None].astype(np.float64)


@pytest.mark.parametrize("sq,window,softcap,causal", [(1, (-1, -1), 0.0, True),
                                                      (3, (5, 0), 1.3, True),
                                                      (2, (-1, -1), 0.0, False)])
def test_int8_decode_reduces_to_plain_decode(sq, window, softcap, causal):
    """On rows the int8 format represents exactly, the int8 step equals the
    16-bit decode step on the same values, and the appended rows' codes and
    scales are those values' exact decomposition."""
    r = rng(11 + sq)
    B, hq, hkv, D = 3, 4, 2, 16
    lens = [7, 1, 20]
    kc = [representable(r, (n, hkv, D)) for n in lens]
    vc = [representable(r, (n, hkv, D)) for n in lens]
    kn = representable(r, (B, sq, hkv, D))
    vn = representable(r, (B, sq, hkv, D))
    q = r.standard_normal((B, sq, hq, D))
    kq = [quantize_int8(x) for x in kc]
    vq = [quantize_int8(x) for x in vc]
    for b in range(B):
        np.testing.assert_array_equal(dequantize_int8(*kq[b]), kc[b])
        np.testing.assert_array_equal(dequantize_int8(*vq[b]), vc[b])
    o8, l8, akc, aks, avc, avs = kvcache_decode_int8(
        q, kn, vn, [c for c, _ in kq], [s for _, s in kq], [c for c, _ in vq], [s for _, s in vq],
        lens, 0.41, causal, window, softcap)
    o, lse, _, _ = kvcache_decode(q, kn, vn, kc, vc, lens, 0.41, causal, window, softcap)
    np.testing.assert_allclose(o8, o, atol=1e-13)
    np.testing.assert_allclose(l8, lse, atol=1e-13)
    for b in range(B):
        np.testing.assert_array_equal(dequantize_int8(akc[b], aks[b]), kn[b])
        np.testing.assert_array_equal(dequantize_int8(avc[b], avs[b]), vn[b])
        # scale = 2^e exactly
        np.testing.assert_array_equal(np.log2(aks[b]), np.round(np.log2(aks[b])))


def test_int8_decode_without_append_and_first_key_only():
    """No append: the cache prefix alone is attended. A one-key sequence
    returns that key's value row exactly (softmax of a single logit is 1)."""
    r = rng(29)
    B, hq, hkv, D = 2, 2, 1, 8
    lens = [1, 6]
    kc = [representable(r, (n, hkv, D)) for n in lens]
    vc = [representable(r, (n, hkv, D)) for n in lens]
    q = r.standard_normal((B, 1, hq, D))
    kq = [quantize_int8(x) for x in kc]
    vq = [quantize_int8(x) for x in vc]
    o8, l8, akc, _, _, _ = kvcache_decode_int8(
        q, None, None, [c for c, _ in kq], [s for _, s in kq], [c for c, _ in vq],
        [s for _, s in vq], lens, 0.5)
    assert akc == []
    for h in range(hq):
        np.testing.assert_array_equal(o8[0, 0, h], vc[0][0, 0])
        np.testing.assert_allclose(l8[0, h, 0], 0.5 * q[0, 0, h] @ kc[0][0, 0], atol=1e-14)
    o, lse, _, _ = kvcache_decode(q, None, None, kc, vc, lens, 0.5)
    np.testing.assert_allclose(o8, o, atol=1e-13)
    np.testing.assert_allclose(l8, lse, atol=1e-13)


def test_int8_decode_close_to_float_on_random_rows():
    """On arbitrary rows the int8 step moves the output by no more than the
    quantisation error of V plus the softmax's response to that of K."""
    r = rng(31)
    B, hq, hkv, D = 2, 4, 2, 64
    lens = [40, 90]
    kc = [r.standard_normal((n, hkv, D)) for n in lens]
    vc = [r.standard_normal((n, hkv, D)) for n in lens]
    q = r.standard_normal((B, 1, hq, D))
    kq = [quantize_int8(x) for x in kc]
    vq = [quantize_int8(x) for x in vc]
    o8, l8, *_ = kvcache_decode_int8(
        q, None, None, [c for c, _ in kq], [s for _, s in kq], [c for c, _ in vq],
        [s for _, s in vq], lens, D ** -0.5)
    o, lse, _, _ = kvcache_decode(q, None, None, kc, vc, lens, D ** -0.5)
    assert np.max(np.abs(o8 - o)) < 0.03
    assert np.max(np.abs(l8 - lse)) < 0.03


def test_int8_decode_accepts_torch_16bit_inputs():
    """q, k_new, v_new may be torch bf16 tensors (as the GPU tests pass them):
    the result equals the one from the same values as float64 arrays."""
    import torch

    r = rng(37)
    B, sq, hq, hkv, D = 2, 2, 4, 2, 16
    lens = [3, 9]
    kq = [quantize_int8(r.standard_normal((n, hkv, D))) for n in lens]
    vq = [quantize_int8(r.standard_normal((n, hkv, D))) for n in lens]
    t = [torch.randn(s, generator=torch.Generator().manual_seed(i)).to(torch.bfloat16)
         for i, s in enumerate(((B, sq, hq, D), (B, sq, hkv, D), (B, sq, hkv, D)))]
    args = ([c for c, _ in kq], [s for _, s in kq], [c for c, _ in vq], [s for _, s in vq], lens, 0.3)
    a = kvcache_decode_int8(*t, *args)
    b = kvcache_decode_int8(*(x.double().numpy() for x in t), *args)
    for x, y in zip(a[:2], b[:2]):
        np.testing.assert_array_equal(x, y)
    for xs, ys in zip(a[2:], b[2:]):
        for x, y in zip(xs, ys):
            np.testing.assert_array_equal(x, y)


# ---- int4 (the same reading with 7 levels per sign; no kernel yet) ----

def test_quantize_int4_hand_rows():
    from oracle import quantize_int4

    # max |x| = 3.5 -> scale 0.5
    codes, scale = quantize_int4(np.array([[3.5, -1.0, 0.25, 0.75, -3.5]]))
    assert scale[0] == np.float32(0.5)
    # 0.25 / 0.5 = 0.5 -> 0 (half to even); 0.75 / 0.5 = 1.5 -> 2
    np.testing.assert_array_equal(codes[0], [7, -2, 0, 2, -7])
    codes, scale = quantize_int4(np.zeros((1, 4)))
    assert scale[0] == 0 and not codes.any()


def test_int4_packing_round_trip_and_layout():
    from oracle import pack_int4, unpack_int4

    codes = np.array([[-7, 7, 0, -1, 3, -8 + 1]], dtype=np.int8)
    packed = pack_int4(codes)
    # byte 0: low nibble -7 + 8 = 1, high nibble 7 + 8 = 15
    assert packed[0, 0] == (1 | (15 << 4))
    assert packed[0, 1] == (8 | (7 << 4))
    np.testing.assert_array_equal(unpack_int4(packed), codes)
    r = rng(41)
    c = r.integers(-7, 8, (5, 3, 64)).astype(np.int8)
    np.testing.assert_array_equal(unpack_int4(pack_int4(c)), c)


def test_quantize_int4_error_bound():
    from oracle import quantize_int4

    r = rng(43)
    x = (r.standard_normal((64, 128)) * r.uniform(0.01, 30.0, (64, 1))).astype(np.float32)
    codes, scale = quantize_int4(x)
    assert np.all(np.abs(codes.astype(np.int32)) <= 7)
    np.testing.assert_array_equal(np.max(np.abs(codes.astype(np.int32)), axis=1), 7)
    err = np.abs(dequantize_int8(codes, scale) - x.astype(np.float64))
    assert np.all(err <= scale.astype(np.float64)[:, None] * (0.5 + 7 * 2.0 ** -22))


def representable4(r, shape, exp_lo=-4, exp_hi=1):
    """Rows of code * 2^e with |code| <= 7 and one +-7 per row: exact in the
    int4 format (scale = 2^e) and in bf16 / fp16."""
    codes = r.integers(-7, 8, shape)
    idx = r.integers(0, shape[-1], shape[:-1])
    np.put_along_axis(codes, idx[..., None], 7 * r.choice([-1, 1], shape[:-1])[..., None], -1)
    e = r.integers(exp_lo, exp_hi + 1, shape[:-1])
    return codes * np.exp2(e)[..., None].astype(np.float64)


@pytest.mark.parametrize("sq,window,softcap,causal", [(1, (-1, -1), 0.0, True),
                                                      (3, (5, 0), 1.3, True)])
def test_int4_decode_reduces_to_plain_decode(sq, window, softcap, causal):
    from oracle import kvcache_decode_int4, quantize_int4

    r = rng(53 + sq)
    B, hq, hkv, D = 2, 4, 2, 16
    lens = [9, 2]
    kc = [representable4(r, (n, hkv, D)) for n in lens]
    vc = [representable4(r, (n, hkv, D)) for n in lens]
    kn = representable4(r, (B, sq, hkv, D))
    vn = representable4(r, (B, sq, hkv, D))
    q = r.standard_normal((B, sq, hq, D))
    kq = [quantize_int4(x) for x in kc]
    vq = [quantize_int4(x) for x in vc]
    for b in range(B):
        np.testing.assert_array_equal(dequantize_int8(*kq[b]), kc[b])
    o4, l4, akc, aks, avc, avs = kvcache_decode_int4(
        q, kn, vn, [c for c, _ in kq], [s for _, s in kq], [c for c, _ in vq], [s for _, s in vq],
        lens, 0.41, causal, window, softcap)
    o, lse, _, _ = kvcache_decode(q, kn, vn, kc, vc, lens, 0.41, causal, window, softcap)
    np.testing.assert_allclose(o4, o, atol=1e-13)
    np.testing.assert_allclose(l4, lse, atol=1e-13)
    for b in range(B):
        np.testing.assert_array_equal(dequantize_int8(akc[b], aks[b]), kn[b])
        np.testing.assert_array_equal(dequantize_int8(avc[b], avs[b]), vn[b])
        assert np.all(np.abs(akc[b].astype(np.int32)) <= 7)
