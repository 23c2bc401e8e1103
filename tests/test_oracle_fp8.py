"""Pins for the oracle's FP8 forward reading and for the FP8 tolerance (no GPU).

"FlashAttention 实战指南" §版本怎么选 says FlashAttention-3 runs an FP8
forward and gives no format. The reading: Q, K, V are FP8 E4M3 codes with one
float32 descale per tensor, each code standing for value(code) * descale, and
the result is exact attention over those values. These tests pin the E4M3
decoder with hand-worked bit patterns and against torch's own float8 type,
pin the descale semantics by invariants and closed forms, and check the
tolerance model of the GPU comparison (tests/parity_utils.py) against a
direct simulation of the one rounding the model describes.
"""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import attention_fwd, attention_fwd_fp8, decode_e4m3, head_fwd, head_probs
from parity_utils import check_fwd_fp8, fp8_sigma


def test_decode_e4m3_hand_values():
    # sign | exponent (bias 7) | mantissa, worked by hand from the format
    cases = {
        0x00: 0.0,
        0x01: 2.0 ** -9,          # smallest subnormal: 1 * 2^-9
        0x07: 7 * 2.0 ** -9,      # largest subnormal
        0x08: 2.0 ** -6,          # smallest normal: e = 1 -> 2^(1-7)
        0x38: 1.0,                # e = 7, m = 0
        0x3C: 1.5,                # e = 7, m = 4 -> 1 + 4/8
        0x40: 2.0,
        0x7E: 448.0,              # e = 15, m = 6 -> 1.75 * 2^8
        0x78: 256.0,              # e = 15, m = 0 is an ordinary value
        0xB8: -1.0,
        0xFE: -448.0,
        0x81: -(2.0 ** -9),
    }
    for code, val in cases.items():
        assert decode_e4m3(np.array([code]))[0] == val, hex(code)
    assert np.isnan(decode_e4m3(np.array([0x7F]))[0])
    assert np.isnan(decode_e4m3(np.array([0xFF]))[0])
    z = decode_e4m3(np.array([0x80]))[0]
    assert z == 0.0 and math.copysign(1.0, z) == -1.0


def test_decode_e4m3_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(decode_e4m3(codes), ref)


def test_input_recipe_roundtrip():
    # the encoding the inputs come with: descale = amax / 448 and every code
    # within half a spacing of x / descale; the largest element maps to 448
    x = torch.randn(4, 64, 2, 128, generator=torch.Generator().manual_seed(1))
    codes, descale = W.to_e4m3(x)
    v = decode_e4m3(codes.numpy())
    y = x.to(torch.float64).numpy() / descale
    assert np.max(np.abs(v)) == 448.0
    spacing = np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6))) - 3)
    assert np.all(np.abs(v - y) <= spacing / 2 + 1e-9 * np.abs(y))


def rand_codes(r, shape, lo=-448.0, hi=448.0):
    x = torch.from_numpy(r.uniform(lo, hi, shape))
    return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_fp8_descales():
    r = np.random.default_rng(2)
    q, k, v = (rand_codes(r, (1, 16, 2, 32)) for _ in range(3))
    o, lse = attention_fwd_fp8(q, k, v, 0.01, 0.02, 0.5, 0.1, causal=True)
    # only the product q_descale * k_descale enters the logits
    o2, lse2 = attention_fwd_fp8(q, k, v, 0.02, 0.01, 0.5, 0.1, causal=True)
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)
    # and the product with scale
    o3, lse3 = attention_fwd_fp8(q, k, v, 0.01, 0.02, 0.5, 1.0, causal=True)
    o4, lse4 = attention_fwd_fp8(q, k, v, 0.1, 0.02, 0.5, 0.1, causal=True)
    np.testing.assert_allclose(o3, o4, rtol=1e-13, atol=1e-12)
    # v_descale scales the output linearly and leaves LSE alone
    o5, lse5 = attention_fwd_fp8(q, k, v, 0.01, 0.02, 1.5, 0.1, causal=True)
    np.testing.assert_allclose(o5, 3.0 * o, rtol=1e-13, atol=1e-12)
    np.testing.assert_array_equal(lse5, lse)


def test_fp8_closed_forms():
    r = np.random.default_rng(3)
    v = rand_codes(r, (1, 10, 1, 16))
    vv = decode_e4m3(v) * 0.25
    k = rand_codes(r, (1, 10, 1, 16))
    q = np.zeros((1, 10, 1, 16), dtype=np.uint8)  # code 0 is 0.0: every logit is 0
    o, lse = attention_fwd_fp8(q, k, v, 1.0, 1.0, 0.25, 0.3, causal=True)
    for i in range(10):
        np.testing.assert_allclose(o[0, i, 0], vv[0, : i + 1, 0].mean(axis=0), rtol=0, atol=1e-13)
        assert abs(lse[0, 0, i] - math.log(i + 1)) < 1e-13
    # one dominant logit selects its V row: q = k_3 (all 448), others 0
    k = np.zeros((1, 10, 1, 16), dtype=np.uint8)
    k[0, 3, 0] = 0x7E
    q = np.full((1, 1, 1, 16), 0x7E, dtype=np.uint8)
    kk = np.concatenate([k], axis=1)
    o, _ = attention_fwd_fp8(np.repeat(q, 10, axis=1), kk, v, 1.0, 1.0, 0.25, 1e-3)
    np.testing.assert_allclose(o[0, 0, 0], vv[0, 3, 0], rtol=1e-12, atol=1e-12)


def test_head_probs():
    r = np.random.default_rng(4)
    q = r.standard_normal((12, 8))
    k = r.standard_normal((12, 8))
    v = r.standard_normal((12, 8))
    for causal, wl, sc in ((False, -1, 0.0), (True, -1, 0.0), (True, 3, 5.0)):
        w = head_probs(q, k, 0.4, causal, wl, -1, sc)
        o, _ = head_fwd(q, k, v, 0.4, causal, wl, -1, sc)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-13)
        np.testing.assert_allclose(w @ v, o, rtol=0, atol=1e-13)
        if causal:
            assert np.all(np.triu(w, 1) == 0.0)


def simulate_fp8_pv(x_log2, v, offset=4.0):
    """The one rounding the tolerance model describes, simulated: P scaled so
    the row max is 2^offset, rounded to E4M3 (torch's float8 cast, round to
    nearest even), multiplied by V exactly and divided by the exact sum of the
    unrounded P."""
    m = np.max(x_log2, axis=1, keepdims=True)
    p = np.exp2(x_log2 - m + offset)
    pq = torch.from_numpy(p).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    return (pq @ v) / p.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("n,spread", [(3, 1.0), (40, 1.0), (2000, 1.0), (2000, 4.0), (500, 12.0)])
def test_tolerance_model_covers_p_rounding(n, spread):
    # rows of n keys with logits of the given spread (in log2 units), as in
    # the FP8 kernel; the simulated error must stay within the derived bound
    r = np.random.default_rng(n)
    x = r.standard_normal((64, n)) * spread
    v = r.standard_normal((n, 16)) * 3.0
    w = np.exp2(x - x.max(axis=1, keepdims=True))
    w /= w.sum(axis=1, keepdims=True)
    exact = w @ v
    sim = simulate_fp8_pv(x, v)
    sigma = fp8_sigma(w, v)
    err = np.abs(sim - exact)
    assert np.all(err <= 6.0 * sigma + 1e-12)
    ratio = np.sqrt(np.mean((err / sigma) ** 2))
    assert 0.05 < ratio <= 1.0, ratio  # below 1, and not vacuous


def test_tolerance_check_rejects_a_wrong_output():
    # the comparison must fail for a plausible kernel mistake: P.V with one
    # key's probability dropped, or V rows shifted by one key
    r = np.random.default_rng(7)
    q = r.standard_normal((64, 32))
    k = r.standard_normal((64, 32))
    v = r.standard_normal((64, 32))
    w = head_probs(q, k, 0.2, True)
    o, lse = head_fwd(q, k, v, 0.2, True)
    sigma = fp8_sigma(w, v)
    check_fwd_fp8(o, lse, o, lse, sigma, "identical")
    shifted = w[:, :-1] @ v[1:]
    bad = o.copy()
    bad[:, :] = np.concatenate([o[:1], shifted[1:]], axis=0)
    with pytest.raises(AssertionError):
        check_fwd_fp8(bad, lse, o, lse, sigma, "shifted V")
    drop = w.copy()
    drop[np.arange(64), np.arange(64)] = 0.0  # the diagonal key's weight lost
    with pytest.raises(AssertionError):
        check_fwd_fp8(drop @ v, lse, o, lse, sigma, "dropped key")


def test_fp8_varlen_recipe_and_gqa():
    d = W.make_fp8_varlen_inputs(4, 2, 32, seed=9, lengths=[5, 17, 1])
    assert d["q"].shape == (23, 4, 32) and d["k"].shape == (23, 2, 32)
    o, lse = attention_fwd_fp8(d["q"].numpy(), d["k"].numpy(), d["v"].numpy(), d["q_descale"],
                               d["k_descale"], d["v_descale"], 0.2, True,
                               cu_seqlens=d["cu_seqlens"].numpy())
    # GQA: equal to the same attention with repeated kv heads
    qv = decode_e4m3(d["q"].numpy()) * d["q_descale"]
    kv = np.repeat(decode_e4m3(d["k"].numpy()) * d["k_descale"], 2, axis=1)
    vv = np.repeat(decode_e4m3(d["v"].numpy()) * d["v_descale"], 2, axis=1)
    o2, lse2 = attention_fwd(qv, kv, vv, 0.2, True, cu_seqlens=d["cu_seqlens"].numpy())
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)
