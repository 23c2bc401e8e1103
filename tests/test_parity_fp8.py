"""GPU parity of the FP8 forward: fa_fwd_fp8 (through the C ABI) vs the fp64
oracle's exact attention over the dequantized E4M3 inputs.

"FlashAttention 实战指南" §版本怎么选 names an FP8 forward; the reading
(E4M3 codes, one descale per tensor) and the tolerance, derived from the
kernel's rounding of the probabilities to E4M3, are stated in
tests/parity_utils.py (check_fwd_fp8). Cases where every probability the
kernel forms is a power of two are exact in E4M3 and are held to the 16-bit
output rounding alone.
"""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import decode_e4m3, head_fwd, head_probs
from parity_utils import check_fwd_fp8, fp8_sigma, to64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")

OUT = {"bf16": torch.bfloat16, "fp16": torch.float16}
BITS = {"bf16": 7, "fp16": 10}


def _run(d, scale, causal, window, softcap, out="bf16", cu=None, max_seqlen=None, alibi=None):
    dev = torch.device("cuda")
    q, k, v = (d[n].to(dev) for n in ("q", "k", "v"))
    o, lse = fa.fwd_fp8(q, k, v, d["q_descale"], d["k_descale"], d["v_descale"], scale=scale,
                        causal=causal, window=window, softcap=softcap,
                        cu_seqlens=None if cu is None else cu.to(dev), max_seqlen=max_seqlen,
                        alibi_slopes=None if alibi is None else alibi.to(dev),
                        out_dtype=OUT[out])
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return o.cpu(), lse.cpu()


def _deq(d):
    return {n: decode_e4m3(d[n].numpy()) * d[n + "_descale"] for n in ("q", "k", "v")}


def _check_head(o, lse, qh, kh, vh, scale, causal, window, softcap, rows, what, bits, slope=0.0):
    o_ref, l_ref = head_fwd(qh, kh, vh, scale, causal, window[0], window[1], softcap, rows=rows,
                            alibi_slope=slope)
    w = head_probs(qh, kh, scale, causal, window[0], window[1], softcap, rows=rows,
                   alibi_slope=slope)
    return check_fwd_fp8(o, lse, o_ref, l_ref, fp8_sigma(w, vh), what, bits)


SMALL = [
    # B, S, Hq, Hkv, D, out, causal, window, softcap
    (1, 128, 2, 2, 128, "bf16", False, (-1, -1), 0.0),
    (2, 200, 4, 2, 128, "bf16", True, (-1, -1), 0.0),      # ragged tail, GQA
    (1, 1, 2, 1, 128, "bf16", True, (-1, -1), 0.0),        # a single token
    (1, 777, 4, 4, 128, "bf16", True, (100, 0), 0.0),      # sliding window
    (1, 640, 4, 2, 128, "fp16", False, (64, 32), 0.0),     # two-sided window, fp16 out
    (1, 513, 2, 2, 128, "bf16", True, (-1, -1), 50.0),     # softcap 50
    (1, 256, 8, 8, 128, "bf16", True, (-1, -1), 2.0),      # softcap that bites
    (3, 1030, 4, 1, 128, "fp16", True, (-1, -1), 0.0),     # several Q blocks, MQA, B > 1
    (1, 384, 2, 2, 128, "bf16", True, (0, 0), 0.0),        # each row sees itself only
    (1, 300, 2, 2, 256, "bf16", True, (-1, -1), 0.0),      # head dim 256
    (2, 513, 4, 2, 256, "fp16", False, (-1, -1), 0.0),
    (1, 640, 2, 1, 256, "bf16", True, (100, 0), 30.0),
]


@pytest.mark.parametrize("B,S,Hq,Hkv,D,out,causal,window,softcap", SMALL)
def test_fp8_small(cuda_ok, B, S, Hq, Hkv, D, out, causal, window, softcap):
    d = W.make_fp8_inputs(B, S, Hq, Hkv, D, seed=S * 11 + Hq + D)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run(d, scale, causal, window, softcap, out)
    x = _deq(d)
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            _check_head(o[b, :, h], lse[b, h], x["q"][b, :, h], x["k"][b, :, h // g],
                        x["v"][b, :, h // g], scale, causal, window, softcap, None,
                        f"B{B} S{S} H{Hq}/{Hkv} D{D} b{b} h{h}", BITS[out])


def test_fp8_equal_logits_exact(cuda_ok):
    # q = 0: every logit is 0, every probability the kernel forms is the same
    # power of two (exact in E4M3), so O is the causal prefix mean of V up to
    # the float32 sums and the bf16 output rounding
    d = W.make_fp8_inputs(1, 700, 2, 2, 128, seed=21)
    d["q"] = torch.zeros_like(d["q"])
    o, lse = _run(d, 0.1, True, (-1, -1), 0.0)
    v = decode_e4m3(d["v"].numpy()) * d["v_descale"]
    ref = np.cumsum(v[0], axis=0) / np.arange(1, 701)[:, None, None]
    err = np.abs(to64(o[0]) - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-5), float(err.max())
    # the row sum comes from the unrounded P, a quarter of which the cubic
    # 2^x of the FMA pipe evaluates with relative error up to 7.5e-5
    lerr = np.abs(to64(lse[0]) - np.log(np.arange(1, 701))[None, :])
    worst = np.unravel_index(np.argmax(lerr), lerr.shape)
    assert lerr.max() <= 1e-4, (float(lerr.max()), worst, float(to64(lse[0])[worst]))


def test_fp8_power_of_two_probabilities_exact(cuda_ok):
    # q, k with entries 0 or 1 (code 0x38) and scale ln 2: every logit is an
    # integer in the exp2 domain, so every probability is a power of two,
    # exact in E4M3 as long as it stays within 2^-9 .. 2^8 of the row max
    r = np.random.default_rng(8)
    S, H, D = 300, 2, 128
    qb = (r.random((1, S, H, D)) < 1 / 8).astype(np.uint8) * 0x38
    kb = (r.random((1, S, H, D)) < 1 / 8).astype(np.uint8) * 0x38
    d = W.make_fp8_inputs(1, S, H, H, D, seed=9)
    d["q"], d["k"] = torch.from_numpy(qb), torch.from_numpy(kb)
    d["q_descale"] = d["k_descale"] = 1.0
    scale = float(np.float32(math.log(2.0)))
    x = _deq(d)
    logits = np.einsum("shd,thd->hst", x["q"][0], x["k"][0])
    assert logits.max() <= 12  # the row spread stays inside E4M3's exact range
    o, lse = _run(d, scale, True, (-1, -1), 0.0)
    for h in range(H):
        o_ref, l_ref = head_fwd(x["q"][0, :, h], x["k"][0, :, h], x["v"][0, :, h], scale, True)
        err = np.abs(to64(o[0, :, h]) - o_ref)
        assert np.all(err <= (2.0 ** -8 + 1e-4) * np.abs(o_ref) + 1e-5), float(err.max())
        np.testing.assert_allclose(to64(lse[0, h]), l_ref, rtol=0, atol=1e-4)


def test_fp8_varlen_gqa_window_softcap(cuda_ok):
    lengths = [1, 130, 257, 600, 33]
    d = W.make_fp8_varlen_inputs(8, 2, 128, seed=31, lengths=lengths)
    scale = 1.0 / math.sqrt(128)
    cu = d["cu_seqlens"]
    o, lse = _run(d, scale, True, (200, 0), 30.0, cu=cu, max_seqlen=max(lengths))
    x = _deq(d)
    for s, n in enumerate(lengths):
        a = int(cu[s])
        for h in range(8):
            _check_head(o[a:a + n, h], lse[h, a:a + n], x["q"][a:a + n, h], x["k"][a:a + n, h // 4],
                        x["v"][a:a + n, h // 4], scale, True, (200, 0), 30.0, None,
                        f"varlen seq{s} h{h}", 7)


def test_fp8_alibi(cuda_ok):
    d = W.make_fp8_inputs(2, 333, 4, 2, 128, seed=41)
    slopes = W.alibi_slopes(4, B=2)
    scale = 1.0 / math.sqrt(128)
    o, lse = _run(d, scale, True, (-1, -1), 0.0, alibi=slopes)
    x = _deq(d)
    for b in range(2):
        for h in range(4):
            _check_head(o[b, :, h], lse[b, h], x["q"][b, :, h], x["k"][b, :, h // 2],
                        x["v"][b, :, h // 2], scale, True, (-1, -1), 0.0, None, f"alibi b{b} h{h}",
                        7, slope=float(slopes[b, h]))


def test_fp8_deterministic(cuda_ok):
    d = W.make_fp8_inputs(2, 700, 8, 2, 128, seed=5)
    a = _run(d, 0.09, True, (-1, -1), 0.0)
    b = _run(d, 0.09, True, (-1, -1), 0.0)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fp8_rejects(cuda_ok):
    d = W.make_fp8_inputs(1, 64, 2, 2, 64, seed=1)
    dev = torch.device("cuda")
    q, k, v = (d[n].to(dev) for n in ("q", "k", "v"))
    with pytest.raises(fa.FaError, match="FA_ERR_UNSUPPORTED"):
        fa.fwd_fp8(q, k, v, 1.0, 1.0, 1.0)
    d = W.make_fp8_inputs(1, 64, 2, 2, 128, seed=1)
    q, k, v = (d[n].to(dev) for n in ("q", "k", "v"))
    with pytest.raises(fa.FaError, match="FA_ERR_INVALID_ARG"):
        fa.fwd_fp8(q, k, v, 0.0, 1.0, 1.0)
    with pytest.raises(fa.FaError, match="FA_ERR_INVALID_ARG"):
        fa.fwd_fp8(q, k, v, 1.0, float("inf"), 1.0)


def _sample_rows(S, rng, extra=40):
    fixed = [0, 1, 127, 128, 255, 256, 257, S // 2, S - 129, S - 128, S - 2, S - 1]
    rows = set(r for r in fixed if 0 <= r < S)
    rows.update(int(x) for x in rng.integers(0, S, extra))
    return np.array(sorted(rows))


@pytest.mark.slow
def test_fp8_full_causal_8k(cuda_ok):
    """The causal B2 H32 S8192 D128 shape in FP8 (the launch configuration
    bench.py times for the FP8 line); sampled rows of sampled heads."""
    c = W.CONFIGS[3]
    d = W.make_fp8_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, seed=1000 + c.cid)
    o, lse = _run(d, c.scale, True, (-1, -1), 0.0)
    x = _deq(d)
    rng = np.random.default_rng(5)
    for b, h in ((0, 0), (1, 31), (0, 17), (1, 5)):
        rows = _sample_rows(c.S, rng)
        _check_head(o[b, rows, h], lse[b, h, rows], x["q"][b, :, h], x["k"][b, :, h],
                    x["v"][b, :, h], c.scale, True, (-1, -1), 0.0, rows, f"fp8 cfg3 b{b} h{h}", 7)
    assert torch.isfinite(o.float()).all()
