"""GPU parity of the int8 KV cache: fa_fwd_kvcache_int8 (paged or contiguous,
split-KV, in-place quantising append, Sq new tokens, rotary, ALiBi) and
fa_kv_quantize_int8 against the oracle's reading of the quantised cache
(per-(token, kv head) rows, scale = max|x| / 127, code = round-half-even(x /
scale) in float32).

The int8 caches the kernel reads are made by the oracle's quantiser on the
CPU and uploaded. Appended rows are compared bitwise (codes and scales);
with rotary, the GPU rotates in float32 and the oracle in float64 before both
round to the 16-bit type, so a key may differ by one rounding step and its
codes by one. Unused slots hold garbage codes and NaN scales, which must not
reach any result.

Outputs are held to the 16-bit cache's bounds (max-abs 1e-2, |dLSE| 1e-3),
and the mean-abs bound 1e-3 is widened by the output's own rounding. An
output row here mixes dequantized rows (code * scale), which are not 16-bit
values, so even a row that sees a single key (window (0, 0)) is rounded once
on output. That rounding averages a quarter of an output ulp, about 2^-10 |O|
for bf16, so the bound is 1e-3 plus the mean of ulp(O_ref) / 4. The 16-bit
cache needs no such term: a one-key row is an exact 16-bit row there."""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import dequantize_int8, kvcache_decode_int8, quantize_int8
from parity_utils import check_fwd_quant as check_fwd_int8

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def _quantised_pools(st, contiguous_capacity=0):
    """The oracle-quantised logical caches of every sequence and the int8
    pools (codes, scales) that hold them (unused slots: code 77, scale NaN)."""
    B = st["q"].shape[0]
    Hkv, D = st["Hkv"], st["D"]
    if contiguous_capacity:
        npg, ps = B, contiguous_capacity
    else:
        npg, ps = st["num_pages"], st["page_size"]
    pools = {n: np.full((npg, ps, Hkv, D), 77, dtype=np.int8) for n in ("kc", "vc")}
    pools.update({n: np.full((npg, Hkv, ps), np.nan, dtype=np.float32) for n in ("ks", "vs")})
    logical = []
    for b in range(B):
        k, v = W.decode_sequence_cache(st, b)
        kc, ks = quantize_int8(k.double().numpy())
        vc, vs = quantize_int8(v.double().numpy())
        logical.append((kc, ks, vc, vs))
        for p in range(k.shape[0]):
            page, slot = (b, p) if contiguous_capacity else (int(st["block_table"][b, p // ps]), p % ps)
            pools["kc"][page, slot] = kc[p]
            pools["vc"][page, slot] = vc[p]
            pools["ks"][page, :, slot] = ks[p]
            pools["vs"][page, :, slot] = vs[p]
    return logical, pools


def _run_case(st, splits, causal=True, window=(-1, -1), softcap=0.0, append=True, heads=None,
              rotary_dim=0, interleaved=False, contiguous_capacity=0, alibi=None):
    dev = torch.device("cuda")
    D = st["D"]
    scale = 1.0 / math.sqrt(D)
    B, Sq, Hq, _ = st["q"].shape
    logical, pools = _quantised_pools(st, contiguous_capacity)
    kc, vc = (torch.from_numpy(pools[n]).to(dev) for n in ("kc", "vc"))
    ks, vs = (torch.from_numpy(pools[n]).to(dev) for n in ("ks", "vs"))
    before = {n: pools[n].copy() for n in pools}
    cos = sin = None
    if rotary_dim:
        cos, sin = W.rotary_tables(st["pages_per_seq"] * st["page_size"] + contiguous_capacity,
                                   rotary_dim)
    bt = None if contiguous_capacity else st["block_table"].to(dev)
    out, lse = fa.fwd_kvcache(st["q"].to(dev), kc, vc, st["cache_seqlens"].to(dev), bt,
                              k_new=st["k_new"].to(dev) if append else None,
                              v_new=st["v_new"].to(dev) if append else None,
                              rotary_cos=None if cos is None else cos.to(dev),
                              rotary_sin=None if sin is None else sin.to(dev),
                              rotary_interleaved=interleaved, scale=scale, causal=causal,
                              window=window, softcap=softcap, num_splits=splits,
                              alibi_slopes=None if alibi is None else alibi.to(dev),
                              k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    rot = {}
    if rotary_dim:
        rot = dict(rotary_cos=cos.double().numpy(), rotary_sin=sin.double().numpy(),
                   rotary_interleaved=interleaved, rotated_dtype=st["dtype"])
    o_ref, l_ref, akc, aks, avc, avs = kvcache_decode_int8(
        st["q"], st["k_new"] if append else None, st["v_new"] if append else None,
        [x[0] for x in logical], [x[1] for x in logical], [x[2] for x in logical],
        [x[3] for x in logical], st["cache_seqlens"].tolist(), scale, causal, window, softcap,
        heads=heads, alibi_slopes=None if alibi is None else alibi.double().numpy(), **rot)
    hs = list(range(Hq)) if heads is None else list(heads)
    check_fwd_int8(out[:, :, hs], lse[:, hs], o_ref[:, :, hs], l_ref[:, hs], st["dtype"],
                   f"int8 decode Sq={Sq} splits={splits} rot={rotary_dim}")
    # the pools: exactly the appended slots changed, to the oracle's codes/scales
    got = {"kc": kc.cpu().numpy(), "vc": vc.cpu().numpy(), "ks": ks.cpu().numpy(),
           "vs": vs.cpu().numpy()}
    expect = {n: before[n].copy() for n in before}
    if append:
        ps = contiguous_capacity or st["page_size"]
        for b in range(B):
            L = int(st["cache_seqlens"][b])
            for t in range(Sq):
                p = L + t
                page, slot = (b, p) if contiguous_capacity else (int(st["block_table"][b, p // ps]), p % ps)
                expect["kc"][page, slot] = akc[b][t]
                expect["ks"][page, :, slot] = aks[b][t]
                expect["vc"][page, slot] = avc[b][t]
                expect["vs"][page, :, slot] = avs[b][t]
                if rotary_dim:
                    # one 16-bit rounding step of the key may move a code by one
                    dk = np.abs(got["kc"][page, slot].astype(np.int32) - akc[b][t].astype(np.int32))
                    assert dk.max() <= 1, f"rotated key codes b{b} t{t}"
                    np.testing.assert_allclose(got["ks"][page, :, slot], aks[b][t], rtol=2.0 ** -7)
                    got["kc"][page, slot] = akc[b][t]
                    got["ks"][page, :, slot] = aks[b][t]
    for n in ("kc", "vc"):
        np.testing.assert_array_equal(got[n], expect[n], err_msg=n)
    for n in ("ks", "vs"):
        np.testing.assert_array_equal(got[n], expect[n], err_msg=n)  # NaN == NaN here
    return out, lse


@pytest.mark.parametrize("splits", [1, 4])
@pytest.mark.parametrize("B,Hq,Hkv,D,dtype,lengths,ps", [
    (3, 8, 2, 128, "bf16", [5, 64, 200], 64),
    (4, 4, 4, 64, "fp16", [0, 63, 127, 500], 128),
    (2, 8, 1, 128, "bf16", [1000, 1], 256),       # MQA, group 8
    (2, 32, 1, 64, "fp16", [129, 700], 64),       # group 32
    (5, 32, 8, 128, "bf16", [1024, 3000, 4095, 4096, 2047], 256),
    (3, 8, 2, 128, "fp16", [5, 300, 1000], 128),  # fp16 queries on the register path
])
def test_int8_decode_small(cuda_ok, B, Hq, Hkv, D, dtype, lengths, ps, splits):
    st = W.make_decode_structure(B, Hq, Hkv, D, 0, max(lengths), ps, dtype,
                                 seed=7 * sum(lengths) + splits, cache_seqlens=lengths)
    _run_case(st, splits)


@pytest.mark.parametrize("window,softcap,causal", [((100, 0), 0.0, True), ((-1, -1), 20.0, True),
                                                   ((37, -1), 0.0, False), ((0, 0), 0.0, True)])
def test_int8_decode_options(cuda_ok, window, softcap, causal):
    st = W.make_decode_structure(3, 8, 2, 128, 0, 700, 64, "bf16", seed=71,
                                 cache_seqlens=[700, 65, 130])
    for splits in (1, 4):
        _run_case(st, splits, causal=causal, window=window, softcap=softcap)


def test_int8_decode_without_append(cuda_ok):
    st = W.make_decode_structure(3, 8, 2, 128, 1, 500, 128, "bf16", seed=73,
                                 cache_seqlens=[1, 129, 500])
    _run_case(st, 1, append=False)
    _run_case(st, 5, append=False)


@pytest.mark.parametrize("Sq,Hq,Hkv,D,dtype,lengths,ps", [
    (2, 8, 2, 128, "bf16", [5, 64, 200], 64),
    (5, 16, 4, 64, "fp16", [3, 300], 128),           # 20 columns, ragged tiles
    (9, 8, 1, 128, "bf16", [700, 31], 64),           # 72 columns: three column blocks
])
@pytest.mark.parametrize("splits", [1, 3])
def test_int8_decode_multi_token(cuda_ok, Sq, Hq, Hkv, D, dtype, lengths, ps, splits):
    st = W.make_decode_structure(len(lengths), Hq, Hkv, D, 0, max(lengths), ps, dtype,
                                 seed=Sq * 101 + sum(lengths), cache_seqlens=lengths, sq=Sq)
    _run_case(st, splits)


@pytest.mark.parametrize("Sq,D,rd,interleaved,dtype", [
    (1, 128, 128, False, "bf16"),
    (3, 128, 64, True, "bf16"),
    (2, 64, 64, False, "fp16"),
])
def test_int8_decode_rotary(cuda_ok, Sq, D, rd, interleaved, dtype):
    st = W.make_decode_structure(3, 8, 2, D, 0, 500, 64, dtype, seed=rd + 3 * Sq,
                                 cache_seqlens=[0, 77, 500], sq=Sq)
    _run_case(st, 2, rotary_dim=rd, interleaved=interleaved)


@pytest.mark.parametrize("Sq,splits,capacity", [(1, 1, 320), (3, 4, 1024), (2, 2, 64)])
def test_int8_decode_contiguous_cache(cuda_ok, Sq, splits, capacity):
    lens = [0, 57, capacity - Sq]
    st = W.make_decode_structure(3, 8, 2, 128, 0, max(lens), 64, "bf16", seed=79 + capacity,
                                 cache_seqlens=lens, sq=Sq)
    _run_case(st, splits, contiguous_capacity=capacity)


def test_int8_decode_alibi(cuda_ok):
    st = W.make_decode_structure(2, 8, 2, 128, 0, 400, 64, "bf16", seed=83,
                                 cache_seqlens=[400, 33], sq=2)
    _run_case(st, 3, alibi=W.alibi_slopes(8))


@pytest.mark.parametrize("D,dtype,ps", [(128, "bf16", 64), (64, "fp16", 128), (128, "fp16", 1)])
def test_kv_quantize_matches_oracle(cuda_ok, D, dtype, ps):
    """fa_kv_quantize_int8 gives the oracle's codes and scales bit for bit,
    zero rows included."""
    g = torch.Generator().manual_seed(D + ps)
    npg, Hkv = 5, 3
    x = (torch.randn(npg, ps, Hkv, D, generator=g) *
         torch.rand(npg, ps, Hkv, 1, generator=g) * 10).to(W.DTYPES[dtype])
    x[0, 0, 1] = 0
    codes, scales = fa.kv_quantize_int8(x.cuda())
    torch.cuda.synchronize()
    rc, rs = quantize_int8(x.double().numpy())
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(scales.cpu().numpy(), np.transpose(rs, (0, 2, 1)))
    assert np.all(dequantize_int8(rc[0, 0, 1], rs[0, 0, 1]) == 0)


@pytest.mark.slow
def test_int8_decode_full_paged_b64(cuda_ok):
    """The bench's decode workload (B64, GQA 32/8, D128, lengths 1024..32768,
    page 256) with an int8 cache; sampled heads."""
    c = W.CONFIGS[5]
    st = W.make_decode_structure(c.B, c.Hq, c.Hkv, c.D, c.len_lo, c.len_hi, c.page_size,
                                 c.dtype, seed=2000 + c.cid)
    for splits in (1, 16):
        _run_case(st, splits, heads=[0, 13, 31])


def test_int8_decode_subnormal_query_column(cuda_ok):
    """A query whose every element is subnormal (the register path scales each
    query column by a power of two into fp16): the result stays finite and
    matches the oracle; other columns of the same block are unaffected."""
    st = W.make_decode_structure(2, 8, 2, 128, 0, 300, 64, "bf16", seed=97,
                                 cache_seqlens=[300, 70])
    st["q"][0, 0, 3] = (torch.randn(128, generator=torch.Generator().manual_seed(1)) * 1e-39).to(
        torch.bfloat16)
    assert st["q"][0, 0, 3].float().abs().max() < 1.2e-38
    _run_case(st, 2)
