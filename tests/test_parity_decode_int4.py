"""GPU parity of the int4 KV cache: fa_fwd_kvcache_int4 (paged or contiguous,
split-KV, in-place quantising append, Sq new tokens, rotary, ALiBi) and
fa_kv_quantize_int4 against the oracle's int4 reading (per-(token, kv head)
rows, scale = max|x| / 7, code = round-half-even(x / scale) in [-7, 7] in
float32, two codes per byte biased by 8, even d in the low nibble).

The cached rows are quantised and packed by the oracle on the CPU and
uploaded; appended rows are compared byte for byte (with rotary, codes
within one step and scales within one 16-bit rounding step, as for int8).
Unused slots hold garbage bytes and NaN scales. Outputs are held to the
quantised-cache bounds of parity_utils.check_fwd_quant."""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import kvcache_decode_int4, pack_int4, quantize_int4, unpack_int4
from parity_utils import check_fwd_quant

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def _pools(st, contiguous_capacity=0):
    B = st["q"].shape[0]
    Hkv, D = st["Hkv"], st["D"]
    npg, ps = (B, contiguous_capacity) if contiguous_capacity else (st["num_pages"], st["page_size"])
    pools = {n: np.full((npg, ps, Hkv, D // 2), 0x5A, dtype=np.uint8) for n in ("kc", "vc")}
    pools.update({n: np.full((npg, Hkv, ps), np.nan, dtype=np.float32) for n in ("ks", "vs")})
    logical = []
    for b in range(B):
        k, v = W.decode_sequence_cache(st, b)
        kc, ks = quantize_int4(k.double().numpy())
        vc, vs = quantize_int4(v.double().numpy())
        logical.append((kc, ks, vc, vs))
        kp, vp = pack_int4(kc), pack_int4(vc)
        for p in range(k.shape[0]):
            page, slot = (b, p) if contiguous_capacity else (int(st["block_table"][b, p // ps]), p % ps)
            pools["kc"][page, slot] = kp[p]
            pools["vc"][page, slot] = vp[p]
            pools["ks"][page, :, slot] = ks[p]
            pools["vs"][page, :, slot] = vs[p]
    return logical, pools


def _run_case(st, splits, causal=True, window=(-1, -1), softcap=0.0, append=True, heads=None,
              rotary_dim=0, interleaved=False, contiguous_capacity=0, alibi=None):
    dev = torch.device("cuda")
    D = st["D"]
    scale = 1.0 / math.sqrt(D)
    B, Sq, Hq, _ = st["q"].shape
    logical, pools = _pools(st, contiguous_capacity)
    kc, vc, ks, vs = (torch.from_numpy(pools[n]).to(dev) for n in ("kc", "vc", "ks", "vs"))
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
    o_ref, l_ref, akc, aks, avc, avs = kvcache_decode_int4(
        st["q"], st["k_new"] if append else None, st["v_new"] if append else None,
        [x[0] for x in logical], [x[1] for x in logical], [x[2] for x in logical],
        [x[3] for x in logical], st["cache_seqlens"].tolist(), scale, causal, window, softcap,
        heads=heads, alibi_slopes=None if alibi is None else alibi.double().numpy(), **rot)
    hs = list(range(Hq)) if heads is None else list(heads)
    check_fwd_quant(out[:, :, hs], lse[:, hs], o_ref[:, :, hs], l_ref[:, hs], st["dtype"],
                    f"int4 decode Sq={Sq} splits={splits} rot={rotary_dim}")
    got = {n: t.cpu().numpy() for n, t in (("kc", kc), ("vc", vc), ("ks", ks), ("vs", vs))}
    expect = {n: before[n].copy() for n in before}
    if append:
        ps = contiguous_capacity or st["page_size"]
        for b in range(B):
            L = int(st["cache_seqlens"][b])
            for t in range(Sq):
                p = L + t
                page, slot = (b, p) if contiguous_capacity else (int(st["block_table"][b, p // ps]), p % ps)
                expect["kc"][page, slot] = pack_int4(akc[b][t])
                expect["ks"][page, :, slot] = aks[b][t]
                expect["vc"][page, slot] = pack_int4(avc[b][t])
                expect["vs"][page, :, slot] = avs[b][t]
                if rotary_dim:
                    dk = np.abs(unpack_int4(got["kc"][page, slot]).astype(np.int32)
                                - akc[b][t].astype(np.int32))
                    assert dk.max() <= 1, f"rotated key codes b{b} t{t}"
                    np.testing.assert_allclose(got["ks"][page, :, slot], aks[b][t], rtol=2.0 ** -7)
                    got["kc"][page, slot] = expect["kc"][page, slot]
                    got["ks"][page, :, slot] = aks[b][t]
    for n in ("kc", "vc", "ks", "vs"):
        np.testing.assert_array_equal(got[n], expect[n], err_msg=n)
    return out, lse


@pytest.mark.parametrize("splits", [1, 4])
@pytest.mark.parametrize("B,Hq,Hkv,D,dtype,lengths,ps", [
    (3, 8, 2, 128, "bf16", [5, 64, 200], 64),
    (2, 8, 1, 128, "bf16", [1000, 1], 256),       # MQA, group 8
    (5, 32, 8, 128, "bf16", [1024, 3000, 4095, 4096, 2047], 256),
    (3, 8, 2, 128, "fp16", [0, 300, 1000], 128),
    (3, 8, 2, 64, "bf16", [5, 64, 200], 64),      # D = 64: the shared-memory scratch path
    (2, 8, 1, 64, "fp16", [1000, 1], 256),
    (5, 32, 8, 64, "bf16", [1024, 3000, 4095, 4096, 2047], 256),
])
def test_int4_decode_small(cuda_ok, B, Hq, Hkv, D, dtype, lengths, ps, splits):
    st = W.make_decode_structure(B, Hq, Hkv, D, 0, max(lengths), ps, dtype,
                                 seed=11 * sum(lengths) + splits, cache_seqlens=lengths)
    _run_case(st, splits)


@pytest.mark.parametrize("window,softcap,causal", [((100, 0), 0.0, True), ((-1, -1), 20.0, True),
                                                   ((37, -1), 0.0, False), ((0, 0), 0.0, True)])
def test_int4_decode_options(cuda_ok, window, softcap, causal):
    st = W.make_decode_structure(3, 8, 2, 128, 0, 700, 64, "bf16", seed=171,
                                 cache_seqlens=[700, 65, 130])
    for splits in (1, 4):
        _run_case(st, splits, causal=causal, window=window, softcap=softcap)


def test_int4_decode_without_append(cuda_ok):
    st = W.make_decode_structure(3, 8, 2, 128, 1, 500, 128, "bf16", seed=173,
                                 cache_seqlens=[1, 129, 500])
    _run_case(st, 1, append=False)
    _run_case(st, 5, append=False)


@pytest.mark.parametrize("Sq,Hq,Hkv,lengths,ps", [(2, 8, 2, [5, 64, 200], 64),
                                                  (9, 8, 1, [700, 31], 64)])
def test_int4_decode_multi_token(cuda_ok, Sq, Hq, Hkv, lengths, ps):
    st = W.make_decode_structure(len(lengths), Hq, Hkv, 128, 0, max(lengths), ps, "bf16",
                                 seed=Sq * 103 + sum(lengths), cache_seqlens=lengths, sq=Sq)
    _run_case(st, 3)


@pytest.mark.parametrize("Sq,rd,interleaved", [(1, 128, False), (3, 64, True)])
def test_int4_decode_rotary(cuda_ok, Sq, rd, interleaved):
    st = W.make_decode_structure(3, 8, 2, 128, 0, 500, 64, "bf16", seed=rd + 5 * Sq,
                                 cache_seqlens=[0, 77, 500], sq=Sq)
    _run_case(st, 2, rotary_dim=rd, interleaved=interleaved)


@pytest.mark.parametrize("Sq,splits,capacity", [(1, 1, 320), (3, 4, 1024)])
def test_int4_decode_contiguous_cache(cuda_ok, Sq, splits, capacity):
    lens = [0, 57, capacity - Sq]
    st = W.make_decode_structure(3, 8, 2, 128, 0, max(lens), 64, "bf16", seed=179 + capacity,
                                 cache_seqlens=lens, sq=Sq)
    _run_case(st, splits, contiguous_capacity=capacity)


def test_int4_decode_alibi(cuda_ok):
    st = W.make_decode_structure(2, 8, 2, 128, 0, 400, 64, "bf16", seed=183,
                                 cache_seqlens=[400, 33], sq=2)
    _run_case(st, 3, alibi=W.alibi_slopes(8))


@pytest.mark.parametrize("D,dtype,ps", [(128, "bf16", 64), (64, "fp16", 128)])
def test_kv_quantize_int4_matches_oracle(cuda_ok, D, dtype, ps):
    g = torch.Generator().manual_seed(D + ps + 4)
    x = (torch.randn(5, ps, 3, D, generator=g) * torch.rand(5, ps, 3, 1, generator=g) * 10).to(
        W.DTYPES[dtype])
    x[0, 0, 1] = 0
    codes, scales = fa.kv_quantize_int4(x.cuda())
    torch.cuda.synchronize()
    rc, rs = quantize_int4(x.double().numpy())
    np.testing.assert_array_equal(codes.cpu().numpy(), pack_int4(rc))
    np.testing.assert_array_equal(scales.cpu().numpy(), np.transpose(rs, (0, 2, 1)))


@pytest.mark.parametrize("D,opts", [(64, dict(window=(30, 0), softcap=20.0)), (64, dict(causal=False))])
def test_int4_decode_head_dim_64_options(cuda_ok, D, opts):
    st = W.make_decode_structure(3, 8, 2, D, 0, 700, 64, "bf16", seed=191 + D,
                                 cache_seqlens=[700, 65, 130], sq=2)
    _run_case(st, 3, **opts)


def test_int4_decode_head_dim_64_rotary_alibi(cuda_ok):
    st = W.make_decode_structure(2, 8, 2, 64, 0, 400, 64, "bf16", seed=197,
                                 cache_seqlens=[400, 33], sq=2)
    _run_case(st, 2, rotary_dim=64, alibi=W.alibi_slopes(8))


def test_int4_decode_rejects_head_dim_256(cuda_ok):
    dev = torch.device("cuda")
    q = torch.zeros(1, 1, 4, 256, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(2, 64, 2, 128, dtype=torch.uint8, device=dev)
    sc = torch.zeros(2, 2, 64, device=dev)
    with pytest.raises(fa.FaError, match="FA_ERR_UNSUPPORTED"):
        fa.fwd_kvcache(q, kc, kc.clone(), torch.zeros(1, dtype=torch.int32, device=dev),
                       torch.zeros(1, 2, dtype=torch.int32, device=dev), k_scale=sc, v_scale=sc)
