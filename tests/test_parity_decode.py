"""GPU decode parity: fa_fwd_kvcache (paged, split-KV, in-place append, Sq
new tokens, rotary) vs the oracle, which attends over a logical contiguous
cache and never reads the page table. The page pool after the call must equal
the pool before it with exactly the appended slots changed: bitwise for plain
appends; with rotary, rotated keys within one 16-bit rounding step of the
oracle's (the GPU rotates in float32, the oracle in float64, and both round
the result to the storage type, so a value lying within float32 error of a
rounding boundary may round the other way)."""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import kvcache_decode
from parity_utils import check_fwd, to64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")

# one rounding step of the storage type, relative, plus the float32 error of
# a rotation of O(1) values (a cos - b sin can cancel)
ROT_RTOL = {"bf16": 2.0 ** -7, "fp16": 2.0 ** -10}
ROT_ATOL = 1e-5


def _slot(st, b, pos, contiguous):
    """(page, slot) of logical position pos of sequence b."""
    if contiguous:
        return b, pos
    ps = st["page_size"]
    return int(st["block_table"][b, pos // ps]), pos % ps


def _run_case(st, splits, causal=True, window=(-1, -1), softcap=0.0, append=True, scale=None,
              heads=None, check_pool=True, rotary_dim=0, interleaved=False, fill=(3.0, -5.0),
              contiguous_capacity=0):
    """contiguous_capacity > 0: a contiguous (B, capacity, Hkv, D) cache and no
    block table instead of the paged pool."""
    dev = torch.device("cuda")
    D = st["D"]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    Hkv = st["Hkv"]
    dt = W.DTYPES[st["dtype"]]
    B, Sq, Hq, _ = st["q"].shape
    contiguous = contiguous_capacity > 0
    if contiguous:
        shape = (B, contiguous_capacity, Hkv, D)
    else:
        shape = (st["num_pages"], st["page_size"], Hkv, D)
    # unused slots hold a recognisable pattern (or NaN) so stray reads show up
    kc = torch.full(shape, fill[0], dtype=dt, device=dev)
    vc = torch.full(shape, fill[1], dtype=dt, device=dev)
    if contiguous:
        for b in range(B):
            k, v = W.decode_sequence_cache(st, b)
            kc[b, :k.shape[0]].copy_(k.to(dev))
            vc[b, :v.shape[0]].copy_(v.to(dev))
    else:
        W.fill_paged_pool(st, kc, vc)
    k_before = kc.clone() if check_pool else None
    v_before = vc.clone() if check_pool else None
    q = st["q"].to(dev)
    kn = st["k_new"].to(dev) if append else None
    vn = st["v_new"].to(dev) if append else None
    cos = sin = None
    if rotary_dim:
        cos, sin = W.rotary_tables(st["pages_per_seq"] * st["page_size"], rotary_dim)
    bt = None if contiguous else st["block_table"].to(dev)
    out, lse = fa.fwd_kvcache(q, kc, vc, st["cache_seqlens"].to(dev), bt,
                              k_new=kn, v_new=vn,
                              rotary_cos=None if cos is None else cos.to(dev),
                              rotary_sin=None if sin is None else sin.to(dev),
                              rotary_interleaved=interleaved, scale=scale, causal=causal,
                              window=window, softcap=softcap, num_splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    assert out.shape == (B, Sq, Hq, D) and lse.shape == (B, Hq, Sq)
    logical = [W.decode_sequence_cache(st, b) for b in range(B)]
    rot = {}
    if rotary_dim:
        rot = dict(rotary_cos=cos.double().numpy(), rotary_sin=sin.double().numpy(),
                   rotary_interleaved=interleaved, rotated_dtype=st["dtype"])
    o_ref, l_ref, ks, vs = kvcache_decode(st["q"], st["k_new"] if append else None,
                                          st["v_new"] if append else None,
                                          [c[0] for c in logical], [c[1] for c in logical],
                                          st["cache_seqlens"].tolist(), scale, causal, window,
                                          softcap, heads=heads, **rot)
    hs = list(range(Hq)) if heads is None else list(heads)
    check_fwd(out[:, :, hs], lse[:, hs], o_ref[:, :, hs], l_ref[:, hs],
              f"decode Sq={Sq} splits={splits} rot={rotary_dim}")
    if check_pool:
        def changed(a, b):
            same = (a == b) | (torch.isnan(a) & torch.isnan(b))
            return (~same).any(dim=(2, 3))

        changed_k = changed(kc, k_before)
        changed_v = changed(vc, v_before)
        expect = torch.zeros_like(changed_k)
        if append:
            for b in range(B):
                L = int(st["cache_seqlens"][b])
                for t in range(Sq):
                    page, slot = _slot(st, b, L + t, contiguous)
                    pos = L + t
                    expect[page, slot] = True
                    assert torch.equal(vc[page, slot].cpu(), st["v_new"][b, t])
                    got_k = kc[page, slot].cpu()
                    if rotary_dim:
                        ref_k = ks[b][pos]
                        err = np.abs(to64(got_k) - ref_k)
                        assert np.all(err <= ROT_RTOL[st["dtype"]] * np.abs(ref_k) + ROT_ATOL), \
                            f"rotated key b{b} t{t}: max err {err.max():.3e}"
                    else:
                        assert torch.equal(got_k, st["k_new"][b, t])
        # a slot may also legitimately keep its value if k_new equals the old one
        assert not (changed_k & ~expect).any() and not (changed_v & ~expect).any()
    return out, lse


SMALL = [
    # B, Hq, Hkv, D, dtype, lengths, page_size
    (3, 8, 2, 128, "bf16", [5, 64, 200], 64),
    (4, 4, 4, 64, "fp16", [0, 63, 127, 500], 128),
    (2, 8, 1, 128, "bf16", [1000, 1], 256),       # MQA, group 8
    (2, 16, 1, 128, "bf16", [300, 77], 64),       # group 16
    (2, 32, 1, 64, "fp16", [129, 700], 64),       # group 32
    (5, 32, 8, 128, "bf16", [1024, 3000, 4095, 4096, 2047], 256),
]


@pytest.mark.parametrize("splits", [1, 3, 16])
@pytest.mark.parametrize("B,Hq,Hkv,D,dtype,lengths,ps", SMALL)
def test_decode_small(cuda_ok, B, Hq, Hkv, D, dtype, lengths, ps, splits):
    st = W.make_decode_structure(B, Hq, Hkv, D, 0, max(lengths), ps, dtype,
                                 seed=sum(lengths) + splits, cache_seqlens=lengths)
    _run_case(st, splits)


@pytest.mark.parametrize("window,softcap,causal", [((100, 0), 0.0, True), ((-1, -1), 20.0, True),
                                                   ((37, -1), 0.0, False), ((0, 0), 0.0, True)])
def test_decode_options(cuda_ok, window, softcap, causal):
    st = W.make_decode_structure(3, 8, 2, 128, 0, 700, 64, "bf16", seed=17,
                                 cache_seqlens=[700, 65, 130])
    for splits in (1, 4):
        _run_case(st, splits, causal=causal, window=window, softcap=softcap)


def test_decode_without_append(cuda_ok):
    st = W.make_decode_structure(3, 8, 2, 128, 1, 500, 128, "bf16", seed=23,
                                 cache_seqlens=[1, 129, 500])
    _run_case(st, 1, append=False)
    _run_case(st, 5, append=False)


@pytest.mark.parametrize("Sq,Hq,Hkv,D,dtype,lengths,ps", [
    (2, 8, 2, 128, "bf16", [5, 64, 200], 64),        # 8 columns: one tile
    (4, 8, 2, 128, "bf16", [0, 61, 1000], 64),       # 16 columns
    (5, 16, 4, 64, "fp16", [3, 300], 128),           # 20 columns, ragged tiles
    (9, 8, 1, 128, "bf16", [700, 31], 64),           # 72 columns: three column blocks
    (3, 32, 1, 128, "bf16", [129, 2000], 256),       # group 32 x 3 tokens
])
@pytest.mark.parametrize("splits", [1, 3])
def test_decode_multi_token(cuda_ok, Sq, Hq, Hkv, D, dtype, lengths, ps, splits):
    """Sq new tokens per sequence: bottom-right causal over the L + Sq keys."""
    st = W.make_decode_structure(len(lengths), Hq, Hkv, D, 0, max(lengths), ps, dtype,
                                 seed=Sq * 100 + sum(lengths), cache_seqlens=lengths, sq=Sq)
    _run_case(st, splits)


@pytest.mark.parametrize("window,softcap,causal", [((7, 0), 0.0, True), ((-1, -1), 5.0, True),
                                                   ((-1, -1), 0.0, False), ((20, 2), 0.0, False),
                                                   ((0, 0), 0.0, True)])
def test_decode_multi_token_options(cuda_ok, window, softcap, causal):
    st = W.make_decode_structure(3, 8, 2, 128, 0, 300, 64, "bf16", seed=41,
                                 cache_seqlens=[300, 3, 128], sq=6)
    for splits in (1, 4):
        _run_case(st, splits, causal=causal, window=window, softcap=softcap)


def test_decode_multi_token_without_append(cuda_ok):
    """No append: the Sq queries sit at L - Sq .. L - 1; with L < Sq the first
    queries precede every key and (causal) see none: O = 0, LSE = -inf."""
    st = W.make_decode_structure(3, 8, 2, 64, 1, 400, 64, "bf16", seed=43,
                                 cache_seqlens=[2, 65, 400], sq=4)
    _run_case(st, 1, append=False)
    _run_case(st, 3, append=False)
    _run_case(st, 2, append=False, causal=False)


@pytest.mark.parametrize("Sq,D,rd,interleaved,dtype", [
    (1, 128, 128, False, "bf16"),
    (1, 128, 128, True, "bf16"),
    (3, 128, 64, False, "bf16"),   # rotary on the first half of the dims only
    (2, 64, 32, True, "fp16"),
    (4, 64, 64, False, "fp16"),
])
@pytest.mark.parametrize("splits", [1, 4])
def test_decode_rotary(cuda_ok, Sq, D, rd, interleaved, dtype, splits):
    """q and the new keys rotated at their positions; the cache keeps the
    rotated keys."""
    st = W.make_decode_structure(3, 8, 2, D, 0, 500, 64, dtype, seed=rd + Sq + splits,
                                 cache_seqlens=[0, 77, 500], sq=Sq)
    _run_case(st, splits, rotary_dim=rd, interleaved=interleaved)


def test_decode_rotary_without_append(cuda_ok):
    """Rotary without k_new: only q is rotated (at L - Sq + t)."""
    st = W.make_decode_structure(2, 8, 2, 128, 4, 300, 64, "bf16", seed=47,
                                 cache_seqlens=[4, 300], sq=3)
    _run_case(st, 2, append=False, rotary_dim=128)


@pytest.mark.parametrize("Sq,splits", [(1, 1), (1, 4), (3, 2)])
def test_decode_ignores_nan_in_unused_slots(cuda_ok, Sq, splits):
    """A pool straight from an uninitialised allocation may hold NaN bit
    patterns past each sequence's end; they must not reach the result (the
    kernel reads whole 64-token chunks of the last page)."""
    st = W.make_decode_structure(3, 8, 2, 128, 0, 300, 64, "bf16", seed=53,
                                 cache_seqlens=[5, 64, 299], sq=Sq)
    nan = float("nan")
    _run_case(st, splits, fill=(nan, nan))
    _run_case(st, splits, fill=(nan, nan), append=False)


@pytest.mark.parametrize("Sq,splits,capacity,rd", [(1, 1, 301, 0), (1, 4, 1000, 0), (4, 3, 310, 64),
                                                    (2, 1, 64, 0)])
def test_decode_contiguous_cache(cuda_ok, Sq, splits, capacity, rd):
    """block_table NULL: a contiguous (B, capacity, Hkv, D) cache, capacity not
    a multiple of the 64-token chunk; the slots past each sequence (and the
    next sequence's rows that a chunk straddles) hold NaN."""
    lens = [0, 57, capacity - Sq]
    st = W.make_decode_structure(3, 8, 2, 128, 0, max(lens), 64, "bf16", seed=59 + capacity,
                                 cache_seqlens=lens, sq=Sq)
    nan = float("nan")
    _run_case(st, splits, fill=(nan, nan), contiguous_capacity=capacity, rotary_dim=rd)


def test_decode_split_counts_agree(cuda_ok):
    """Different num_splits give the same answer up to rounding."""
    st = W.make_decode_structure(2, 8, 2, 128, 0, 2000, 256, "bf16", seed=29,
                                 cache_seqlens=[2000, 1500])
    outs = [_run_case(st, s, check_pool=False)[0].float() for s in (1, 2, 7, 32)]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() < 1e-2


@pytest.mark.slow
def test_decode_full_paged_b64(cuda_ok):
    """B64, GQA 32/8, D128, cache lengths 1024..32768, page 256, block table a
    random permutation; num_splits 1, 4, 16 (the workload bench.py times)."""
    c = W.CONFIGS[5]
    st = W.make_decode_structure(c.B, c.Hq, c.Hkv, c.D, c.len_lo, c.len_hi, c.page_size,
                                 c.dtype, seed=1000 + c.cid)
    for splits in c.splits:
        _run_case(st, splits, heads=[0, 13, 31], check_pool=(splits == 1))


@pytest.mark.parametrize("B,Hq,Hkv,Sq,dtype,lengths,ps,rd,splits", [
    (3, 8, 2, 1, "bf16", [5, 64, 700], 64, 0, 1),          # head dim 256, one column tile
    (3, 8, 2, 1, "fp16", [0, 129, 1000], 128, 0, 4),
    (2, 8, 1, 3, "bf16", [300, 77], 64, 128, 3),           # 24 columns: two tiles, two blocks
    (2, 32, 8, 1, "bf16", [2047, 4096], 256, 256, 16),     # rotary over the whole head
])
def test_decode_head_dim_256(cuda_ok, B, Hq, Hkv, Sq, dtype, lengths, ps, rd, splits):
    """Head dim 256 on a 16-bit cache (the guide's §版本怎么选: head dims up to
    256): three 64 KB stages, at most two 8-column tiles per CTA."""
    st = W.make_decode_structure(B, Hq, Hkv, 256, 0, max(lengths), ps, dtype,
                                 seed=sum(lengths) + Sq + splits, cache_seqlens=lengths, sq=Sq)
    _run_case(st, splits, rotary_dim=rd)


def test_decode_head_dim_256_options(cuda_ok):
    st = W.make_decode_structure(2, 8, 2, 256, 0, 500, 64, "bf16", seed=61,
                                 cache_seqlens=[500, 33], sq=2)
    nan = float("nan")
    _run_case(st, 2, window=(100, 0), softcap=20.0, fill=(nan, nan))
    _run_case(st, 1, causal=False, append=False)
    _run_case(st, 3, contiguous_capacity=600)
