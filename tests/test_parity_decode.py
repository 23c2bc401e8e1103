"""GPU decode parity: fa_fwd_kvcache (paged, split-KV, in-place append) vs the
oracle, which attends over a logical contiguous cache and never reads the
page table. The page pool after the call must equal the pool before it with
exactly the appended slots changed (bitwise)."""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import head_fwd, kvcache_decode
from parity_utils import check_fwd, to64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def _run_case(st, splits, causal=True, window=(-1, -1), softcap=0.0, append=True, scale=None,
              heads=None, check_pool=True):
    dev = torch.device("cuda")
    D = st["D"]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    Hkv = st["Hkv"]
    dt = W.DTYPES[st["dtype"]]
    shape = (st["num_pages"], st["page_size"], Hkv, D)
    # unused slots hold a recognisable non-zero pattern so stray reads show up
    kc = torch.full(shape, 3.0, dtype=dt, device=dev)
    vc = torch.full(shape, -5.0, dtype=dt, device=dev)
    W.fill_paged_pool(st, kc, vc)
    k_before = kc.clone() if check_pool else None
    v_before = vc.clone() if check_pool else None
    q = st["q"].to(dev)
    kn = st["k_new"].to(dev) if append else None
    vn = st["v_new"].to(dev) if append else None
    out, lse = fa.fwd_kvcache(q, kc, vc, st["cache_seqlens"].to(dev), st["block_table"].to(dev),
                              k_new=kn, v_new=vn, scale=scale, causal=causal, window=window,
                              softcap=softcap, num_splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    B = st["q"].shape[0]
    Hq = st["q"].shape[2]
    g = Hq // Hkv
    logical = [W.decode_sequence_cache(st, b) for b in range(B)]
    if append:
        o_ref, l_ref, ks, vs = kvcache_decode(st["q"], st["k_new"], st["v_new"],
                                              [c[0] for c in logical], [c[1] for c in logical],
                                              st["cache_seqlens"].tolist(), scale, causal, window,
                                              softcap, heads=heads)
    else:
        o_ref = np.zeros((B, 1, Hq, D))
        l_ref = np.zeros((B, Hq, 1))
        for b in range(B):
            for h in (range(Hq) if heads is None else heads):
                o1, l1 = head_fwd(st["q"][b, :, h], logical[b][0][:, h // g], logical[b][1][:, h // g],
                                  scale, causal, window[0], window[1], softcap)
                o_ref[b, 0, h] = o1[0]
                l_ref[b, h, 0] = l1[0]
    hs = list(range(Hq)) if heads is None else list(heads)
    check_fwd(out[:, :, hs], lse[:, hs], o_ref[:, :, hs], l_ref[:, hs],
              f"decode splits={splits}")
    if check_pool:
        ps = st["page_size"]
        changed_k = (kc != k_before).any(dim=(2, 3))
        changed_v = (vc != v_before).any(dim=(2, 3))
        expect = torch.zeros_like(changed_k)
        if append:
            for b in range(B):
                L = int(st["cache_seqlens"][b])
                page = int(st["block_table"][b, L // ps])
                expect[page, L % ps] = True
                assert torch.equal(kc[page, L % ps].cpu(), st["k_new"][b, 0])
                assert torch.equal(vc[page, L % ps].cpu(), st["v_new"][b, 0])
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
