"""GPU parity with ALiBi slopes (the guide's alibi_slopes option): forward,
backward and the kv-cache step through the C ABI against the fp64 oracle,
which adds -slope * |i + Sk - Sq - j| to each scaled, softcapped logit."""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import attention_bwd, attention_fwd, kvcache_decode
from parity_utils import check_bwd, check_fwd

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")

CASES = [
    # B, S, Hq, Hkv, D, dtype, causal, window, softcap, per-batch slopes, slope scale
    (2, 300, 4, 2, 128, "bf16", True, (-1, -1), 0.0, False, 1.0),
    (1, 513, 8, 8, 64, "fp16", False, (-1, -1), 0.0, False, 0.05),    # gentle decay, both sides
    (2, 257, 4, 1, 128, "bf16", True, (100, 0), 20.0, True, 0.2),     # window + softcap, (B, Hq)
    (1, 640, 2, 2, 128, "bf16", False, (64, 32), 0.0, False, 0.5),
]


def _slopes(Hq, B, per_batch, scale):
    return W.alibi_slopes(Hq, B if per_batch else None, scale)


@pytest.mark.parametrize("B,S,Hq,Hkv,D,dtype,causal,window,softcap,per_batch,sc", CASES)
def test_alibi_fwd_bwd(cuda_ok, B, S, Hq, Hkv, D, dtype, causal, window, softcap, per_batch, sc):
    dev = torch.device("cuda")
    inp = W.make_fwd_inputs(B, S, Hq, Hkv, D, dtype, seed=S + 5 * Hq, with_do=True)
    slopes = _slopes(Hq, B, per_batch, sc)
    scale = 1.0 / math.sqrt(D)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    al = slopes.to(dev)
    o, lse = fa.fwd(q, k, v, scale=scale, causal=causal, window=window, softcap=softcap,
                    alibi_slopes=al)
    grads = fa.bwd(q, k, v, o, lse, do, scale=scale, causal=causal, window=window,
                   softcap=softcap, alibi_slopes=al)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    sl = slopes.double().numpy()
    o_ref, lse_ref = attention_fwd(inp["q"], inp["k"], inp["v"], scale, causal, window, softcap,
                                   alibi_slopes=sl)
    check_fwd(o, lse, o_ref, lse_ref, f"alibi fwd B{B} S{S}")
    ref = attention_bwd(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal, window, softcap,
                        alibi_slopes=sl)
    check_bwd([g.cpu() for g in grads], ref, f"alibi bwd B{B} S{S}")


def test_alibi_varlen(cuda_ok):
    dev = torch.device("cuda")
    lengths = [130, 1, 400, 77]
    inp = W.make_varlen_inputs(lengths, 4, 2, 128, "bf16", seed=61, with_do=True)
    slopes = W.alibi_slopes(4, len(lengths), 0.3)
    cu = inp["cu_seqlens"].to(dev)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, causal=True, cu_seqlens=cu, max_seqlen=max(lengths),
                    alibi_slopes=slopes.to(dev))
    grads = fa.bwd(q, k, v, o, lse, do, causal=True, cu_seqlens=cu, max_seqlen=max(lengths),
                   alibi_slopes=slopes.to(dev))
    torch.cuda.synchronize()
    scale = 1.0 / math.sqrt(128)
    cun = inp["cu_seqlens"].numpy()
    o_ref, lse_ref = attention_fwd(inp["q"], inp["k"], inp["v"], scale, True, cu_seqlens=cun,
                                   alibi_slopes=slopes.double().numpy())
    check_fwd(o, lse, o_ref, lse_ref, "alibi varlen fwd")
    ref = attention_bwd(inp["q"], inp["k"], inp["v"], inp["do"], scale, True, cu_seqlens=cun,
                        alibi_slopes=slopes.double().numpy())
    check_bwd([g.cpu() for g in grads], ref, "alibi varlen bwd")


@pytest.mark.parametrize("Sq,Hq,Hkv,splits,per_batch", [(1, 8, 2, 1, False), (1, 32, 8, 4, True),
                                                         (3, 8, 2, 3, False), (5, 16, 4, 2, True)])
def test_alibi_kvcache(cuda_ok, Sq, Hq, Hkv, splits, per_batch):
    """Each query head of a GQA group has its own slope, and each new token
    its own position."""
    dev = torch.device("cuda")
    lengths = [0, 200, 1000]
    B, D = len(lengths), 128
    st = W.make_decode_structure(B, Hq, Hkv, D, 0, max(lengths), 64, "bf16", seed=67 + Sq,
                                 cache_seqlens=lengths, sq=Sq)
    shape = (st["num_pages"], 64, Hkv, D)
    kc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    W.fill_paged_pool(st, kc, vc)
    slopes = W.alibi_slopes(Hq, B if per_batch else None, 0.5)
    out, lse = fa.fwd_kvcache(st["q"].to(dev), kc, vc, st["cache_seqlens"].to(dev),
                              st["block_table"].to(dev), k_new=st["k_new"].to(dev),
                              v_new=st["v_new"].to(dev), num_splits=splits,
                              alibi_slopes=slopes.to(dev))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    logical = [W.decode_sequence_cache(st, b) for b in range(B)]
    o_ref, l_ref, _, _ = kvcache_decode(st["q"], st["k_new"], st["v_new"], [c[0] for c in logical],
                                        [c[1] for c in logical], lengths, 1.0 / math.sqrt(D), True,
                                        alibi_slopes=slopes.double().numpy())
    check_fwd(out, lse, o_ref, l_ref, f"alibi decode Sq={Sq} splits={splits}")
