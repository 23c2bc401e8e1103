"""GPU backward parity: fa_bwd (through the C ABI) vs the fp64 oracle's
analytic gradients. The oracle recomputes everything from q, k, v and dO;
the GPU backward consumes the GPU forward's out and lse, as a caller would.
Bar: relative Frobenius error <= 1e-2 on each of dQ, dK, dV."""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import attention_bwd, head_bwd
from parity_utils import check_bwd, rel_fro, to64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def _gpu_fwd_bwd(inp, scale, causal, window, softcap, cu=None, max_seqlen=None):
    dev = torch.device("cuda")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    cud = cu.to(dev) if cu is not None else None
    o, lse = fa.fwd(q, k, v, scale=scale, causal=causal, window=window, softcap=softcap,
                    cu_seqlens=cud, max_seqlen=max_seqlen)
    dq, dk, dv = fa.bwd(q, k, v, o, lse, do, scale=scale, causal=causal, window=window,
                        softcap=softcap, cu_seqlens=cud, max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    st = fa.fa_get_device_status()
    assert st == 0, fa.fa_last_error()
    return dq.cpu(), dk.cpu(), dv.cpu()


SMALL = [
    # B, S, Hq, Hkv, D, dtype, causal, window, softcap
    (1, 128, 2, 2, 64, "bf16", False, (-1, -1), 0.0),
    (2, 200, 4, 2, 128, "bf16", True, (-1, -1), 0.0),     # ragged, GQA
    (1, 300, 8, 1, 64, "fp16", False, (-1, -1), 0.0),     # MQA
    (1, 777, 4, 4, 128, "bf16", True, (100, 0), 0.0),     # window
    (1, 640, 4, 2, 128, "bf16", False, (64, 32), 0.0),    # two-sided window
    (1, 513, 2, 2, 128, "bf16", True, (-1, -1), 50.0),    # softcap 50
    (1, 256, 4, 4, 128, "bf16", True, (-1, -1), 2.0),     # softcap that bites
    (2, 512, 16, 16, 64, "fp16", True, (-1, -1), 0.0),    # B2 H16 S512 D64 fp16
    (1, 1, 2, 1, 128, "bf16", True, (-1, -1), 0.0),       # a single token
    (1, 1030, 4, 1, 128, "fp16", True, (-1, -1), 0.0),    # many Q tiles per key tile
    # the pre pass takes 512 / Hq whole tokens a block: 85 tokens at Hq = 6
    # (blocks of 85, 85, 85, 45), one token at Hq = 520 (GQA group 65)
    (1, 300, 6, 2, 64, "bf16", True, (-1, -1), 0.0),
    (1, 40, 520, 8, 64, "bf16", False, (-1, -1), 0.0),
    # head dim 256: a dV pass and a dK pass of 32-row items, dQ with dO in
    # shared memory and 32-key blocks
    (1, 300, 2, 2, 256, "bf16", True, (-1, -1), 0.0),     # causal, ragged
    (2, 513, 4, 2, 256, "fp16", False, (-1, -1), 0.0),    # GQA, non-causal, B > 1
    (1, 640, 2, 1, 256, "bf16", True, (100, 0), 30.0),    # window + softcap, MQA
    (1, 256, 4, 4, 256, "bf16", True, (-1, -1), 2.0),     # softcap that bites
    (1, 1, 2, 2, 256, "bf16", True, (-1, -1), 0.0),       # a single token
    (1, 700, 2, 2, 256, "fp16", False, (64, 32), 0.0),    # two-sided window
]


@pytest.mark.parametrize("B,S,Hq,Hkv,D,dtype,causal,window,softcap", SMALL)
def test_bwd_small(cuda_ok, B, S, Hq, Hkv, D, dtype, causal, window, softcap):
    inp = W.make_fwd_inputs(B, S, Hq, Hkv, D, dtype, seed=S * 3 + Hq, with_do=True)
    scale = 1.0 / math.sqrt(D)
    got = _gpu_fwd_bwd(inp, scale, causal, window, softcap)
    ref = attention_bwd(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal, window, softcap)
    check_bwd(got, ref, f"B{B} S{S} H{Hq}/{Hkv} D{D} {dtype} w{window} c{softcap}")


@pytest.mark.parametrize("lengths,Hq,Hkv,D,causal,window,softcap", [
    ([1, 130, 257, 600, 33], 8, 2, 128, True, (200, 0), 30.0),
    ([128, 5, 384, 1], 4, 4, 64, False, (-1, -1), 0.0),
    ([200, 1, 333, 97], 4, 2, 256, True, (-1, -1), 0.0),
    ([1, 130, 257, 600, 33], 4, 1, 256, True, (200, 0), 30.0),
])
def test_bwd_varlen(cuda_ok, lengths, Hq, Hkv, D, causal, window, softcap):
    inp = W.make_varlen_inputs(lengths, Hq, Hkv, D, "bf16", seed=len(lengths) * 31 + D, with_do=True)
    scale = 1.0 / math.sqrt(D)
    got = _gpu_fwd_bwd(inp, scale, causal, window, softcap, cu=inp["cu_seqlens"],
                       max_seqlen=max(lengths))
    ref = attention_bwd(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal, window, softcap,
                        cu_seqlens=inp["cu_seqlens"].numpy())
    check_bwd(got, ref, f"varlen {lengths}")


def test_bwd_d256_is_deterministic(cuda_ok):
    inp = W.make_fwd_inputs(1, 400, 4, 2, 256, "bf16", seed=19, with_do=True)
    a = _gpu_fwd_bwd(inp, 0.06, True, (-1, -1), 0.0)
    b = _gpu_fwd_bwd(inp, 0.06, True, (-1, -1), 0.0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_is_deterministic(cuda_ok):
    """dK and dV come from one CTA per key tile and dQ from one CTA per query
    tile, with no atomics: repeated runs are bitwise identical (a race would
    show up here)."""
    inp = W.make_fwd_inputs(1, 600, 4, 2, 128, "bf16", seed=9, with_do=True)
    a = _gpu_fwd_bwd(inp, 0.088, True, (-1, -1), 0.0)
    b = _gpu_fwd_bwd(inp, 0.088, True, (-1, -1), 0.0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.slow
def test_bwd_full_causal_8k(cuda_ok):
    """B2 H32 S8192 D128 bf16 causal: gradients of two whole heads against the
    oracle (each head is a full 8192 x 8192 problem in fp64)."""
    c = W.CONFIGS[3]
    inp = W.make_fwd_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, c.dtype, seed=1000 + c.cid, with_do=True)
    dq, dk, dv = _gpu_fwd_bwd(inp, c.scale, c.causal, c.window, c.softcap)
    for b, h in ((0, 3), (1, 30)):
        ref = head_bwd(inp["q"][b, :, h], inp["k"][b, :, h], inp["v"][b, :, h], inp["do"][b, :, h],
                       c.scale, c.causal, c.window[0], c.window[1], c.softcap)
        check_bwd((dq[b, :, h], dk[b, :, h], dv[b, :, h]), ref, f"cfg3 b{b} h{h}")
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
