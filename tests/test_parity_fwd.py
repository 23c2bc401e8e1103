"""GPU forward parity: fa_fwd (through the C ABI) vs the fp64 oracle.

Small cases span several 128-row tiles, ragged tails, S = 1, GQA/MQA,
windows, softcap and varlen packing; the full-size workloads (causal
B2 H32 S8192 D128, and varlen 65536 tokens with GQA 32/8, window (4096, 0)
and softcap 50) are checked on sampled rows the oracle computes one by one.
"""

import math

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import attention_fwd, head_fwd
from parity_utils import check_fwd, to64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")

SMALL = [
    # B, S, Hq, Hkv, D, dtype, causal, window, softcap
    (1, 128, 2, 2, 64, "bf16", False, (-1, -1), 0.0),     # the B1 H2 S128 D64 workload
    (2, 512, 16, 16, 64, "fp16", True, (-1, -1), 0.0),    # the B2 H16 S512 D64 fp16 workload
    (1, 1, 2, 1, 128, "bf16", True, (-1, -1), 0.0),       # a single token
    (2, 200, 4, 2, 128, "bf16", True, (-1, -1), 0.0),     # ragged tail, GQA
    (1, 300, 8, 1, 64, "fp16", False, (-1, -1), 0.0),     # MQA, ragged
    (1, 777, 4, 4, 128, "bf16", True, (100, 0), 0.0),     # sliding window
    (1, 640, 4, 2, 128, "bf16", False, (64, 32), 0.0),    # two-sided window
    (1, 513, 2, 2, 128, "bf16", True, (-1, -1), 50.0),    # softcap 50
    (1, 256, 8, 8, 128, "bf16", True, (-1, -1), 2.0),     # softcap that bites
    (1, 384, 2, 2, 64, "fp16", True, (0, 0), 0.0),        # each row sees itself only
    (3, 1030, 4, 1, 128, "fp16", True, (-1, -1), 0.0),    # several Q blocks, B > 1
    (1, 260, 2, 2, 128, "bf16", False, (-1, -1), 0.0),    # non-causal ragged
    # head dim 256: one 128-row Q tile per CTA
    (1, 300, 2, 2, 256, "bf16", True, (-1, -1), 0.0),     # ragged, several Q tiles
    (2, 513, 4, 2, 256, "fp16", False, (-1, -1), 0.0),    # GQA, non-causal, B > 1
    (1, 640, 2, 1, 256, "bf16", True, (100, 0), 30.0),    # window + softcap, MQA
    (1, 1, 2, 2, 256, "bf16", True, (-1, -1), 0.0),       # a single token
]


def _run_fwd(q, k, v, scale, causal, window, softcap, cu=None, max_seqlen=None):
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    cud = cu.to(dev) if cu is not None else None
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=causal, window=window, softcap=softcap,
                    cu_seqlens=cud, max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return o, lse


@pytest.mark.parametrize("B,S,Hq,Hkv,D,dtype,causal,window,softcap", SMALL)
def test_fwd_small(cuda_ok, B, S, Hq, Hkv, D, dtype, causal, window, softcap):
    inp = W.make_fwd_inputs(B, S, Hq, Hkv, D, dtype, seed=S * 7 + Hq)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run_fwd(inp["q"], inp["k"], inp["v"], scale, causal, window, softcap)
    o_ref, lse_ref = attention_fwd(inp["q"], inp["k"], inp["v"], scale, causal, window, softcap)
    check_fwd(o, lse, o_ref, lse_ref, f"B{B} S{S} H{Hq}/{Hkv} D{D} {dtype}")


@pytest.mark.parametrize("q_mult,softcap", [
    (0.25, 50.0),   # every |scale * s / softcap| below 1/8: the cubic tanh on every tile
    (1.0, 50.0),    # mostly the cubic, a few tiles on the degree-2 polynomial
    (1.0, 25.0),    # the degree-2 polynomial (|y| <= 1/4)
    (1.0, 12.0),    # the degree-4 polynomial (|y| <= 1/2)
    (1.0, 3.0),     # the exp-based tanh
])
def test_fwd_softcap_paths(cuda_ok, q_mult, softcap):
    """Each way the forward evaluates tanh for softcap (chosen per tile from
    the largest |scale * s / softcap| of a warp's rows) against the oracle;
    non-causal S = 512, so no tile is masked and every tile may take the
    cubic."""
    inp = W.make_fwd_inputs(1, 512, 4, 4, 128, "bf16", seed=int(softcap * 10 + q_mult * 3))
    q = (inp["q"].float() * q_mult).to(inp["q"].dtype)
    scale = 1.0 / math.sqrt(128)
    o, lse = _run_fwd(q, inp["k"], inp["v"], scale, False, (-1, -1), softcap)
    o_ref, lse_ref = attention_fwd(q, inp["k"], inp["v"], scale, False, (-1, -1), softcap)
    check_fwd(o, lse, o_ref, lse_ref, f"softcap {softcap} q x {q_mult}")


def test_fwd_deterministic(cuda_ok):
    inp = W.make_fwd_inputs(2, 700, 8, 2, 128, "bf16", seed=5)
    a = _run_fwd(inp["q"], inp["k"], inp["v"], 0.09, True, (-1, -1), 0.0)
    b = _run_fwd(inp["q"], inp["k"], inp["v"], 0.09, True, (-1, -1), 0.0)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("lengths,Hq,Hkv,D,causal,window,softcap", [
    ([1, 130, 257, 600, 33], 8, 2, 128, True, (200, 0), 30.0),
    ([128, 5, 384, 1], 4, 4, 64, False, (-1, -1), 0.0),
    ([513, 129], 4, 1, 128, True, (-1, -1), 0.0),
    ([200, 1, 333], 4, 2, 256, True, (-1, -1), 0.0),
    # empty sequences; at most 64 sequences number the blocks sequence by
    # sequence, more take the padded grid
    ([0, 300, 0, 1, 513, 0], 4, 2, 128, True, (-1, -1), 0.0),
    ([(5 * i) % 29 for i in range(64)], 4, 2, 64, True, (-1, -1), 0.0),
    ([(7 * i) % 37 + 1 for i in range(70)], 4, 2, 64, False, (-1, -1), 0.0),
])
def test_fwd_varlen(cuda_ok, lengths, Hq, Hkv, D, causal, window, softcap):
    inp = W.make_varlen_inputs(lengths, Hq, Hkv, D, "bf16", seed=len(lengths) * 13 + D)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run_fwd(inp["q"], inp["k"], inp["v"], scale, causal, window, softcap,
                      cu=inp["cu_seqlens"], max_seqlen=max(lengths))
    o_ref, lse_ref = attention_fwd(inp["q"], inp["k"], inp["v"], scale, causal, window, softcap,
                                   cu_seqlens=inp["cu_seqlens"].numpy())
    check_fwd(o, lse, o_ref, lse_ref, f"varlen {lengths}")


def _sample_rows(S, rng, extra=48):
    fixed = [0, 1, 127, 128, 255, 256, 257, S // 2, S - 129, S - 128, S - 2, S - 1]
    rows = set(r for r in fixed if 0 <= r < S)
    rows.update(int(x) for x in rng.integers(0, S, extra))
    return np.array(sorted(rows))


@pytest.mark.slow
def test_fwd_full_causal_8k(cuda_ok):
    """B2 H32 S8192 D128 bf16 causal, the launch configuration bench.py times;
    sampled rows of sampled heads against the oracle."""
    c = W.CONFIGS[3]
    inp = W.make_fwd_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, c.dtype, seed=1000 + c.cid)
    o, lse = _run_fwd(inp["q"], inp["k"], inp["v"], c.scale, c.causal, c.window, c.softcap)
    o, lse = o.cpu(), lse.cpu()
    rng = np.random.default_rng(3)
    for b, h in ((0, 0), (1, 31), (0, 17), (1, 5)):
        rows = _sample_rows(c.S, rng)
        o_ref, l_ref = head_fwd(inp["q"][b, :, h], inp["k"][b, :, h], inp["v"][b, :, h], c.scale,
                                c.causal, c.window[0], c.window[1], c.softcap, rows=rows)
        check_fwd(o[b, rows, h], lse[b, h, rows], o_ref, l_ref, f"cfg3 b{b} h{h}")
    assert torch.isfinite(o.float()).all()


@pytest.mark.slow
def test_fwd_full_varlen_gqa_window_softcap(cuda_ok):
    """65536 packed tokens, GQA 32/8, D128, causal window (4096, 0), softcap 50."""
    c = W.CONFIGS[4]
    inp = W.make_varlen_inputs(None, c.Hq, c.Hkv, c.D, c.dtype, seed=1000 + c.cid,
                               total=c.total, len_lo=c.len_lo, len_hi=c.len_hi)
    lens = inp["lengths"]
    cu = inp["cu_seqlens"]
    o, lse = _run_fwd(inp["q"], inp["k"], inp["v"], c.scale, c.causal, c.window, c.softcap,
                      cu=cu, max_seqlen=max(lens))
    o, lse = o.cpu(), lse.cpu()
    rng = np.random.default_rng(4)
    g = c.Hq // c.Hkv
    for s, n in enumerate(lens):
        a = int(cu[s])
        for h in (0, 13, 31):
            rows = _sample_rows(n, rng, extra=16)
            o_ref, l_ref = head_fwd(inp["q"][a:a + n, h], inp["k"][a:a + n, h // g],
                                    inp["v"][a:a + n, h // g], c.scale, c.causal, c.window[0],
                                    c.window[1], c.softcap, rows=rows)
            check_fwd(o[a + rows, h], lse[h, a + rows], o_ref, l_ref, f"cfg4 seq{s} h{h}")
