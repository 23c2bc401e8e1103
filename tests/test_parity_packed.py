"""GPU parity of the qkv-packed entry points (the guide's
flash_attn_qkvpacked_func): q, k, v interleaved per token in one
(B, S, 3, H, D) tensor, read in place. The results must equal those of the
unpacked entry points on the same values bitwise (the same kernels run with
strided addressing), and the oracle's within the usual tolerances."""

import math

import pytest
import torch

import attn_workloads as W
from oracle import attention_bwd, attention_fwd
from parity_utils import check_bwd, check_fwd

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


@pytest.mark.parametrize("B,S,H,D,dtype,causal,window,softcap,alibi", [
    (2, 300, 4, 128, "bf16", True, (-1, -1), 0.0, False),
    (1, 513, 2, 64, "fp16", False, (64, 32), 0.0, False),
    (2, 200, 4, 128, "bf16", True, (-1, -1), 10.0, True),
    (1, 300, 2, 256, "bf16", True, (-1, -1), 0.0, True),   # head dim 256
])
def test_qkvpacked_matches_unpacked_and_oracle(cuda_ok, B, S, H, D, dtype, causal, window, softcap,
                                               alibi):
    dev = torch.device("cuda")
    inp = W.make_fwd_inputs(B, S, H, H, D, dtype, seed=S + H + D, with_do=True)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    qkv = torch.stack([q, k, v], dim=2).contiguous()  # (B, S, 3, H, D)
    al = W.alibi_slopes(H, None, 0.3).to(dev) if alibi else None
    kw = dict(causal=causal, window=window, softcap=softcap, alibi_slopes=al)
    o_p, l_p = fa.fwd_qkvpacked(qkv, **kw)
    dqkv = fa.bwd_qkvpacked(qkv, o_p, l_p, do, **kw)
    o_u, l_u = fa.fwd(q, k, v, **kw)
    dq, dk, dv = fa.bwd(q, k, v, o_u, l_u, do, **kw)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    assert torch.equal(o_p, o_u) and torch.equal(l_p, l_u)
    assert torch.equal(dqkv[:, :, 0], dq) and torch.equal(dqkv[:, :, 1], dk)
    assert torch.equal(dqkv[:, :, 2], dv)
    scale = 1.0 / math.sqrt(D)
    sl = al.double().cpu().numpy() if alibi else None
    o_ref, l_ref = attention_fwd(inp["q"], inp["k"], inp["v"], scale, causal, window, softcap,
                                 alibi_slopes=sl)
    check_fwd(o_p, l_p, o_ref, l_ref, "qkvpacked fwd")
    ref = attention_bwd(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal, window, softcap,
                        alibi_slopes=sl)
    check_bwd([dqkv[:, :, i].cpu() for i in range(3)], ref, "qkvpacked bwd")


@pytest.mark.parametrize("alibi", [False, True])
def test_qkvpacked_fwd_head_dim_256(cuda_ok, alibi):
    """D = 256 (forward only): the packed forward equals the unpacked one
    bitwise and the oracle within the usual tolerances, with and without
    ALiBi slopes."""
    dev = torch.device("cuda")
    B, S, H, D = 2, 333, 2, 256
    inp = W.make_fwd_inputs(B, S, H, H, D, "bf16", seed=256 + int(alibi))
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    qkv = torch.stack([q, k, v], dim=2).contiguous()
    al = W.alibi_slopes(H, B, 0.2).to(dev) if alibi else None
    o_p, l_p = fa.fwd_qkvpacked(qkv, causal=True, alibi_slopes=al)
    o_u, l_u = fa.fwd(q, k, v, causal=True, alibi_slopes=al)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    assert torch.equal(o_p, o_u) and torch.equal(l_p, l_u)
    o_ref, l_ref = attention_fwd(inp["q"], inp["k"], inp["v"], 1.0 / math.sqrt(D), True,
                                 alibi_slopes=al.double().cpu().numpy() if alibi else None)
    check_fwd(o_p, l_p, o_ref, l_ref, f"qkvpacked fwd D256 alibi={alibi}")


def test_qkvpacked_varlen(cuda_ok):
    dev = torch.device("cuda")
    lengths = [130, 1, 400, 77]
    inp = W.make_varlen_inputs(lengths, 4, 4, 128, "bf16", seed=89, with_do=True)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    qkv = torch.stack([q, k, v], dim=1).contiguous()  # (T, 3, H, D)
    cu = inp["cu_seqlens"].to(dev)
    o, lse = fa.fwd_qkvpacked(qkv, causal=True, cu_seqlens=cu, max_seqlen=max(lengths))
    dqkv = fa.bwd_qkvpacked(qkv, o, lse, do, causal=True, cu_seqlens=cu, max_seqlen=max(lengths))
    o_u, l_u = fa.fwd(q, k, v, causal=True, cu_seqlens=cu, max_seqlen=max(lengths))
    dq, dk, dv = fa.bwd(q, k, v, o_u, l_u, do, causal=True, cu_seqlens=cu, max_seqlen=max(lengths))
    torch.cuda.synchronize()
    assert torch.equal(o, o_u) and torch.equal(lse, l_u)
    assert torch.equal(dqkv[:, 0], dq) and torch.equal(dqkv[:, 1], dk) and torch.equal(dqkv[:, 2], dv)
