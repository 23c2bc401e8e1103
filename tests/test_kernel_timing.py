"""Per-kernel timing through the C ABI: while enabled, every call records
CUDA events around each kernel it launches on the caller's stream."""

import pytest
import torch

import attn_workloads as W

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def test_timing_counts_each_launch(cuda_ok):
    dev = torch.device("cuda")
    inp = W.make_fwd_inputs(1, 512, 4, 2, 128, "bf16", seed=3, with_do=True)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    fa.fa_kernel_timing_reset()
    fa.fa_kernel_timing_enable(True)
    try:
        for _ in range(3):
            o, lse = fa.fwd(q, k, v, causal=True)
        fa.bwd(q, k, v, o, lse, do, causal=True)
        torch.cuda.synchronize()
    finally:
        fa.fa_kernel_timing_enable(False)
    ms, n = fa.fa_kernel_timing_read("fwd")
    assert n == 3 and ms > 0.0
    for name in ("bwd_pre", "bwd_dkdv", "bwd_dq"):
        ms, n = fa.fa_kernel_timing_read(name)
        assert n == 1 and ms > 0.0, name
    assert fa.fa_kernel_timing_read("decode_split") == (0.0, 0)
    fa.fa_kernel_timing_reset()
    assert fa.fa_kernel_timing_read("fwd") == (0.0, 0)
    # disabled: nothing is recorded
    fa.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_kernel_timing_read("fwd") == (0.0, 0)
