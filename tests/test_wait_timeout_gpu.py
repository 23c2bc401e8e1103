"""The bounded waits in their safe failure form: a test build of the forward
kernel never issues one K tile load, its waits run out after 10 ms, and the
kernel returns FA_ERR_TIMEOUT through the device status word instead of
hanging or faulting. Nothing is left in flight (the withheld copy is never
issued; every issued copy and tensor-core operation is waited for), so the
context stays usable: a normal call right after it is correct."""

import math

import pytest
import torch

import attn_workloads as W
from oracle import attention_fwd
from parity_utils import check_fwd

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def _normal(inp, dev):
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o, lse = fa.fwd(q, k, v, scale=1 / math.sqrt(128))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    o_ref, l_ref = attention_fwd(inp["q"], inp["k"], inp["v"], 1 / math.sqrt(128))
    check_fwd(o, lse, o_ref, l_ref, "normal call")


def test_withheld_load_times_out_and_the_context_survives(cuda_ok):
    dev = torch.device("cuda")
    inp = W.make_fwd_inputs(1, 256, 1, 1, 128, "bf16", seed=71)
    _normal(inp, dev)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    lse = torch.empty((1, 1, 256), dtype=torch.float32, device=dev)
    fa.fa_selftest_fwd_timeout(q, k, v, out, lse, 1, 1, 256, 1 / math.sqrt(128), 10_000_000, 0)
    torch.cuda.synchronize()  # the call returns: no hang, no fault
    assert fa.fa_get_device_status() == fa.FA_ERR_TIMEOUT
    assert fa.fa_get_device_status() == 0  # reading clears the word
    _normal(inp, dev)
