"""The allocation-free decode entry point, fa_fwd_kvcache_noalloc.

It serves callers that cannot allocate device memory on their decode path
(a server that gave all free memory to its KV-cache pool up front, a host
runtime that owns the allocator, a latency-bound loop that must not call
cudaMalloc/cudaFree). Instead of a caller workspace it keeps the split
partials in the library's static device array. This file checks, through
the C ABI, that two calls in a row give what fa_fwd_kvcache gives with a
workspace, within the forward tolerances. The second call uses another
shape and split count, so stale partials left by the first call would show.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""

import ctypes
import math

import pytest
import torch

import attn_workloads as W
from parity_utils import check_fwd

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def _decode_both_ways(B, Hq, Hkv, D, lengths, page_size, splits, seed, sq=1, rotary_dim=0):
    dev = torch.device("cuda")
    st = W.make_decode_structure(B, Hq, Hkv, D, 0, max(lengths), page_size, "bf16", seed=seed,
                                 cache_seqlens=lengths, sq=sq)
    shape = (st["num_pages"], page_size, Hkv, D)
    kc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    W.fill_paged_pool(st, kc, vc)
    kc2, vc2 = kc.clone(), vc.clone()
    q = st["q"].to(dev)
    kn, vn = st["k_new"].to(dev), st["v_new"].to(dev)
    cs, bt = st["cache_seqlens"].to(dev), st["block_table"].to(dev)
    rows = st["pages_per_seq"] * page_size
    cos = sin = None
    if rotary_dim:
        cos, sin = (t.to(dev) for t in W.rotary_tables(rows, rotary_dim))
    scale = 1.0 / math.sqrt(D)
    # reference: the workspace entry point
    ws = torch.empty(fa.fa_kvcache_workspace_size(B, sq, Hq, D, splits, rotary_dim),
                     dtype=torch.uint8, device=dev)
    out_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, Hq, sq), dtype=torch.float32, device=dev)
    fa.fa_fwd_kvcache(q, kn, vn, kc, vc, bt, cs, cos, sin, out_ref, lse_ref, B, sq, Hq, Hkv, D,
                      page_size, bt.shape[1], st["num_pages"], rows, rotary_dim, False, scale,
                      True, -1, -1, 0.0, None, 0, splits, 0, ws, ws.numel())
    # the allocation-free entry point, called straight through the C ABI
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, sq), float("nan"), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    status = fa.lib.fa_fwd_kvcache_noalloc(
        q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc2.data_ptr(), vc2.data_ptr(), bt.data_ptr(),
        cs.data_ptr(), ptr(cos), ptr(sin), out.data_ptr(), lse.data_ptr(), B, sq, Hq, Hkv, D,
        page_size, bt.shape[1], st["num_pages"], rows if rotary_dim else 0, rotary_dim, 0,
        ctypes.c_float(scale), 1, -1, -1, ctypes.c_float(0.0), None, 0, splits, 0,
        ctypes.c_void_p(stream))
    assert status == 0, fa.fa_last_error()
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    check_fwd(out, lse, out_ref.cpu().double().numpy(), lse_ref.cpu().double().numpy(),
              f"noalloc vs workspace, splits={splits}")
    assert torch.equal(kc2, kc) and torch.equal(vc2, vc)  # same in-place append


def test_noalloc_matches_workspace_entry_point_twice(cuda_ok):
    _decode_both_ways(4, 32, 8, 128, [1500, 64, 777, 3000], 256, 4, seed=101)
    # the second call also keeps rotated queries of 3 new tokens in the scratch
    _decode_both_ways(3, 8, 2, 128, [200, 1000, 5], 64, 7, seed=202, sq=3, rotary_dim=128)


def test_noalloc_rejects_oversized_partials(cuda_ok):
    # B=64, Hq=64, D=128, 32 splits need 64*64*129*4*32 bytes > 24 MiB
    need = fa.fa_kvcache_workspace_size(64, 1, 64, 128, 32)
    assert need > fa.FA_NOALLOC_SCRATCH_BYTES
    status = fa.lib.fa_fwd_kvcache_noalloc(16, 16, 16, 16, 16, 16, 16, None, None, 16, 16, 64, 1,
                                           64, 8, 128, 256, 4, 8, 0, 0, 0, ctypes.c_float(0.1), 1,
                                           -1, -1, ctypes.c_float(0.0), None, 0, 32, 0, None)
    assert status == 1 and "scratch" in fa.fa_last_error()
