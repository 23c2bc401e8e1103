"""Seeded synthetic workloads for the attention library and its oracle.

This module only draws random inputs and lays them out (shapes, lengths,
page tables, paged pools). It holds none of the attention arithmetic, so both
the oracle-side tests and the CUDA-side tests/bench can use it.

Recipes (the pages benchmark fp16/bf16, head dim 64/128, sequence lengths
512..16k, "FlashAttention 实战指南" §实测数据; these seeded draws stand in for
that benchmark since it ships no dataset):

* every value tensor is ``randn`` in fp32 rounded to the 16-bit dtype
  (round-to-nearest-even), i.e. N(0, 1);
* generator ``torch.Generator('cpu').manual_seed(1000 + config_id)``;
  structure (lengths, cache lengths, page permutation) is drawn first, then
  q, k, v, then dO or (k_new, v_new);
* decode cache contents are drawn per sequence from a generator seeded with
  ``(1000 + config_id) * 1_000_003 + b`` so that any one sequence can be
  regenerated on its own (the pool is several GB).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "CONFIGS",
    "FwdConfig",
    "VarlenConfig",
    "DecodeConfig",
    "make_fwd_inputs",
    "make_varlen_lengths",
    "make_varlen_inputs",
    "make_decode_structure",
    "decode_sequence_cache",
    "fill_paged_pool",
    "rotary_tables",
    "alibi_slopes",
    "visible_pairs",
    "fwd_flops",
    "bwd_flops",
    "varlen_visible_pairs",
    "decode_kv_bytes",
    "to_e4m3",
    "make_fp8_inputs",
    "make_fp8_varlen_inputs",
]

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


@dataclass(frozen=True)
class FwdConfig:
    cid: int
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    dtype: str
    causal: bool
    scale: float
    window: tuple = (-1, -1)
    softcap: float = 0.0
    backward: bool = False
    name: str = ""


@dataclass(frozen=True)
class VarlenConfig:
    cid: int
    total: int
    len_lo: int
    len_hi: int
    Hq: int
    Hkv: int
    D: int
    dtype: str
    causal: bool
    scale: float
    window: tuple = (-1, -1)
    softcap: float = 0.0
    name: str = ""


@dataclass(frozen=True)
class DecodeConfig:
    cid: int
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: str
    len_lo: int
    len_hi: int
    page_size: int
    scale: float
    causal: bool = True
    window: tuple = (-1, -1)
    softcap: float = 0.0
    splits: tuple = (1, 4, 16)
    name: str = ""


CONFIGS = {
    1: FwdConfig(1, B=1, Hq=2, Hkv=2, S=128, D=64, dtype="bf16", causal=False,
                 scale=1.0 / 8.0, name="fwd non-causal B1 H2 S128 D64 bf16"),
    2: FwdConfig(2, B=2, Hq=16, Hkv=16, S=512, D=64, dtype="fp16", causal=True,
                 scale=1.0 / 8.0, name="fwd causal B2 H16 S512 D64 fp16"),
    3: FwdConfig(3, B=2, Hq=32, Hkv=32, S=8192, D=128, dtype="bf16", causal=True,
                 scale=1.0 / math.sqrt(128.0), backward=True,
                 name="fwd+bwd causal B2 H32 S8192 D128 bf16"),
    4: VarlenConfig(4, total=65536, len_lo=512, len_hi=16384, Hq=32, Hkv=8, D=128,
                    dtype="bf16", causal=True, scale=1.0 / math.sqrt(128.0),
                    window=(4096, 0), softcap=50.0,
                    name="fwd varlen 65536 tok GQA 32/8 D128 window(4096,0) softcap50 bf16"),
    5: DecodeConfig(5, B=64, Hq=32, Hkv=8, D=128, dtype="bf16", len_lo=1024, len_hi=32768,
                    page_size=256, scale=1.0 / math.sqrt(128.0),
                    name="decode paged B64 GQA 32/8 D128 L1024..32768 page256 bf16"),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator("cpu")
    g.manual_seed(seed)
    return g


def _randn(g: torch.Generator, shape, dtype: str) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(DTYPES[dtype])


def make_fwd_inputs(B, S, Hq, Hkv, D, dtype="bf16", seed=0, with_do=False):
    """q (B,S,Hq,D), k, v (B,S,Hkv,D) [, dO (B,S,Hq,D)] as CPU 16-bit tensors."""
    g = _gen(seed)
    q = _randn(g, (B, S, Hq, D), dtype)
    k = _randn(g, (B, S, Hkv, D), dtype)
    v = _randn(g, (B, S, Hkv, D), dtype)
    out = {"q": q, "k": k, "v": v}
    if with_do:
        out["do"] = _randn(g, (B, S, Hq, D), dtype)
    return out


def to_e4m3(x: torch.Tensor):
    """Per-tensor FP8 E4M3 encoding as a caller would prepare the FP8
    forward's inputs: descale = max|x| / 448 (rounded to float32, the type the
    library takes it in), codes = x / descale clamped to the finite range
    and cast to torch.float8_e4m3fn (round to nearest even). Returns (codes
    as a uint8 tensor of bit patterns, descale as a Python float)."""
    amax = float(x.detach().abs().max().to(torch.float64))
    descale = float(np.float32(amax / 448.0)) if amax > 0 else 1.0
    y = (x.detach().to(torch.float64) / descale).clamp(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), descale


def make_fp8_inputs(B, S, Hq, Hkv, D, seed=0):
    """FP8 forward inputs: q, k, v drawn as make_fwd_inputs draws them (fp32
    N(0, 1), same generator order) and encoded per tensor by to_e4m3.
    Returns {"q", "k", "v"} uint8 code tensors and {"q_descale", ...}."""
    raw = make_fwd_inputs(B, S, Hq, Hkv, D, "fp32", seed)
    out = {}
    for n in ("q", "k", "v"):
        out[n], out[n + "_descale"] = to_e4m3(raw[n])
    return out


def make_fp8_varlen_inputs(Hq, Hkv, D, seed=0, total=None, len_lo=None, len_hi=None,
                           lengths=None):
    """make_varlen_inputs in fp32, then every tensor encoded by to_e4m3."""
    raw = make_varlen_inputs(lengths, Hq, Hkv, D, "fp32", seed, total, len_lo, len_hi)
    out = {"lengths": raw["lengths"], "cu_seqlens": raw["cu_seqlens"]}
    for n in ("q", "k", "v"):
        out[n], out[n + "_descale"] = to_e4m3(raw[n])
    return out


def make_varlen_lengths(total, lo, hi, g: torch.Generator):
    """Lengths drawn uniformly from the integers [lo, hi] until their sum
    reaches ``total``; the last one is cut to the remainder (so it may be
    shorter than ``lo``)."""
    lens = []
    acc = 0
    while acc < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=g).item())
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    return lens


def make_varlen_inputs(lengths=None, Hq=32, Hkv=8, D=128, dtype="bf16", seed=0, total=None,
                       len_lo=None, len_hi=None, with_do=False):
    """Packed q (T,Hq,D), k, v (T,Hkv,D) and cu_seqlens (int32, B+1).
    Either give ``lengths`` or (total, len_lo, len_hi) to draw them."""
    g = _gen(seed)
    if lengths is None:
        lengths = make_varlen_lengths(total, len_lo, len_hi, g)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    t = cu[-1]
    out = {
        "lengths": list(lengths),
        "cu_seqlens": torch.tensor(cu, dtype=torch.int32),
        "q": _randn(g, (t, Hq, D), dtype),
        "k": _randn(g, (t, Hkv, D), dtype),
        "v": _randn(g, (t, Hkv, D), dtype),
    }
    if with_do:
        out["do"] = _randn(g, (t, Hq, D), dtype)
    return out


def make_decode_structure(B, Hq, Hkv, D, len_lo, len_hi, page_size, dtype="bf16", seed=0,
                          cache_seqlens=None, pages_per_seq=None, sq=1):
    """Structure and per-step inputs of one decode step with sq new tokens.

    Returns dict with cache_seqlens (int32, B), block_table (int32,
    B x pages_per_seq: a random permutation of all physical pages), q
    (B,sq,Hq,D), k_new, v_new (B,sq,Hkv,D), num_pages, page_size, seed.
    ``pages_per_seq`` defaults to ceil((len_hi + sq) / page_size) so the
    appended tokens always have a page.
    """
    g = _gen(seed)
    if cache_seqlens is None:
        cache_seqlens = torch.randint(len_lo, len_hi + 1, (B,), generator=g, dtype=torch.int64)
    cache_seqlens = torch.as_tensor(cache_seqlens, dtype=torch.int64)
    if pages_per_seq is None:
        pages_per_seq = -(-(int(len_hi) + sq) // page_size)
    num_pages = B * pages_per_seq
    perm = torch.randperm(num_pages, generator=g)
    block_table = perm.view(B, pages_per_seq).to(torch.int32)
    q = _randn(g, (B, sq, Hq, D), dtype)
    k_new = _randn(g, (B, sq, Hkv, D), dtype)
    v_new = _randn(g, (B, sq, Hkv, D), dtype)
    return {
        "cache_seqlens": cache_seqlens.to(torch.int32),
        "block_table": block_table,
        "q": q,
        "k_new": k_new,
        "v_new": v_new,
        "num_pages": num_pages,
        "page_size": page_size,
        "pages_per_seq": pages_per_seq,
        "Hkv": Hkv,
        "D": D,
        "dtype": dtype,
        "seed": seed,
    }


def decode_sequence_cache(st, b):
    """Logical (contiguous) cache contents of sequence b: k, v of shape
    (cache_seqlens[b], Hkv, D), drawn from that sequence's own generator."""
    n = int(st["cache_seqlens"][b])
    g = _gen(st["seed"] * 1_000_003 + b)
    k = _randn(g, (n, st["Hkv"], st["D"]), st["dtype"])
    v = _randn(g, (n, st["Hkv"], st["D"]), st["dtype"])
    return k, v


def fill_paged_pool(st, k_pool, v_pool, batches=None):
    """Scatter each sequence's logical cache into the paged pools
    (num_pages, page_size, Hkv, D) through block_table: logical position p of
    sequence b lives in page block_table[b, p // page_size], slot
    p % page_size. Pools may live on any device; untouched slots keep their
    contents."""
    ps = st["page_size"]
    bt = st["block_table"]
    for b in range(bt.shape[0]) if batches is None else batches:
        k, v = decode_sequence_cache(st, b)
        n = k.shape[0]
        kd = k.to(k_pool.device)
        vd = v.to(v_pool.device)
        for p in range(0, n, ps):
            page = int(bt[b, p // ps])
            m = min(ps, n - p)
            k_pool[page, :m].copy_(kd[p:p + m])
            v_pool[page, :m].copy_(vd[p:p + m])


def rotary_tables(rows, rotary_dim, base=10000.0):
    """Angle tables a caller passes for the rotary encoding: float32 cos and
    sin of shape (rows, rotary_dim / 2) with angle(p, i) = p * base^(-2i /
    rotary_dim), the common frequency ladder (evaluated in float64)."""
    inv = base ** (-np.arange(0, rotary_dim, 2, dtype=np.float64) / rotary_dim)
    ang = np.arange(rows, dtype=np.float64)[:, None] * inv[None, :]
    return (torch.from_numpy(np.cos(ang).astype(np.float32)),
            torch.from_numpy(np.sin(ang).astype(np.float32)))


def alibi_slopes(H, B=None, scale=1.0):
    """ALiBi slopes a caller passes: the geometric sequence 2^(-8 (h+1) / H)
    for H heads (times `scale`), float32 (H,); with B, a (B, H) array whose
    row b is scaled by (b + 1), so that every sequence has its own slopes."""
    base = scale * 2.0 ** (-8.0 * (np.arange(H, dtype=np.float64) + 1.0) / H)
    if B is None:
        return torch.from_numpy(base.astype(np.float32))
    rows = np.stack([base * (b + 1) for b in range(B)])
    return torch.from_numpy(rows.astype(np.float32))


# ---------------------------------------------------------------------------
# work accounting (visible pairs, FLOPs, bytes); no attention arithmetic
# ---------------------------------------------------------------------------
def visible_pairs(sq, sk, causal, window_left=-1, window_right=-1):
    """Number of (query, key) pairs that the causal / window mask lets
    through, with bottom-right alignment and inclusive bounds."""
    delta = sk - sq
    right = 0 if causal else window_right
    total = 0
    # closed form per row, summed in O(sq)
    for i in range(sq):
        hi = sk - 1
        if right >= 0:
            hi = min(hi, i + delta + right)
        lo = 0
        if window_left >= 0:
            lo = max(lo, i + delta - window_left)
        if hi >= lo:
            total += hi - lo + 1
    return total


def fwd_flops(pairs, D, Hq):
    """Forward FLOPs counted as 4*D per visible pair and query head
    (two matmuls, QK^T and PV, each 2*D per pair)."""
    return 4 * D * pairs * Hq


def bwd_flops(pairs, D, Hq):
    """Backward FLOPs counted as 10*D per visible pair and query head
    (five matmuls: QK^T recompute, dP, dV, dK, dQ)."""
    return 10 * D * pairs * Hq


def varlen_visible_pairs(lengths, causal, window_left=-1, window_right=-1):
    return sum(visible_pairs(n, n, causal, window_left, window_right) for n in lengths)


def decode_kv_bytes(cache_seqlens, Hkv, D, elem_bytes=2):
    """Algorithmic K+V bytes read by one decode step: every visible key and
    value row of every kv head, once (L_b + 1 keys per sequence)."""
    n = int(torch.as_tensor(cache_seqlens, dtype=torch.int64).sum().item()) + len(cache_seqlens)
    return 2 * n * Hkv * D * elem_bytes


def decode_kv_bytes_int4(cache_seqlens, Hkv, D):
    """The same for an int4 cache: per row D / 2 code bytes and a 4-byte
    float32 scale."""
    n = int(torch.as_tensor(cache_seqlens, dtype=torch.int64).sum().item()) + len(cache_seqlens)
    return 2 * n * Hkv * (D // 2 + 4)


def decode_kv_bytes_int8(cache_seqlens, Hkv, D):
    """The same for an int8 cache: per row D one-byte codes and a 4-byte
    float32 scale."""
    n = int(torch.as_tensor(cache_seqlens, dtype=torch.int64).sum().item()) + len(cache_seqlens)
    return 2 * n * Hkv * (D + 4)
