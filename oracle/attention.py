"""Plain fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The CUDA library never calls it, and this module imports nothing from
the CUDA library or its Python binding.

Sources (web pages; cited by title and section):

* "FlashAttention 实战指南:如何把训练内存省 20 倍、速度提 4 倍" (kwkr.cn)
  - §长序列注意力为什么会爆内存: attention is three steps, QK^T, softmax, then
    multiply by V; the tiled method is exact, i.e. it equals this plain
    definition up to floating-point rounding. So the oracle is the plain
    definition, with the full score matrix materialised and masked explicitly.
  - §上手…三步走: tensors are (batch, seqlen, nheads, headdim); causal=True for
    autoregressive use; a varlen family handles unequal lengths in a batch.
  - §进阶参数: window_size=(left, right), (-1, -1) meaning unbounded; softcap
    bounds the logits to [-softcap, softcap]; K/V may have fewer heads than Q
    as long as Hq is an integer multiple of Hkv (MQA/GQA).
  - §增量解码场景 flash_attn_with_kvcache: the new K, V are appended to the
    existing cache and attention is then done in place; cache_seqlens marks
    each sample's valid length; block_table pages the cache; num_splits
    splits the KV range.
* "AI模型推理优化 Flash Attention原理" (52runoob.com)
  - §先搞清楚原理: the standard attention function, scores = Q K^T / sqrt(d),
    softmax over the last dim, then times V.
  - §实际怎么用: the KVCache class, whose update writes the new k, v at the
    current position and returns the prefix up to the new position.

Readings where the pages leave a step open (each one is listed in the design
notes of the repository):

* softcap is the tanh form ``c * tanh(x / c)``, applied after ``scale`` and
  before masking; ``softcap == 0`` disables it. It keeps every logit inside
  (-c, c), which is what the guide's sentence asks for.
* window bounds are inclusive; causal means ``window_right = 0``.
* when Sq != Sk the diagonal is aligned bottom-right: query i may see key j iff
  ``i + (Sk - Sq) - L <= j <= i + (Sk - Sq) + R``.
* a row with no visible key gets O = 0 and LSE = -inf (and zero gradients).
* LSE is the natural-log log-sum-exp of the (scaled, softcapped) logits.
* GQA maps query head h to kv head ``h // (Hq // Hkv)``.
* ``cache_seqlens[b]`` is the length *before* the append; the new token lands
  at position ``cache_seqlens[b]`` and attention covers ``cache_seqlens[b]+1``
  keys.
* "FlashAttention技术深度解析：重塑LLM推理性能的新范式" §发展趋势 /
  量化技术融合 mentions an INT8/INT4 quantised KV cache but gives no format.
  The int8 cache here is symmetric with one float32 scale per (token, kv
  head) row: ``scale = max|x| / 127`` and ``code = round-half-even(x /
  scale)``, both in float32 (the precision the kernel takes the integer
  decision in), an all-zero row having scale 0 and codes 0. A cached row
  stands for ``code * scale``; a new key is rotated (with rotary) and rounded
  to the 16-bit input type first, as the 16-bit cache stores it, then
  quantised. The int4 reading is the same with ``scale = max|x| / 7`` and
  codes in [-7, 7], stored two per byte (the code of even d in the low
  nibble, both biased by 8).
* The guide (§版本怎么选) says FlashAttention-3 runs an FP8 forward and gives
  no format. The reading here is the common one: Q, K and V are FP8 E4M3
  tensors (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0
  is subnormal, the all-ones pattern is NaN, no infinities; largest finite
  value 448) with one float32 descale per tensor, so an element stands for
  ``value(code) * descale``. The FP8 forward is then exact attention over
  those values; its output is 16-bit. How close a kernel that feeds the
  probabilities to the tensor cores in E4M3 comes to it is a tolerance,
  derived in the tests (not emulated here).

Every array is float64. 16-bit inputs are converted exactly (every bf16 and
fp16 value is representable in float64), so the oracle sees the same values
the GPU sees.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "visible_mask",
    "scores",
    "head_fwd",
    "head_bwd",
    "attention_fwd",
    "attention_bwd",
    "kvcache_decode",
    "kvcache_decode_int8",
    "kvcache_decode_int4",
    "decode_e4m3",
    "attention_fwd_fp8",
    "head_probs",
    "quantize_int8",
    "dequantize_int8",
    "quantize_int4",
    "pack_int4",
    "unpack_int4",
    "lse_combine",
    "rotary",
    "round_to",
]


def _f64(x) -> np.ndarray:
    """Exact upcast of a numpy array or a CPU torch tensor to float64."""
    if hasattr(x, "detach"):  # torch tensor (bf16 has no numpy dtype)
        import torch

        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def visible_mask(sq: int, sk: int, causal: bool, window_left: int, window_right: int,
                 rows: np.ndarray | None = None) -> np.ndarray:
    """Boolean [len(rows), sk] matrix: True where query i may attend key j.

    Guide §进阶参数: window (left, right) with -1 meaning unbounded; causal is
    the window with right = 0. Alignment is bottom-right (delta = sk - sq).
    """
    if rows is None:
        rows = np.arange(sq)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(sk, dtype=np.int64)[None, :]
    delta = sk - sq
    right = 0 if causal else window_right
    ok = np.ones((i.shape[0], sk), dtype=bool)
    if right >= 0:
        ok &= j <= i + delta + right
    if window_left >= 0:
        ok &= j >= i + delta - window_left
    return ok


def scores(q_h: np.ndarray, k_h: np.ndarray, scale: float, softcap: float):
    """Logits of one head: returns (X, Y) with Y = scale * q k^T and
    X = softcap * tanh(Y / softcap) (X = Y when softcap == 0).

    Notes §先搞清楚原理 (scores = Q K^T * scale); guide §进阶参数 (softcap).
    """
    y = scale * (_f64(q_h) @ _f64(k_h).T)
    if softcap > 0.0:
        x = softcap * np.tanh(y / softcap)
    else:
        x = y
    return x, y


def alibi_bias(sq: int, sk: int, slope: float, rows=None) -> np.ndarray:
    """ALiBi bias of one head, [len(rows), sk]: -slope * |i + (sk - sq) - j|,
    the distance between query i and key j under the bottom-right alignment
    of visible_mask. Guide §进阶参数: alibi_slopes is a position bias that
    makes attention to distant keys decay, with no explicit position
    encoding; the linear-in-distance form is the reading."""
    if rows is None:
        rows = np.arange(sq)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(sk, dtype=np.int64)[None, :]
    return -float(slope) * np.abs(i + (sk - sq) - j).astype(np.float64)


def _slope(alibi_slopes, b: int, h: int) -> float:
    """Slope of (batch b, head h) from a (Hq,) or (B, Hq) array, 0 if None."""
    if alibi_slopes is None:
        return 0.0
    a = np.asarray(alibi_slopes, dtype=np.float64)
    return float(a[h] if a.ndim == 1 else a[b, h])


def head_fwd(q_h, k_h, v_h, scale: float, causal: bool = False, window_left: int = -1,
             window_right: int = -1, softcap: float = 0.0, rows=None, _score_hook=None,
             alibi_slope: float = 0.0):
    """One head of the forward pass.

    q_h: [Sq, D]; k_h, v_h: [Sk, D]. ``rows`` optionally selects query rows
    (indices into 0..Sq-1) so that sampled rows of a long sequence can be
    checked without the whole matrix. Returns (O [rows, D], LSE [rows]).

    Steps, in the order of the notes' standard attention: logits, mask,
    softmax along the keys, weighted sum of V. The softmax is evaluated as
    exp(X - m) / sum(exp(X - m)) with m the row max, which is the same value.
    """
    q_h = _f64(q_h)
    k_h = _f64(k_h)
    v_h = _f64(v_h)
    sq, sk = q_h.shape[0], k_h.shape[0]
    if rows is None:
        rows = np.arange(sq)
    rows = np.asarray(rows, dtype=np.int64)
    x, _ = scores(q_h[rows], k_h, scale, softcap)
    if alibi_slope != 0.0:
        x = x + alibi_bias(sq, sk, alibi_slope, rows)
    if _score_hook is not None:
        x = _score_hook(x)
    vis = visible_mask(sq, sk, causal, window_left, window_right, rows)
    x = np.where(vis, x, -np.inf)
    m = np.max(x, axis=1, initial=-np.inf)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    p = np.exp(x - m_safe[:, None])  # exp(-inf) = 0 on masked entries
    l = p.sum(axis=1)
    o = np.zeros((rows.shape[0], v_h.shape[1]))
    o[has] = (p[has] / l[has, None]) @ v_h
    lse = np.full(rows.shape[0], -np.inf)
    lse[has] = m[has] + np.log(l[has])
    return o, lse


def head_bwd(q_h, k_h, v_h, do_h, scale: float, causal: bool = False, window_left: int = -1,
             window_right: int = -1, softcap: float = 0.0, alibi_slope: float = 0.0):
    """One head of the backward pass of ``head_fwd`` (all rows).

    With P the row-normalised softmax probabilities (zero where masked):
      dV = P^T dO,  dP = dO V^T,  Drow = rowsum(P * dP),  dX = P * (dP - Drow)
    and through softcap X = c tanh(Y / c): dY = dX * (1 - tanh(Y / c)^2),
      dQ = scale * dY K,  dK = scale * dY^T Q.
    This is the chain rule of the definition; the guide (§长序列…) says the
    tiled backward recomputes these quantities rather than storing P. The
    ALiBi bias is a constant added to X, so it changes P and nothing else.
    """
    q_h = _f64(q_h)
    k_h = _f64(k_h)
    v_h = _f64(v_h)
    do_h = _f64(do_h)
    sq, sk = q_h.shape[0], k_h.shape[0]
    x, y = scores(q_h, k_h, scale, softcap)
    if alibi_slope != 0.0:
        x = x + alibi_bias(sq, sk, alibi_slope)
    vis = visible_mask(sq, sk, causal, window_left, window_right)
    x = np.where(vis, x, -np.inf)
    m = np.max(x, axis=1, initial=-np.inf)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    p = np.exp(x - m_safe[:, None])
    l = p.sum(axis=1)
    l_safe = np.where(has, l, 1.0)
    p = p / l_safe[:, None]
    dv = p.T @ do_h
    dp = do_h @ v_h.T
    drow = np.sum(p * dp, axis=1)
    dx = p * (dp - drow[:, None])
    if softcap > 0.0:
        t = np.tanh(y / softcap)
        dy = dx * (1.0 - t * t)
    else:
        dy = dx
    dq = scale * (dy @ k_h)
    dk = scale * (dy.T @ q_h)
    return dq, dk, dv


def _segments(q, cu_seqlens):
    """Yield (b, q-token slice) for fixed-length (B,S,...) or varlen inputs."""
    if cu_seqlens is None:
        for b in range(q.shape[0]):
            yield b, (b,)
    else:
        cu = [int(c) for c in np.asarray(cu_seqlens).tolist()]
        for b in range(len(cu) - 1):
            yield b, (slice(cu[b], cu[b + 1]),)


def attention_fwd(q, k, v, scale: float, causal: bool = False, window=(-1, -1),
                  softcap: float = 0.0, cu_seqlens=None, alibi_slopes=None):
    """Full forward over all batches and heads.

    Fixed length: q (B, S, Hq, D), k/v (B, S, Hkv, D) -> O (B, S, Hq, D),
    LSE (B, Hq, S). Varlen (cu_seqlens given, int prefix sums of length B+1):
    q (total, Hq, D), k/v (total, Hkv, D) -> O (total, Hq, D), LSE (Hq, total);
    each segment is an independent sequence with Sq = Sk = its length (guide
    §上手…三步走, varlen family). alibi_slopes: None, (Hq,) or (B, Hq).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    hq, hkv = q.shape[-2], k.shape[-2]
    assert hq % hkv == 0, "Hq must be an integer multiple of Hkv"
    g = hq // hkv
    o = np.zeros(q.shape)
    if cu_seqlens is None:
        lse = np.zeros((q.shape[0], hq, q.shape[1]))
    else:
        lse = np.zeros((hq, q.shape[0]))
    for b, sl in _segments(q, cu_seqlens):
        qb, kb, vb = q[sl], k[sl], v[sl]
        for h in range(hq):
            ob, lb = head_fwd(qb[:, h], kb[:, h // g], vb[:, h // g], scale, causal,
                              window[0], window[1], softcap,
                              alibi_slope=_slope(alibi_slopes, b, h))
            if cu_seqlens is None:
                o[b, :, h] = ob
                lse[b, h] = lb
            else:
                o[sl[0], h] = ob
                lse[h, sl[0]] = lb
    return o, lse


def attention_bwd(q, k, v, do, scale: float, causal: bool = False, window=(-1, -1),
                  softcap: float = 0.0, cu_seqlens=None, alibi_slopes=None):
    """Gradients (dQ, dK, dV) of sum(O * dO); same layouts as attention_fwd.
    For GQA the per-query-head dK/dV contributions of a group are summed into
    their shared kv head."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    hq, hkv = q.shape[-2], k.shape[-2]
    g = hq // hkv
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b, sl in _segments(q, cu_seqlens):
        for h in range(hq):
            a, bb, c = head_bwd(q[sl][:, h], k[sl][:, h // g], v[sl][:, h // g], do[sl][:, h],
                                scale, causal, window[0], window[1], softcap,
                                alibi_slope=_slope(alibi_slopes, b, h))
            if cu_seqlens is None:
                dq[b, :, h] = a
                dk[b, :, h // g] += bb
                dv[b, :, h // g] += c
            else:
                dq[sl[0], h] = a
                dk[sl[0], h // g] += bb
                dv[sl[0], h // g] += c
    return dq, dk, dv


def round_to(x, dtype):
    """Round float64 values to a 16-bit type (round to nearest even) and back.
    "bf16": through float32 bits; "fp16": numpy float16; None: unchanged."""
    x = np.asarray(x, dtype=np.float64)
    if dtype is None:
        return x
    if dtype == "fp16":
        with np.errstate(over="ignore"):  # beyond the fp16 range -> +-inf, as a cast gives
            return x.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        b = x.astype(np.float32).view(np.uint32).astype(np.uint64)
        b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
        return b.astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def rotary(x, pos, cos, sin, interleaved=False):
    """Rotary position embedding of the last dimension of x (..., T, H, D) at
    integer positions pos (T,): with r = rotary dim (2 * cos.shape[1]) and
    angle tables cos, sin of shape (positions, r/2), each pair (a, b) of the
    first r dimensions becomes (a cos - b sin, a sin + b cos). Pairs are
    (i, i + r/2) by default, (2i, 2i + 1) when interleaved; dimensions from r
    on are unchanged. (Guide §增量解码场景: rotary_cos / rotary_sin apply the
    rotary position encoding inside the call; the pairing is a reading.)"""
    x = _f64(x).copy()
    cos = _f64(cos)
    sin = _f64(sin)
    half = cos.shape[1]
    pos = np.asarray(pos)
    if pos.size and (pos.min() < 0 or pos.max() >= cos.shape[0]):
        raise ValueError("rotary position outside the angle table")
    c = cos[np.asarray(pos)][:, None, :]  # (T, 1, r/2)
    sn = sin[np.asarray(pos)][:, None, :]
    if interleaved:
        a = x[..., 0:2 * half:2].copy()
        b = x[..., 1:2 * half:2].copy()
        x[..., 0:2 * half:2] = a * c - b * sn
        x[..., 1:2 * half:2] = a * sn + b * c
    else:
        a = x[..., :half].copy()
        b = x[..., half:2 * half].copy()
        x[..., :half] = a * c - b * sn
        x[..., half:2 * half] = a * sn + b * c
    return x


def kvcache_decode(q, k_new, v_new, k_cache_logical, v_cache_logical, cache_seqlens,
                   scale: float, causal: bool = True, window=(-1, -1), softcap: float = 0.0,
                   heads=None, rotary_cos=None, rotary_sin=None, rotary_interleaved=False,
                   rotated_dtype=None, alibi_slopes=None):
    """One step against a *logical, contiguous* per-sequence cache.

    q (B, Sq, Hq, D); k_new, v_new (B, Sq, Hkv, D) or None; k/v_cache_logical:
    sequence of B arrays, each holding at least cache_seqlens[b] rows of shape
    (rows, Hkv, D). Following the notes' KVCache.update, the Sq new keys and
    values are written at positions L_b .. L_b + Sq - 1 (L_b =
    cache_seqlens[b]) and the prefix of length Lk = L_b + Sq is used (without
    an append, Lk = L_b). Query token t sits at position Lk - Sq + t and
    attends over the Lk keys with bottom-right alignment (causal: keys up to
    its own position). With rotary tables, q and the new keys are rotated at
    those positions before the append (guide §增量解码场景); `rotated_dtype`
    rounds the rotated values to the 16-bit type the cache and the matmul
    operands hold. The paged layout and block_table are not used here.

    ``heads`` optionally restricts the query heads evaluated (others left 0).
    Returns (O (B, Sq, Hq, D), LSE (B, Hq, Sq), appended_k list, appended_v list).
    """
    q = _f64(q)
    bsz, sq, hq, d = q.shape
    append = k_new is not None
    if append:
        k_new = _f64(k_new)
        v_new = _f64(v_new)
        hkv = k_new.shape[2]
    else:
        hkv = _f64(k_cache_logical[0]).shape[1]
    g = hq // hkv
    o = np.zeros((bsz, sq, hq, d))
    lse = np.zeros((bsz, hq, sq))
    ks, vs = [], []
    for b in range(bsz):
        n = int(cache_seqlens[b])
        lk = n + (sq if append else 0)
        pos = np.arange(lk - sq, lk)
        qb = q[b]
        kn = k_new[b] if append else None
        if rotary_cos is not None:
            qb = round_to(rotary(qb, pos, rotary_cos, rotary_sin, rotary_interleaved), rotated_dtype)
            if append:
                kn = round_to(rotary(kn, pos, rotary_cos, rotary_sin, rotary_interleaved),
                              rotated_dtype)
        kc = _f64(k_cache_logical[b])[:n]
        vc = _f64(v_cache_logical[b])[:n]
        kb = np.concatenate([kc, kn], axis=0) if append else kc
        vb = np.concatenate([vc, v_new[b]], axis=0) if append else vc
        ks.append(kb)
        vs.append(vb)
        for h in (range(hq) if heads is None else heads):
            ob, lb = head_fwd(qb[:, h], kb[:, h // g], vb[:, h // g], scale, causal,
                              window[0], window[1], softcap,
                              alibi_slope=_slope(alibi_slopes, b, h))
            o[b, :, h] = ob
            lse[b, h, :] = lb
    return o, lse, ks, vs


def quantize_int8(x):
    """Symmetric int8 quantisation of each row (the last axis) of ``x``.

    In float32, as the reading in the module header states: ``scale = max|x| /
    127`` and ``code = round-half-even(x / scale)`` (IEEE division, numpy's
    ``rint``); a row of zeros gets scale 0 and codes 0. Returns (codes int8 of
    x's shape, scales float32 of x's shape without the last axis).
    """
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    div = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    codes = np.rint((x32 / div[..., None]).astype(np.float32))
    codes = np.where(scale[..., None] > 0, codes, np.float32(0.0))
    return np.clip(codes, -127, 127).astype(np.int8), scale


def quantize_int4(x):
    """Symmetric int4 quantisation of each row (the last axis) of ``x``: as
    quantize_int8 with 7 in place of 127, codes in [-7, 7] (an int8 array,
    one code per element; pack_int4 stores them two per byte). Returns
    (codes, scales float32)."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale = (amax / np.float32(7.0)).astype(np.float32)
    div = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    codes = np.rint((x32 / div[..., None]).astype(np.float32))
    codes = np.where(scale[..., None] > 0, codes, np.float32(0.0))
    return np.clip(codes, -7, 7).astype(np.int8), scale


def pack_int4(codes):
    """int4 codes (..., D), D even -> bytes (..., D / 2): byte i holds code
    2i + 8 in its low nibble and code 2i + 1 + 8 in its high nibble."""
    c = np.asarray(codes, dtype=np.int16) + 8
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed):
    """The inverse of pack_int4."""
    b = np.asarray(packed, dtype=np.int16)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int8)
    out[..., 0::2] = (b & 15) - 8
    out[..., 1::2] = (b >> 4) - 8
    return out


def dequantize_int8(codes, scales):
    """The values an int8 cache stands for: ``code * scale`` per row (float64)."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[..., None]


def kvcache_decode_int8(q, k_new, v_new, k_codes_logical, k_scales_logical, v_codes_logical,
                        v_scales_logical, cache_seqlens, scale: float, causal: bool = True,
                        window=(-1, -1), softcap: float = 0.0, heads=None, rotary_cos=None,
                        rotary_sin=None, rotary_interleaved=False, rotated_dtype=None,
                        alibi_slopes=None):
    """kvcache_decode against an int8 cache (the quantised-cache reading above).

    k/v_codes_logical: B arrays of at least cache_seqlens[b] rows (rows, Hkv, D)
    of int8 codes; k/v_scales_logical: B arrays (rows, Hkv) of float32 scales.
    The Sq new rows are quantised (keys after rotation and rounding to
    ``rotated_dtype``) and appended; then every cached row is replaced by the
    value it stands for and the step is kvcache_decode's, with the appended
    rows already in the cache. Returns (O, LSE, appended k codes, k scales,
    v codes, v scales), the last four as lists of the B sequences' new rows.
    """
    return _kvcache_decode_quant(quantize_int8, q, k_new, v_new, k_codes_logical,
                                 k_scales_logical, v_codes_logical, v_scales_logical,
                                 cache_seqlens, scale, causal, window, softcap, heads, rotary_cos,
                                 rotary_sin, rotary_interleaved, rotated_dtype, alibi_slopes)


def kvcache_decode_int4(q, k_new, v_new, k_codes_logical, k_scales_logical, v_codes_logical,
                        v_scales_logical, cache_seqlens, scale: float, causal: bool = True,
                        window=(-1, -1), softcap: float = 0.0, heads=None, rotary_cos=None,
                        rotary_sin=None, rotary_interleaved=False, rotated_dtype=None,
                        alibi_slopes=None):
    """kvcache_decode_int8 with the int4 reading: codes in [-7, 7] (one per
    element, unpacked; pack_int4 gives the stored bytes), appended rows
    quantised by quantize_int4."""
    return _kvcache_decode_quant(quantize_int4, q, k_new, v_new, k_codes_logical,
                                 k_scales_logical, v_codes_logical, v_scales_logical,
                                 cache_seqlens, scale, causal, window, softcap, heads, rotary_cos,
                                 rotary_sin, rotary_interleaved, rotated_dtype, alibi_slopes)


def _kvcache_decode_quant(quantize, q, k_new, v_new, k_codes_logical, k_scales_logical,
                          v_codes_logical, v_scales_logical, cache_seqlens, scale, causal,
                          window, softcap, heads, rotary_cos, rotary_sin, rotary_interleaved,
                          rotated_dtype, alibi_slopes):
    """The quantised-cache step shared by the int8 and int4 readings."""
    bsz, sq = tuple(q.shape)[:2]
    append = k_new is not None
    kd, vd, kc_new, ks_new, vc_new, vs_new = [], [], [], [], [], []
    lengths = []
    for b in range(bsz):
        n = int(cache_seqlens[b])
        kc = np.asarray(k_codes_logical[b])[:n]
        ksc = np.asarray(k_scales_logical[b])[:n]
        vc = np.asarray(v_codes_logical[b])[:n]
        vsc = np.asarray(v_scales_logical[b])[:n]
        if append:
            kn = _f64(k_new[b])
            if rotary_cos is not None:
                pos = np.arange(n, n + sq)
                kn = round_to(rotary(kn, pos, rotary_cos, rotary_sin, rotary_interleaved),
                              rotated_dtype)
            a_kc, a_ks = quantize(kn)
            a_vc, a_vs = quantize(_f64(v_new[b]))
            kc_new.append(a_kc)
            ks_new.append(a_ks)
            vc_new.append(a_vc)
            vs_new.append(a_vs)
            kc, ksc = np.concatenate([kc, a_kc]), np.concatenate([ksc, a_ks])
            vc, vsc = np.concatenate([vc, a_vc]), np.concatenate([vsc, a_vs])
        kd.append(dequantize_int8(kc, ksc))
        vd.append(dequantize_int8(vc, vsc))
        lengths.append(kc.shape[0])
    o, lse, _, _ = kvcache_decode(q, None, None, kd, vd, np.asarray(lengths), scale, causal,
                                  window, softcap, heads, rotary_cos, rotary_sin,
                                  rotary_interleaved, rotated_dtype, alibi_slopes)
    return o, lse, kc_new, ks_new, vc_new, vs_new


def lse_combine(o_parts, lse_parts):
    """Merge attention results computed over disjoint key ranges.

    o_parts: [n, ..., D] each normalised over its own range; lse_parts [n, ...].
    LSE = log(sum_s exp(LSE_s)); O = sum_s exp(LSE_s - LSE) * O_s. This is the
    identity that lets num_splits (guide §增量解码场景) split the KV range.
    Parts with LSE_s = -inf (no visible key) carry zero weight.
    """
    o_parts = _f64(o_parts)
    lse_parts = _f64(lse_parts)
    m = np.max(lse_parts, axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - m_safe[None])
    s = w.sum(axis=0)
    has = s > 0
    lse = np.where(has, m_safe + np.log(np.where(has, s, 1.0)), -np.inf)
    wn = np.where(has[None], w / np.where(has, s, 1.0)[None], 0.0)
    o = np.sum(wn[..., None] * o_parts, axis=0)
    return o, lse


def decode_e4m3(codes) -> np.ndarray:
    """Float64 values of FP8 E4M3 bit patterns (uint8 codes), from the
    format's definition: bit 7 is the sign, bits 6..3 the exponent e (bias 7),
    bits 2..0 the mantissa m. e = 0 gives the subnormal m * 2^-9; otherwise
    (1 + m / 8) * 2^(e - 7); e = 15 with m = 7 is NaN (the format has no
    infinities, and e = 15 with m < 7 are ordinary values up to 448)."""
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where((c & 0x80) != 0, -mag, mag)


def attention_fwd_fp8(q_codes, k_codes, v_codes, q_descale: float, k_descale: float,
                      v_descale: float, scale: float, causal: bool = False, window=(-1, -1),
                      softcap: float = 0.0, cu_seqlens=None, alibi_slopes=None):
    """The FP8 forward (reading in the module header): every E4M3 code times
    its tensor's descale is the element it stands for, and the result is
    attention_fwd over those values, in the layouts of attention_fwd."""
    q = decode_e4m3(q_codes) * float(q_descale)
    k = decode_e4m3(k_codes) * float(k_descale)
    v = decode_e4m3(v_codes) * float(v_descale)
    return attention_fwd(q, k, v, scale, causal, window, softcap, cu_seqlens, alibi_slopes)


def head_probs(q_h, k_h, scale: float, causal: bool = False, window_left: int = -1,
               window_right: int = -1, softcap: float = 0.0, rows=None,
               alibi_slope: float = 0.0) -> np.ndarray:
    """The attention probabilities of one head, [len(rows), Sk]: the softmax
    step of the definition (logits, mask, row-normalised exponentials), zero
    where masked and on rows with no visible key. O = head_probs @ V."""
    q_h = _f64(q_h)
    k_h = _f64(k_h)
    sq, sk = q_h.shape[0], k_h.shape[0]
    if rows is None:
        rows = np.arange(sq)
    rows = np.asarray(rows, dtype=np.int64)
    x, _ = scores(q_h[rows], k_h, scale, softcap)
    if alibi_slope != 0.0:
        x = x + alibi_bias(sq, sk, alibi_slope, rows)
    x = np.where(visible_mask(sq, sk, causal, window_left, window_right, rows), x, -np.inf)
    m = np.max(x, axis=1, initial=-np.inf)
    has = np.isfinite(m)
    p = np.exp(x - np.where(has, m, 0.0)[:, None])
    l = p.sum(axis=1)
    return np.where(has[:, None], p / np.where(has, l, 1.0)[:, None], 0.0)
