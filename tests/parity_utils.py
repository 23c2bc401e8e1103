"""Shared helpers of the GPU parity tests: tolerances and comparisons.

Tolerances for N(0, 1) inputs: forward max-abs(O) <= 1e-2, mean-abs(O) <=
1e-3, |dLSE| <= 1e-3; backward relative Frobenius error <= 1e-2 for each of
dQ, dK, dV (max-abs <= 1e-3 where the exact gradient is identically zero).
Outputs are 16-bit, so their own rounding (half an ulp: 2^-9
relative for bf16) is part of the error budget.
"""

import numpy as np
import torch

FWD_MAX_ABS = 1e-2
FWD_MEAN_ABS = 1e-3
LSE_ABS = 1e-3
BWD_REL_FRO = 1e-2
ZERO_GRAD_ABS = 1e-3


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_fwd(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o = to64(o_gpu) if hasattr(o_gpu, "detach") else np.asarray(o_gpu, dtype=np.float64)
    lse = to64(lse_gpu) if hasattr(lse_gpu, "detach") else np.asarray(lse_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert o.shape == o_ref.shape, (what, o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - o_ref)
    assert err.max() <= FWD_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= FWD_MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin), f"{what}: LSE finiteness differs"
    if fin.any():
        lerr = np.abs(lse[fin] - lse_ref[fin])
        assert lerr.max() <= LSE_ABS, f"{what}: LSE max-abs {lerr.max():.3e}"
    return float(err.max()), float(err.mean())


def rel_fro(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-30))


def check_bwd(grads_gpu, grads_ref, what=""):
    out = []
    for name, g, r in zip(("dq", "dk", "dv"), grads_gpu, grads_ref):
        g64 = to64(g) if hasattr(g, "detach") else np.asarray(g, dtype=np.float64)
        assert np.all(np.isfinite(g64)), f"{what}: non-finite {name}"
        r = np.asarray(r, dtype=np.float64)
        if np.linalg.norm(r) < 1e-8:
            # degenerate case: the exact gradient is zero (e.g. every row sees a
            # single key, so the softmax has no slope); a relative error is
            # undefined, so bound the absolute error instead
            e = float(np.abs(g64).max())
            assert e <= ZERO_GRAD_ABS, f"{what}: {name} should be 0, max-abs {e:.3e}"
        else:
            e = rel_fro(g64, r)
            assert e <= BWD_REL_FRO, f"{what}: {name} rel-Frobenius {e:.3e}"
        out.append(e)
    return out


# Quantised KV caches (int8 / int4): the forward bounds, with the mean-abs
# bound widened by the output's own rounding. An output row mixes
# dequantized rows (code * scale), which are not 16-bit values, so even a
# one-key row is rounded once on output; that rounding averages a quarter of
# an output ulp.
MANTISSA_BITS = {"bf16": 7, "fp16": 10}


def check_fwd_quant(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what):
    o, lse = to64(o_gpu), to64(lse_gpu)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert o.shape == o_ref.shape and np.all(np.isfinite(o)), what
    err = np.abs(o - o_ref)
    assert err.max() <= FWD_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    mag = np.abs(o_ref)
    ulp = np.where(mag > 0, np.exp2(np.floor(np.log2(np.where(mag > 0, mag, 1.0))) - MANTISSA_BITS[dtype]), 0.0)
    bound = FWD_MEAN_ABS + float(np.mean(ulp)) / 4
    assert err.mean() <= bound, f"{what}: mean-abs {err.mean():.3e} > {bound:.3e}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin), f"{what}: LSE finiteness differs"
    if fin.any():
        lerr = np.abs(lse[fin] - lse_ref[fin])
        assert lerr.max() <= LSE_ABS, f"{what}: LSE max-abs {lerr.max():.3e}"
