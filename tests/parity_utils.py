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


# FP8 forward: tolerance derived from where the kernel rounds.
#
# q, k, v are exact E4M3 values times their descales on both sides, and the
# tensor cores multiply them exactly with float32 accumulation, so the only
# rounding of consequence is the probabilities': the kernel forms
# P_j = 2^(x_j - m), with m a running max kept so that the largest P of a row
# lies in [2^4, 2^8], rounds every P_j to E4M3 for the P.V product, and
# divides by the float32 sum l of the unrounded P. Hence
#     O = sum_j w_j (1 + d_j) V_j,   error e = sum_j w_j d_j V_j,
# with w the exact probabilities and d_j the relative rounding error of P_j.
# Round to nearest with 3 mantissa bits leaves an error uniform over at most
# one spacing, and the spacing of E4M3 values at P is at most 2^-3 P (at most
# 2^-9 absolute below 2^-6, the subnormals, which is at most 2^-13 of the
# row's largest probability since that P is >= 2^4). Taking the d_j as
# independent and zero-mean,
#     sigma^2 = sum_j s_j^2 V_j^2 / 12,  s_j = max(2^-3 w_j, 2^-13 max_j w_j).
# A row of n keys can reach at most sqrt(3 n) sigma (Cauchy-Schwarz on the
# uniform errors), so 6 sigma is a hard bound up to n = 12 and a 6-sigma
# Gaussian tail beyond. Add the 16-bit output rounding (half an ulp, 2^-9
# relative for bf16) and 1e-4 relative for the float32 row sum (the exp2
# approximations err by at most 7.5e-5 relative). In aggregate, the rms of
# e / sigma must not exceed 1 (sigma uses the largest possible spacing).
# LSE is formed from the unrounded P, so its bound is the 16-bit one.
FP8_SIGMAS = 6.0


def fp8_sigma(w, v):
    """Noise scale of the FP8 forward's output per element: w [rows, Sk] the
    exact probabilities of one head, v [Sk, D] its (dequantized) values."""
    w = np.asarray(w, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    wmax = np.max(w, axis=1, keepdims=True)
    s = np.maximum(w * 2.0 ** -3, wmax * 2.0 ** -13)
    return np.sqrt((s * s) @ (v * v) / 12.0)


def check_fwd_fp8(o_gpu, lse_gpu, o_ref, lse_ref, sigma, what="", out_bits=7):
    """Compare an FP8 forward with the exact attention over the dequantized
    inputs: |e| <= 6 sigma + 2^-(bits+1) |O| + 1e-4 |O| elementwise, the
    rms over elements of (|e| beyond the rounding terms) / sigma <= 1, and the
    LSE bound of the 16-bit forward."""
    o = to64(o_gpu) if hasattr(o_gpu, "detach") else np.asarray(o_gpu, dtype=np.float64)
    lse = to64(lse_gpu) if hasattr(lse_gpu, "detach") else np.asarray(lse_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    sigma = np.asarray(sigma, dtype=np.float64)
    assert o.shape == o_ref.shape == sigma.shape, (what, o.shape, o_ref.shape, sigma.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - o_ref)
    bound = FP8_SIGMAS * sigma + (2.0 ** -(out_bits + 1) + 1e-4) * np.abs(o_ref) + 1e-6
    worst = np.argmax(err - bound)
    assert np.all(err <= bound), (
        f"{what}: error {err.flat[worst]:.3e} > bound {bound.flat[worst]:.3e} "
        f"(sigma {sigma.flat[worst]:.3e}, |O| {abs(o_ref.flat[worst]):.3e})")
    pos = sigma > 0
    if pos.any():
        # the part of the error beyond the output rounding, in sigmas
        noise = np.maximum(err - (2.0 ** -(out_bits + 1) + 1e-4) * np.abs(o_ref), 0.0)
        ratio = float(np.sqrt(np.mean((noise[pos] / sigma[pos]) ** 2)))
        assert ratio <= 1.0, f"{what}: rms(e / sigma) = {ratio:.3f} > 1"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin), f"{what}: LSE finiteness differs"
    if fin.any():
        lerr = np.abs(lse[fin] - lse_ref[fin])
        assert lerr.max() <= LSE_ABS, f"{what}: LSE max-abs {lerr.max():.3e}"
    return float(err.max()), (ratio if pos.any() else 0.0)
