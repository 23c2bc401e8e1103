"""The FMA-pipe approximations of the forward kernels, evaluated on the GPU
(fa_selftest_poly) over dense sweeps of their domains and compared with
CUDA's exp2f / tanhf on the same inputs and with numpy's float64 functions.

The coefficients come from the Remez fits in csrc/fit_polynomials.py. Each
bound is the fit's float64 relative error (printed by that script), plus
the rounding of the coefficients to float32, plus the float32 evaluation (a
few roundings of the Horner steps, bounded here by 3 ulp of the result):
relative 7.49e-5 + 3 * 2^-23 for the cubic 2^x, and for tanh
7.3e-8 |tanh| + 3 ulp (degree 4, |y| <= 0.5) and 4.6e-7 |tanh| + 3 ulp
(degree 2, |y| <= 0.25). Against CUDA's functions the bound adds their own
documented error (2 ulp).
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_149_b200")


def run(which, x):
    dev = torch.device("cuda")
    xd = torch.from_numpy(x).to(dev)
    po = torch.empty_like(xd)
    ro = torch.empty_like(xd)
    fa.fa_selftest_poly(which, xd, po, ro, x.size)
    torch.cuda.synchronize()
    return po.cpu().numpy().astype(np.float64), ro.cpu().numpy().astype(np.float64)


def ulp(y):
    y = np.abs(y).astype(np.float32)
    return (np.nextafter(y, np.float32(np.inf)) - y).astype(np.float64)


# float64 relative error of each fit, plus the rounding of its coefficients
# to float32 (at most one float32 spacing, 6e-8 relative, on the leading one)
EX2_FIT = 7.48e-5 + 6e-8
TANH_FIT = {1: 1.32e-8 + 6e-8, 2: 3.96e-7 + 6e-8}


def test_ex2_poly(cuda_ok):
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    poly, ref = run(0, x)
    exact = np.exp2(x.astype(np.float64))
    bound = EX2_FIT + 3 * 2.0 ** -23
    rel = np.abs(poly - exact) / exact
    assert rel.max() <= bound, rel.max()
    rel_cuda = np.abs(poly - ref) / ref
    assert rel_cuda.max() <= bound + 2 * 2.0 ** -23, rel_cuda.max()
    # integers map to exact powers of two up to the fit's error at f = 0
    xi = np.arange(-125, 9, dtype=np.float32)
    pi, _ = run(0, xi)
    assert np.all(np.abs(pi / np.exp2(xi.astype(np.float64)) - 1) <= bound)


@pytest.mark.parametrize("which,ymax", [(1, 0.5), (2, 0.25)])
def test_tanh_poly(cuda_ok, which, ymax):
    half = np.linspace(0.0, ymax, 1_000_001).astype(np.float32)
    x = np.concatenate([-half[::-1], half[1:]])  # exactly symmetric about 0
    poly, ref = run(which, x)
    exact = np.tanh(x.astype(np.float64))
    bound = TANH_FIT[which] * np.abs(exact) + 3 * ulp(exact)
    err = np.abs(poly - exact)
    assert np.all(err <= bound), float((err - bound).max())
    err_cuda = np.abs(poly - ref)
    assert np.all(err_cuda <= bound + 2 * ulp(ref)), err_cuda.max()
    # odd symmetry is exact (every step is odd or even in y)
    np.testing.assert_array_equal(poly, -poly[::-1])
