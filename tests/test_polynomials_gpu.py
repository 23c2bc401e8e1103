"""The FMA-pipe approximations of the forward kernels, evaluated on the GPU
(fa_selftest_poly) over dense sweeps of their domains and compared with
CUDA's exp2f / tanhf on the same inputs and with numpy's float64 functions.

The coefficients come from the Remez fits in csrc/fit_polynomials.py; the
bounds asserted are the ones stated there (and in include/fa.h): relative
7.5e-5 for the cubic 2^x, absolute 4e-8 for the degree-4 tanh on
|y| <= 0.5 and 1.1e-7 for the degree-2 tanh on |y| <= 0.25. Against CUDA's
functions the bound adds their own documented error (2 ulp).
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


def test_ex2_poly(cuda_ok):
    x = np.linspace(-126.0, 8.0, 2_000_001).astype(np.float32)
    poly, ref = run(0, x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(poly - exact) / exact
    assert rel.max() <= 7.5e-5, rel.max()
    rel_cuda = np.abs(poly - ref) / ref
    assert rel_cuda.max() <= 7.5e-5 + 2 * 2.0 ** -23, rel_cuda.max()
    # integers map to exact powers of two up to the fit's error at f = 0
    xi = np.arange(-126, 9, dtype=np.float32)
    pi, _ = run(0, xi)
    assert np.all(np.abs(pi / np.exp2(xi.astype(np.float64)) - 1) <= 7.5e-5)


@pytest.mark.parametrize("which,ymax,bound", [(1, 0.5, 4.0e-8), (2, 0.25, 1.1e-7)])
def test_tanh_poly(cuda_ok, which, ymax, bound):
    x = np.linspace(-ymax, ymax, 2_000_001).astype(np.float32)
    poly, ref = run(which, x)
    exact = np.tanh(x.astype(np.float64))
    err = np.abs(poly - exact)
    assert err.max() <= bound, err.max()
    err_cuda = np.abs(poly - ref)
    assert np.all(err_cuda <= bound + 2 * ulp(ref)), err_cuda.max()
    # odd symmetry is exact
    np.testing.assert_array_equal(poly, -poly[::-1])
