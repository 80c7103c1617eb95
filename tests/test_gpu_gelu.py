"""The GELU of the GEMM and fused-FFN epilogues, checked on the device
against the erf-form GELU in float64.

gelu_erf_as (csrc/lf_gelu.cuh) evaluates 0.5 x (1 + erf(x / sqrt 2)) with
erf from Abramowitz & Stegun, Handbook of Mathematical Functions, formula
7.1.26 (|error| <= 1.5e-7), its reciprocal and exponential on the MUFU unit.
The test compiles the function into a small kernel, runs it over a dense
grid of [-12, 12] and special values, and bounds its error by the formula's
bound (1.5e-7 on erf, 0.75e-7 |x| on GELU), the MUFU reciprocal and
exponential (relative errors near 2^-22 on 1 - erf, up to 2.4e-7 |x|) and
the fp32 rounding of the few operations: |got - ref| <= 5e-7 |x| + 1e-9,
about a two-thousandth of an fp16 ulp of the result, which the epilogues
round to the dtype.  The same kernel also evaluates CUDA's erff form, whose
error on the grid is of the same size (4.9e-7 against 4.2e-7 measured).
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch
from scipy.special import erf

from sparse_attention_banded_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_attention_banded_b200", "csrc")

PROBE = r"""
#include "lf_gelu.cuh"
__global__ void gelu_values(const float* x, float* y, float* z, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        y[i] = lf::gelu_erf_as(x[i]);
        z[i] = 0.5f * x[i] * (1.0f + erff(x[i] * 0.70710678118654752f));
    }
}
extern "C" int run_gelu(const float* x, float* y, float* z, int n) {
    gelu_values<<<(n + 255) / 256, 256>>>(x, y, z, n);
    return (int)cudaGetLastError();
}
"""


@pytest.fixture(scope="module")
def probe():
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    src = os.path.join(out_dir, "gelu_probe.cu")
    so = os.path.join(out_dir, "gelu_probe.so")
    with open(src, "w") as f:
        f.write(PROBE)
    cmd = [build.nvcc()] + build.ARCH + ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", CSRC,
                                         src, "-o", so]
    subprocess.run(cmd, check=True, capture_output=True)
    lib = ctypes.CDLL(so)
    lib.run_gelu.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    lib.run_gelu.restype = ctypes.c_int
    return lib


def _eval(lib, x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    xd = torch.from_numpy(x).cuda()
    yd, zd = torch.empty_like(xd), torch.empty_like(xd)
    assert lib.run_gelu(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yd.data_ptr()),
                        ctypes.c_void_p(zd.data_ptr()), x.size) == 0
    torch.cuda.synchronize()
    return x, yd.cpu().numpy(), zd.cpu().numpy()


def _gelu64(x):
    x = x.astype(np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def test_gelu_error_on_dense_grid(probe):
    grid = np.linspace(-12.0, 12.0, 1 << 21, dtype=np.float64).astype(np.float32)
    special = np.array([0.0, -0.0, 1e-30, -1e-30, 1e-6, -1e-6, 0.5, -0.5, 1.0, -1.0, 3.0, -3.0, 8.0, -8.0,
                        30.0, -30.0, 1e4, -1e4], dtype=np.float32)
    x, y, z = _eval(probe, np.concatenate([grid, special]))
    ref = _gelu64(x)
    bound = 5e-7 * np.abs(x.astype(np.float64)) + 1e-9
    err = np.abs(y.astype(np.float64) - ref)
    err_cuda = np.abs(z.astype(np.float64) - ref)
    print("gelu_erf_as on [-12, 12]: max |err| %.3e, max |err| / bound %.3f; erff form max |err| %.3e"
          % (err.max(), (err / bound).max(), err_cuda.max()))
    assert np.all(np.isfinite(y))
    assert np.all(err <= bound)


def test_gelu_limits(probe):
    """GELU(0) = 0 exactly, GELU(x) = x for large x and 0 for very negative x,
    and GELU(x) - GELU(-x) = x."""
    x, y, _ = _eval(probe, np.array([0.0, 20.0, 1e4, -20.0, -1e4], dtype=np.float32))
    assert y[0] == 0.0 and y[1] == 20.0 and y[2] == 1e4
    assert abs(float(y[3])) < 1e-30 and abs(float(y[4])) < 1e-30
    g = np.linspace(0.0, 10.0, 4097, dtype=np.float32)
    _, yp, _ = _eval(probe, g)
    _, yn, _ = _eval(probe, -g)
    assert np.abs((yp.astype(np.float64) - yn) - g).max() <= 5e-7 * 10.0 + 1e-6
