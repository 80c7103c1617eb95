"""The FMA-pipe exponential of the attention kernel's softmax, checked on
the device against exp2 in float64.

exp2_poly2 (csrc/lf_pair_math.cuh) evaluates 2^x for a pair of floats
without the MUFU unit: Cody-Waite reduction x = n + f with |f| <= 1/2, a
fitted cubic for 2^f (documented maximum relative error 7.5e-5), and n
added to the exponent bits; x is clamped at -125 so the result stays a
normal number.  The test compiles the function into a small kernel, runs it
over a dense grid of [-125, 0] plus the reduction's edge points, and checks
the relative error against numpy's float64 exp2 of the same float32 inputs.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from sparse_attention_banded_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_attention_banded_b200", "csrc")

PROBE = r"""
#include "lf_pair_math.cuh"
__global__ void exp2_pairs(const float* x, float* y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        const float2 r = lf::exp2_poly2(make_float2(x[i], x[i + 1]));
        y[i] = r.x;
        y[i + 1] = r.y;
    }
}
extern "C" int run_exp2_pairs(const float* x, float* y, int n) {
    const int pairs = n / 2;
    exp2_pairs<<<(pairs + 255) / 256, 256>>>(x, y, n);
    return (int)cudaGetLastError();
}
"""


@pytest.fixture(scope="module")
def probe():
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    src = os.path.join(out_dir, "exp2_probe.cu")
    so = os.path.join(out_dir, "exp2_probe.so")
    with open(src, "w") as f:
        f.write(PROBE)
    cmd = [build.nvcc()] + build.ARCH + ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", CSRC,
                                         src, "-o", so]
    subprocess.run(cmd, check=True, capture_output=True)
    lib = ctypes.CDLL(so)
    lib.run_exp2_pairs.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.run_exp2_pairs.restype = ctypes.c_int
    return lib


def _eval(lib, x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    assert lib.run_exp2_pairs(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yd.data_ptr()), x.size) == 0
    torch.cuda.synchronize()
    return x, yd.cpu().numpy()


def test_exp2_poly2_relative_error_on_dense_grid(probe):
    grid = np.linspace(-125.0, 0.0, 1 << 21, dtype=np.float64).astype(np.float32)
    # the reduction's edges: integers and half-integers (|f| = 1/2), and their float neighbours
    edges = np.arange(-125.0, 0.5, 0.5, dtype=np.float32)
    edges = np.concatenate([edges, np.nextafter(edges, np.float32(-np.inf)), np.nextafter(edges, np.float32(np.inf))])
    edges = edges[(edges >= -125.0) & (edges <= 0.0)]
    x, y = _eval(probe, np.concatenate([grid, edges]))
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - ref) / ref
    print("exp2_poly2 on [-125, 0]: max relative error %.3e over %d points" % (rel.max(), x.size))
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert rel.max() <= 7.5e-5


def test_exp2_poly2_clamps_below_minus_125(probe):
    """Inputs below -125 (masked scores) give the value at -125: a normal
    float within the relative bound of 2^-125."""
    x, y = _eval(probe, np.array([-125.5, -126.0, -200.0, -1e4, -np.inf, -125.0], dtype=np.float32))
    assert np.all(y[:5] == y[5])
    assert abs(float(y[5]) / 2.0 ** -125 - 1.0) <= 7.5e-5
