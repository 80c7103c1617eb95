"""Failure detection on the GPU without a GPU fault.

Every device-side wait of the library's kernels is bounded: when one gives
up, the kernel records LF_ERR_DEVICE_TIMEOUT in the device status word and
returns, so the host sees an error status instead of a hang.  The
self-test entry point runs that same bounded wait on an mbarrier phase that
nothing completes (nothing else in flight), with a limit of about a
millisecond; these tests check that the call returns, that the status word
reports the timeout, and that the context stays usable afterwards.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_banded_b200 import build, inputs, lf
from tests._util import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    lf.lib()
    lf.lf_device_status(reset=True)
    yield


@pytest.mark.parametrize("limit_ns", [1_000_000, 20_000_000])
def test_bounded_wait_runs_out_and_reports_timeout(limit_ns):
    assert lf.lf_device_status(reset=True) == 0
    t0 = time.perf_counter()
    lf.lf_selftest_bounded_wait(limit_ns)
    st = lf.lf_device_status(reset=True)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert st == 10, lf.status_string(st)
    assert elapsed >= limit_ns * 1e-9 * 0.5
    assert elapsed < 5.0
    assert lf.lf_device_status(reset=True) == 0  # the reset cleared it


def test_context_usable_after_a_timeout():
    lf.lf_selftest_bounded_wait(1_000_000)
    assert lf.lf_device_status(reset=True) == 10
    B, H, L, w = 1, 2, 512, 64
    t = inputs.attention_inputs(B, H, L, "f16", seed=41)
    lm, gm = inputs.masks(B, L, [8], [20])
    dev = [t[n].cuda() for n in inputs.NAMES]
    out = lf.lf_attention_forward(*dev, lm.cuda(), gm.cuda(), w)
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
    ref = oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, w)
    got = out.float().cpu().numpy().reshape(B, L, H, 64)
    assert np.abs(got - ref).max() <= TOL[torch.float16]
