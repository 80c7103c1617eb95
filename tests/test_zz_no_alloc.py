"""The entry point that allocates no device memory.

Callers inside another framework's memory pool, or on allocation-free
real-time paths, cannot let the library cudaMalloc its scratch; they use
lf_attention_forward_noalloc, whose scratch is a fixed array in the library's
device image.  This file is collected last on purpose: it must pass both in a
fresh process and after every other test.
"""
import pytest
import torch

from sparse_attention_banded_b200 import build, inputs, lf
from tests._util import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    lf.lib()
    yield


@pytest.mark.parametrize("cid,shape", [
    (2, None),                                   # fp16 L=4096 w=256 workload
    (None, (2, 3, 640, 128, "bf16", [5, 128], [0, 77])),
])
def test_noalloc_matches_regular_entry_point_twice(cid, shape):
    if cid is not None:
        wl, t, lm, gm = inputs.workload_inputs(cid)
        w = wl.w
    else:
        B, H, L, w, dtype, g, pad = shape
        t = inputs.attention_inputs(B, H, L, dtype, seed=21)
        lm, gm = inputs.masks(B, L, g, pad)
    dev = [t[n].cuda() for n in inputs.NAMES]
    lmc, gmc = lm.cuda(), gm.cuda()
    ref = lf.lf_attention_forward(*dev, lmc, gmc, w)
    for _ in range(2):
        out = lf.lf_attention_forward_noalloc(*dev, lmc, gmc, w)
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= TOL[out.dtype], err


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # B*H = 64 heads at L = 16384, w = 256 needs far more than 32 MiB of scratch
    B, H, L, w = 4, 16, 16384, 256
    assert lf.lf_attention_scratch_bytes(B, H, L, w, torch.float16) > (32 << 20)
    q = torch.empty(16, dtype=torch.float16, device="cuda")
    m = torch.empty(4, dtype=torch.float32, device="cuda")
    st = lf.lib().lf_attention_forward_noalloc(*([lf._ptr(q)] * 6), lf._ptr(m), lf._ptr(m), B, H, L, w,
                                               lf.LF_F16, lf._stream(None), lf._ptr(q))
    assert st == 14
