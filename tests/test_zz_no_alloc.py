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

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    lf.lib()
    yield


def _case(cid, shape):
    if cid is not None:
        wl, t, lm, gm = inputs.workload_inputs(cid)
        return t, lm, gm, wl.w
    B, H, L, w, dtype, g, pad = shape
    t = inputs.attention_inputs(B, H, L, dtype, seed=21)
    lm, gm = inputs.masks(B, L, g, pad)
    return t, lm, gm, w


@pytest.mark.parametrize("cid,shape", [
    (2, None),                                   # fp16 L=4096 w=256 workload
    (None, (2, 3, 640, 128, "bf16", [5, 128], [0, 77])),
])
def test_noalloc_matches_regular_entry_point_twice(cid, shape):
    """Two calls in a row give exactly the regular entry point's output, and
    neither changes the device's free memory: the library scratch is
    released first and the reference is computed only afterwards, so a
    stray allocation on this path would show."""
    t, lm, gm, w = _case(cid, shape)
    dev = [t[n].cuda() for n in inputs.NAMES]
    lmc, gmc = lm.cuda(), gm.cuda()
    B, H, L, _ = dev[0].shape
    outs = [torch.empty(B, L, H * 64, dtype=dev[0].dtype, device="cuda") for _ in range(3)]
    lf.lf_release_scratch()
    lf.lf_noalloc_device_status(reset=True)
    # first call on the device resolves the array's address (module loading)
    lf.lf_attention_forward_noalloc(*dev, lmc, gmc, w, out=outs[2])
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for k in range(2):
        lf.lf_attention_forward_noalloc(*dev, lmc, gmc, w, out=outs[k])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert lf.lf_noalloc_device_status(reset=True) == 0
    ref = lf.lf_attention_forward(*dev, lmc, gmc, w)
    torch.cuda.synchronize()
    for k in range(2):
        assert torch.equal(outs[k], ref)


def test_noalloc_content_errors_are_readable():
    """g_b > w (zero output for that sample) and a global token after the
    prefix are recorded in the entry point's own status word."""
    B, H, L, w = 2, 1, 512, 64
    t = inputs.attention_inputs(B, H, L, "f16", seed=22)
    lm, gm = inputs.masks(B, L, [3, 2], [0, 0])
    dev = [t[n].cuda() for n in inputs.NAMES]
    lmc = lm.cuda()
    lf.lf_noalloc_device_status(reset=True)
    gm_bad = gm.clone()
    gm_bad[1, :w + 1] = 0.0
    out = lf.lf_attention_forward_noalloc(*dev, lmc, gm_bad.cuda(), w)
    assert lf.lf_noalloc_device_status(reset=True) == 5
    assert torch.all(out[1] == 0)
    gm_bad = gm.clone()
    gm_bad[0, 300] = 0.0
    lf.lf_attention_forward_noalloc(*dev, lmc, gm_bad.cuda(), w)
    assert lf.lf_noalloc_device_status(reset=True) == 6
    out = lf.lf_attention_forward_noalloc(*dev, lmc, gm.cuda(), w)
    assert lf.lf_noalloc_device_status(reset=True) == 0
    assert torch.equal(out, lf.lf_attention_forward(*dev, lmc, gm.cuda(), w))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # B*H = 64 heads at L = 16384, w = 256 needs far more than 32 MiB of scratch
    B, H, L, w = 4, 16, 16384, 256
    assert lf.lf_attention_scratch_bytes(B, H, L, w, torch.float16) > (32 << 20)
    q = torch.empty(16, dtype=torch.float16, device="cuda")
    m = torch.empty(4, dtype=torch.float32, device="cuda")
    st = lf.lib().lf_attention_forward_noalloc(*([lf._ptr(q)] * 6), lf._ptr(m), lf._ptr(m), B, H, L, w,
                                               lf.LF_F16, lf._stream(None), lf._ptr(q))
    assert st == 14
