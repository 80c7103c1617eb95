"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/lf.h declares, and rejects bad arguments on the host before
touching the device."""
import ctypes
import os

import pytest

from sparse_attention_banded_b200 import build, lf

HERE = os.path.dirname(__file__)


@pytest.fixture(scope="module")
def L():
    build.build()
    return lf.lib()


def test_exports_every_declared_function(L):
    names = lf.declared_functions()
    assert {"lf_init_global_idx", "lf_attention_forward", "lf_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(14):
        assert lf.status_string(code).startswith("LF_")
    assert lf.status_string(999) == "unknown lf_status"


FAKE = 0x10000  # 16-byte aligned dummy address; never dereferenced on these paths


def _attn(L, B=1, H=1, Ln=512, w=64, dtype=1, ptrs=None, out=FAKE):
    p = ptrs or [FAKE] * 8
    return L.lf_attention_forward(*[ctypes.c_void_p(x) for x in p], B, H, Ln, w, dtype, None,
                                  ctypes.c_void_p(out))


@pytest.mark.parametrize("kw,status", [
    (dict(ptrs=[FAKE] * 7 + [0]), 1),
    (dict(out=0), 1),
    (dict(B=0), 2), (dict(H=-1), 2), (dict(w=0), 2), (dict(Ln=0), 2),
    (dict(Ln=500, w=64), 3),
    (dict(Ln=64, w=64), 4),
    (dict(dtype=7), 7),
    (dict(ptrs=[FAKE + 8] + [FAKE] * 7), 8),
    (dict(out=FAKE + 2), 8),
])
def test_attention_host_validation(L, kw, status):
    assert _attn(L, **kw) == status


@pytest.mark.parametrize("args,status", [
    ((0, 1, 512, 64, FAKE, FAKE), 1),
    ((FAKE, 0, 512, 64, FAKE, FAKE), 2),
    ((FAKE, 1, 500, 64, FAKE, FAKE), 3),
    ((FAKE, 1, 64, 64, FAKE, FAKE), 4),
    ((FAKE, 1, 512, 64, FAKE + 4, FAKE), 8),
])
def test_global_idx_host_validation(L, args, status):
    gm, B, Ln, w, idx, nums = args
    assert L.lf_init_global_idx(ctypes.c_void_p(gm), B, Ln, w, ctypes.c_void_p(idx),
                                ctypes.c_void_p(nums), None, None) == status


def test_scratch_bytes_host_only(L):
    import torch
    assert lf.lf_attention_scratch_bytes(1, 16, 4096, 256, torch.float16) > 0
    assert lf.lf_attention_scratch_bytes(1, 2, 512, 64, torch.float32) == 0
    assert lf.lf_attention_scratch_bytes(1, 2, 500, 64, torch.float16) == 0
