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
    for code in range(15):
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
    (dict(B=1, H=1 << 16, Ln=1 << 16, w=64), 13),   # B*H*L >= 2^31
    (dict(B=1 << 23, H=1, Ln=128, w=64), 13),
])
def test_attention_host_validation(L, kw, status):
    assert _attn(L, **kw) == status


def _attn_idx(L, B=1, H=1, Ln=512, w=64, dtype=1, ptrs=None, out=FAKE, gidx=FAKE, gnum=FAKE):
    p = ptrs or [FAKE] * 8
    return L.lf_attention_forward_idx(*[ctypes.c_void_p(x) for x in p], B, H, Ln, w, dtype, None,
                                      ctypes.c_void_p(out), ctypes.c_void_p(gidx), ctypes.c_void_p(gnum))


@pytest.mark.parametrize("kw,status", [
    (dict(ptrs=[FAKE] * 7 + [0]), 1),
    (dict(gidx=0), 1),
    (dict(gnum=0), 1),
    (dict(B=0), 2),
    (dict(Ln=500, w=64), 3),
    (dict(Ln=64, w=64), 4),
    (dict(dtype=7), 7),
    (dict(out=FAKE + 2), 8),
    (dict(gidx=FAKE + 4), 8),
    (dict(gnum=FAKE + 4), 8),
    (dict(gidx=FAKE + 4, Ln=500), 3),   # shape errors come before alignment
])
def test_attention_idx_host_validation(L, kw, status):
    assert _attn_idx(L, **kw) == status


def _attn_any(L, B=1, H=1, Ln=512, w=64, dtype=1, ptrs=None, out=FAKE):
    p = ptrs or [FAKE] * 8
    return L.lf_attention_forward_any_globals(*[ctypes.c_void_p(x) for x in p], B, H, Ln, w, dtype, None,
                                              ctypes.c_void_p(out))


@pytest.mark.parametrize("kw,status", [
    (dict(ptrs=[FAKE] * 7 + [0]), 1),
    (dict(ptrs=[0] + [FAKE] * 7), 1),
    (dict(out=0), 1),
    (dict(B=0), 2), (dict(H=-1), 2), (dict(w=0), 2), (dict(Ln=0), 2),
    (dict(Ln=500, w=64), 3),
    (dict(Ln=64, w=64), 4),
    (dict(dtype=7), 7),
    (dict(ptrs=[FAKE] * 6 + [FAKE + 4, FAKE]), 8),
    (dict(out=FAKE + 2), 8),
    (dict(B=1, H=1 << 16, Ln=1 << 16, w=64), 13),
])
def test_attention_any_globals_host_validation(L, kw, status):
    """The entry point for global tokens at any position rejects bad
    arguments on the host, before any device call."""
    assert _attn_any(L, **kw) == status


def test_any_globals_scratch_bytes_host_only(L):
    import torch
    B, H, Ln, w = 2, 16, 4096, 256
    tc = lf.lf_attention_scratch_bytes(B, H, Ln, w, torch.float16)
    anyb = lf.lf_attention_any_globals_scratch_bytes(B, H, Ln, w, torch.float16)
    # partition outputs (idx, counts, rank) plus qg/k/v slot buffers and slot masks
    slots = 3 * B * H * 256 * 64 * 2 + B * 256 * 4
    assert anyb >= tc + B * Ln * 4 + B * 4 + B * (Ln + 1) * 4 + slots
    assert anyb < tc + B * Ln * 4 + B * (Ln + 1) * 4 + slots + 8 * 256
    f32 = lf.lf_attention_any_globals_scratch_bytes(B, H, Ln, w, torch.float32)
    assert B * Ln * 4 < f32 < B * Ln * 4 + B * (Ln + 1) * 4 + 4 * 256
    assert lf.lf_attention_any_globals_scratch_bytes(1, 2, 500, 64, torch.float16) == 0


@pytest.mark.parametrize("args,status", [
    ((0, 1, 512, 64, FAKE, FAKE), 1),
    ((FAKE, 0, 512, 64, FAKE, FAKE), 2),
    ((FAKE, 1, 500, 64, FAKE, FAKE), 3),
    ((FAKE, 1, 64, 64, FAKE, FAKE), 4),
    ((FAKE, 1, 512, 64, FAKE + 4, FAKE), 8),
    ((FAKE, 1 << 16, 1 << 16, 64, FAKE, FAKE), 13),  # B*L >= 2^31
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


def _layer(L, B=1, H=4, Ln=512, w=64, ffn=512, dtype=1, ws_bytes=1 << 30, weights="ok", x=FAKE, ws=FAKE,
           fn="lf_encoder_layer_forward"):
    if weights == "null":
        wp = None
    else:
        vals = [FAKE] * len(lf.LAYER_FIELDS)
        if weights == "one_null":
            vals[4] = 0  # W_o
        if weights == "misaligned":
            vals[2] = FAKE + 2
        wp = ctypes.byref(lf.LayerWeights(ffn, *vals))
    return getattr(L, fn)(ctypes.c_void_p(x), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), wp,
                          B, H, Ln, w, 0.125, 1e-5, dtype, ctypes.c_void_p(ws), ws_bytes, None,
                          ctypes.c_void_p(FAKE))


@pytest.mark.parametrize("kw,status", [
    (dict(weights="null"), 1),
    (dict(weights="one_null"), 1),
    (dict(x=0), 1),
    (dict(B=0), 2),
    (dict(H=1), 2),             # hidden 64 is not a multiple of 128
    (dict(H=32), 2),            # hidden 2048 > 1024
    (dict(ffn=200), 2),         # FFN width not a multiple of 128
    (dict(Ln=500), 3),
    (dict(Ln=64), 4),
    (dict(dtype=0), 7),         # fp32 layer: no tensor-core path
    (dict(weights="misaligned"), 8),
    (dict(ws_bytes=1024), 12),  # workspace smaller than lf_encoder_layer_workspace_bytes
    (dict(ws=FAKE + 16), 12),   # workspace not 256-byte aligned
])
@pytest.mark.parametrize("fn", ["lf_encoder_layer_forward", "lf_encoder_layer_forward_any_globals"])
def test_layer_host_validation(L, kw, status, fn):
    assert _layer(L, fn=fn, **kw) == status


def test_layer_workspace_bytes_host_only(L):
    import torch
    n = lf.lf_encoder_layer_workspace_bytes(1, 16, 4096, 256, 4096, torch.float16)
    # five projections + qg + attention output + fp32 residual sum + h + FFN intermediate + scratch
    D, rows = 1024, 4096
    assert n >= (5 + 1 + 1 + 2 + 1) * rows * D * 2 + rows * 4096 * 2
    assert lf.lf_encoder_layer_workspace_bytes(1, 1, 512, 64, 512, torch.float16) == 0   # hidden 64
    assert lf.lf_encoder_layer_workspace_bytes(1, 4, 512, 64, 512, torch.float32) == 0


def _encoder(L, n=3, ffns=(512, 512, 512), bad_layer=None, ws_bytes=1 << 30, layers="ok", fn="lf_encoder_forward"):
    arr = (lf.LayerWeights * max(n, 1))()
    for j in range(min(n, len(ffns))):
        vals = [FAKE] * len(lf.LAYER_FIELDS)
        if bad_layer == j:
            vals[8] = 0  # W_1 of that layer
        arr[j] = lf.LayerWeights(ffns[j], *vals)
    lp = None if layers == "null" else arr
    return getattr(L, fn)(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), lp, n,
                          1, 4, 512, 64, 0.125, 1e-5, 1, ctypes.c_void_p(FAKE), ws_bytes, None,
                          ctypes.c_void_p(FAKE + 256))


@pytest.mark.parametrize("kw,status", [
    (dict(layers="null"), 1),
    (dict(n=0), 2),
    (dict(ffns=(512, 384, 512)), 2),  # the layers must share the FFN width
    (dict(bad_layer=2), 1),           # the last layer's missing weight is caught before any launch
    (dict(ws_bytes=1024), 12),
])
@pytest.mark.parametrize("fn", ["lf_encoder_forward", "lf_encoder_forward_any_globals"])
def test_encoder_host_validation(L, kw, status, fn):
    assert _encoder(L, fn=fn, **kw) == status


def test_encoder_workspace_bytes_host_only(L):
    import torch
    one = lf.lf_encoder_layer_workspace_bytes(1, 4, 512, 64, 512, torch.float16)
    assert lf.lf_encoder_workspace_bytes(1, 1, 4, 512, 64, 512, torch.float16) == one
    act = 512 * 256 * 2  # one [B, L, D] buffer, D = 256
    assert lf.lf_encoder_workspace_bytes(24, 1, 4, 512, 64, 512, torch.float16) == one + 2 * act
    assert lf.lf_encoder_workspace_bytes(0, 1, 4, 512, 64, 512, torch.float16) == 0


def test_any_globals_layer_workspace_bytes_host_only(L):
    import torch
    B, H, Ln, w, F = 1, 16, 4096, 256, 4096
    pre = lf.lf_encoder_layer_workspace_bytes(B, H, Ln, w, F, torch.float16)
    anyb = lf.lf_encoder_layer_any_globals_workspace_bytes(B, H, Ln, w, F, torch.float16)
    D, gcap = H * 64, 256
    # no position-indexed qg buffer; the partition, rank table, slot buffers
    # and the gathered rows of x instead
    extra = (Ln * 4 + Ln * 4 + 3 * B * H * gcap * 64 * 2 + B * gcap * 4 + B * gcap * D * 2)
    assert anyb == pytest.approx(pre - B * Ln * D * 2 + extra, abs=16 * 256)
    act = B * Ln * D * 2
    assert lf.lf_encoder_any_globals_workspace_bytes(3, B, H, Ln, w, F, torch.float16) == anyb + 2 * act
    assert lf.lf_encoder_layer_any_globals_workspace_bytes(1, 4, 512, 64, 512, torch.float32) == 0


def test_version(L):
    """1.4: the partition and the attention in one call."""
    assert L.lf_version() == 104


def test_selftest_wait_limits_checked_on_host(L):
    """Wait limits outside [1 us, 100 ms] are rejected before anything is
    launched (no GPU needed)."""
    import ctypes
    for bad in (0, 999, 100000001):
        assert L.lf_selftest_bounded_wait(ctypes.c_ulonglong(bad), None) == 2


def _ffn(L, rows=256, D=1024, F=4096, dtype=1, path=0, ws=FAKE, ws_bytes=1 << 30, h=FAKE, z=FAKE, w1=FAKE):
    return L.lf_gelu_ffn_forward(ctypes.c_void_p(h), ctypes.c_void_p(w1), ctypes.c_void_p(FAKE),
                                 ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), rows, D, F, dtype, path,
                                 ctypes.c_void_p(ws), ws_bytes, None, ctypes.c_void_p(z))


@pytest.mark.parametrize("kw,status", [
    (dict(h=0), 1),
    (dict(z=0), 1),
    (dict(w1=FAKE + 4), 8),
    (dict(dtype=0), 7),
    (dict(rows=0), 2),
    (dict(D=64), 2),            # not a multiple of 128
    (dict(D=2048), 2),          # > 1024
    (dict(F=200), 2),           # not a multiple of 128
    (dict(path=3), 2),          # unknown path
    (dict(F=640, path=2), 2),   # the fused path needs F a multiple of 4 * 128 at D = 1024
    (dict(F=640, path=1, ws_bytes=1024), 12),
    (dict(F=640, path=0, ws=FAKE + 16), 12),  # auto runs F = 640 unfused: workspace misaligned
])
def test_ffn_host_validation(L, kw, status):
    assert _ffn(L, **kw) == status


def test_ffn_workspace_bytes_and_path_setting(L):
    import torch
    f16 = torch.float16
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 1024, 4096, f16, "unfused") == 4096 * 4096 * 2
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 1024, 4096, f16, "fused") == 0
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 1024, 640, f16, "fused") == 0      # not taken: invalid
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 1024, 640, f16, "auto") == 4096 * 640 * 2
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 1024, 4096, torch.float32, "auto") == 0
    # auto: fused (no workspace) where one CTA holds a row tile's output, else the two GEMMs
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 256, 1024, f16, "auto") == 0
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 512, 2048, f16, "auto") == 4096 * 2048 * 2
    assert lf.lf_gelu_ffn_workspace_bytes(4096, 1024, 4096, f16, "auto") == 4096 * 4096 * 2
    assert L.lf_set_ffn_path(7) == 2
    before = lf.lf_get_ffn_path()
    for p in ("unfused", "fused", "auto"):
        lf.lf_set_ffn_path(p)
        assert lf.lf_get_ffn_path() == p
    lf.lf_set_ffn_path(before)
