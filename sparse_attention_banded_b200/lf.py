"""ctypes binding of liblf.so (argument marshalling only).

Each function mirrors the C entry point of the same name in ``include/lf.h``:
it takes torch CUDA tensors, passes their device pointers, sizes and the
current CUDA stream to the library, and raises :class:`LFError` on a non-zero
status.  All computation happens in the library's CUDA kernels; if the
library is missing this module raises instead of falling back to anything.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblf.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "lf.h")

LF_F32, LF_F16, LF_BF16 = 0, 1, 2
DTYPE_CODE = {torch.float32: LF_F32, torch.float16: LF_F16, torch.bfloat16: LF_BF16}

_lib = None

LAYER_FIELDS = ("W_qkv_kgvg", "b_qkv_kgvg", "W_qg", "b_qg", "W_o", "b_o", "ln1_gamma", "ln1_beta",
                "W_1", "b_1", "W_2", "b_2", "ln2_gamma", "ln2_beta")


class LayerWeights(ctypes.Structure):
    """lf_layer_weights of include/lf.h."""
    _fields_ = [("ffn_dim", ctypes.c_int)] + [(n, ctypes.c_void_p) for n in LAYER_FIELDS]


class LFError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s" % (where, status_string(status)))


def lib():
    """Load liblf.so once (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("liblf.so is not built; run `python -m sparse_attention_banded_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
        L.lf_status_string.argtypes = [i]
        L.lf_status_string.restype = ctypes.c_char_p
        L.lf_version.restype = i
        L.lf_device_status.argtypes = [vp, i]
        L.lf_device_status.restype = st
        L.lf_init_global_idx.argtypes = [vp, i, i, i, vp, vp, ctypes.POINTER(ctypes.c_int), vp]
        L.lf_init_global_idx.restype = st
        L.lf_attention_forward.argtypes = [vp] * 8 + [i, i, i, i, i, vp, vp]
        L.lf_attention_forward_idx.argtypes = [vp] * 8 + [i, i, i, i, i, vp, vp, vp, vp]
        L.lf_attention_forward_idx.restype = st
        L.lf_attention_forward.restype = st
        L.lf_attention_scratch_bytes.argtypes = [i, i, i, i, i]
        L.lf_attention_scratch_bytes.restype = ctypes.c_size_t
        L.lf_attention_forward_any_globals.argtypes = [vp] * 8 + [i, i, i, i, i, vp, vp]
        L.lf_attention_forward_any_globals.restype = st
        L.lf_attention_any_globals_scratch_bytes.argtypes = [i, i, i, i, i]
        L.lf_attention_any_globals_scratch_bytes.restype = ctypes.c_size_t
        L.lf_release_scratch.restype = st
        L.lf_attention_forward_noalloc.argtypes = [vp] * 8 + [i, i, i, i, i, vp, vp]
        L.lf_attention_forward_noalloc.restype = st
        L.lf_noalloc_device_status.argtypes = [vp, i]
        L.lf_noalloc_device_status.restype = st
        L.lf_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, vp]
        L.lf_selftest_bounded_wait.restype = st
        L.lf_encoder_layer_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.lf_encoder_layer_workspace_bytes.restype = ctypes.c_size_t
        L.lf_encoder_layer_forward.argtypes = [vp, vp, vp, ctypes.POINTER(LayerWeights), i, i, i, i,
                                               ctypes.c_float, ctypes.c_float, i, vp, ctypes.c_size_t, vp, vp]
        L.lf_encoder_layer_forward.restype = st
        L.lf_encoder_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        L.lf_encoder_workspace_bytes.restype = ctypes.c_size_t
        L.lf_encoder_forward.argtypes = [vp, vp, vp, ctypes.POINTER(LayerWeights), i, i, i, i, i,
                                         ctypes.c_float, ctypes.c_float, i, vp, ctypes.c_size_t, vp, vp]
        L.lf_encoder_layer_any_globals_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.lf_encoder_layer_any_globals_workspace_bytes.restype = ctypes.c_size_t
        L.lf_encoder_layer_forward_any_globals.argtypes = L.lf_encoder_layer_forward.argtypes
        L.lf_encoder_layer_forward_any_globals.restype = st
        L.lf_encoder_any_globals_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        L.lf_encoder_any_globals_workspace_bytes.restype = ctypes.c_size_t
        L.lf_encoder_forward_any_globals.argtypes = L.lf_encoder_forward.argtypes
        L.lf_encoder_forward_any_globals.restype = st
        L.lf_encoder_forward.restype = st
        L.lf_gelu_ffn_workspace_bytes.argtypes = [i, i, i, i, i]
        L.lf_gelu_ffn_workspace_bytes.restype = ctypes.c_size_t
        L.lf_gelu_ffn_forward.argtypes = [vp] * 5 + [i, i, i, i, i, vp, ctypes.c_size_t, vp, vp]
        L.lf_gelu_ffn_forward.restype = st
        L.lf_set_ffn_path.argtypes = [i]
        L.lf_set_ffn_path.restype = st
        L.lf_get_ffn_path.argtypes = []
        L.lf_get_ffn_path.restype = i
        _lib = L
    return _lib


def declared_functions():
    """Names of the functions include/lf.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*\s]+?\b(lf_\w+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    return lib().lf_status_string(int(status)).decode()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _check(status, where):
    if status != 0:
        raise LFError(status, where)


def lf_device_status(reset: bool = False, stream=None) -> int:
    """Synchronise and return the device status word (see lf.h)."""
    return lib().lf_device_status(_stream(stream), 1 if reset else 0)


def lf_init_global_idx(global_mask, w: int, global_idx=None, global_token_nums=None, sync: bool = True,
                       stream=None):
    """Global-token partition.  Returns (global_idx, global_token_nums,
    max_g); max_g is None when sync is False (then content errors go to the
    device status word)."""
    B, L = global_mask.shape
    if global_idx is None:
        global_idx = torch.empty(B, L, dtype=torch.int32, device=global_mask.device)
    if global_token_nums is None:
        global_token_nums = torch.empty(B, dtype=torch.int32, device=global_mask.device)
    mx = ctypes.c_int(-1)
    st = lib().lf_init_global_idx(_ptr(global_mask), B, L, w, _ptr(global_idx), _ptr(global_token_nums),
                                  ctypes.byref(mx) if sync else None, _stream(stream))
    _check(st, "lf_init_global_idx")
    return global_idx, global_token_nums, (mx.value if sync else None)


def lf_attention_forward(q, k, v, qg, kg, vg, local_mask, global_mask, w: int, out=None, stream=None):
    """Longformer attention; q..vg [B, H, L, 64], masks [B, L] float32.
    Returns out [B, L, H*64] in the input dtype."""
    B, H, L, _ = q.shape
    if out is None:
        out = torch.empty(B, L, H * 64, dtype=q.dtype, device=q.device)
    code = DTYPE_CODE.get(q.dtype, 99)
    st = lib().lf_attention_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg),
                                    _ptr(local_mask), _ptr(global_mask), B, H, L, w, code,
                                    _stream(stream), _ptr(out))
    _check(st, "lf_attention_forward")
    return out


def lf_attention_forward_idx(q, k, v, qg, kg, vg, local_mask, global_mask, w: int, out=None, global_idx=None,
                             global_token_nums=None, stream=None):
    """The partition of lf_init_global_idx and the attention in one call
    (one kernel launch for fp16 / bf16).  Returns (out, global_idx,
    global_token_nums)."""
    B, H, L, _ = q.shape
    if out is None:
        out = torch.empty(B, L, H * 64, dtype=q.dtype, device=q.device)
    if global_idx is None:
        global_idx = torch.empty(B, L, dtype=torch.int32, device=q.device)
    if global_token_nums is None:
        global_token_nums = torch.empty(B, dtype=torch.int32, device=q.device)
    code = DTYPE_CODE.get(q.dtype, 99)
    st = lib().lf_attention_forward_idx(_ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg),
                                        _ptr(local_mask), _ptr(global_mask), B, H, L, w, code,
                                        _stream(stream), _ptr(out), _ptr(global_idx), _ptr(global_token_nums))
    _check(st, "lf_attention_forward_idx")
    return out, global_idx, global_token_nums


def lf_attention_scratch_bytes(B: int, H: int, L: int, w: int, dtype) -> int:
    return lib().lf_attention_scratch_bytes(B, H, L, w, DTYPE_CODE[dtype])


def lf_attention_forward_any_globals(q, k, v, qg, kg, vg, local_mask, global_mask, w: int, out=None,
                                     stream=None):
    """Same as :func:`lf_attention_forward` with the global tokens
    (global_mask == 0.0) at any positions of the sequence."""
    B, H, L, _ = q.shape
    if out is None:
        out = torch.empty(B, L, H * 64, dtype=q.dtype, device=q.device)
    code = DTYPE_CODE.get(q.dtype, 99)
    st = lib().lf_attention_forward_any_globals(_ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg),
                                                _ptr(local_mask), _ptr(global_mask), B, H, L, w, code,
                                                _stream(stream), _ptr(out))
    _check(st, "lf_attention_forward_any_globals")
    return out


def lf_attention_any_globals_scratch_bytes(B: int, H: int, L: int, w: int, dtype) -> int:
    return lib().lf_attention_any_globals_scratch_bytes(B, H, L, w, DTYPE_CODE[dtype])


def lf_release_scratch():
    _check(lib().lf_release_scratch(), "lf_release_scratch")


def lf_attention_forward_noalloc(q, k, v, qg, kg, vg, local_mask, global_mask, w: int, out=None, stream=None):
    """Same as :func:`lf_attention_forward` through the entry point that
    allocates no device memory (fp16/bf16; scratch limited to 32 MiB)."""
    B, H, L, _ = q.shape
    if out is None:
        out = torch.empty(B, L, H * 64, dtype=q.dtype, device=q.device)
    code = DTYPE_CODE.get(q.dtype, 99)
    st = lib().lf_attention_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(qg), _ptr(kg), _ptr(vg),
                                            _ptr(local_mask), _ptr(global_mask), B, H, L, w, code,
                                            _stream(stream), _ptr(out))
    _check(st, "lf_attention_forward_noalloc")
    return out


def lf_noalloc_device_status(reset: bool = False, stream=None) -> int:
    """Synchronise and return the status word of the no-allocation entry
    point (see lf.h)."""
    return lib().lf_noalloc_device_status(_stream(stream), 1 if reset else 0)


def lf_selftest_bounded_wait(limit_ns: int, stream=None):
    """Launch the one-CTA kernel whose bounded wait runs out after limit_ns
    (see lf.h); the result is read with :func:`lf_device_status`."""
    _check(lib().lf_selftest_bounded_wait(int(limit_ns), _stream(stream)), "lf_selftest_bounded_wait")


FFN_PATH = {"auto": 0, "unfused": 1, "fused": 2}


def lf_gelu_ffn_workspace_bytes(rows: int, d_model: int, ffn_dim: int, dtype, path: str = "auto") -> int:
    return lib().lf_gelu_ffn_workspace_bytes(rows, d_model, ffn_dim, DTYPE_CODE[dtype], FFN_PATH[path])


def lf_gelu_ffn_forward(h, W_1, b_1, W_2, b_2, path: str = "auto", out=None, workspace=None, stream=None):
    """z = h + b_2 + GELU(h W_1^T + b_1) W_2^T (fp32) for h [rows, D];
    path "unfused" (two GEMMs), "fused" (one kernel, the intermediate kept
    on chip) or "auto" (see lf.h)."""
    rows, D = h.shape
    F = W_1.shape[0]
    if out is None:
        out = torch.empty(rows, D, dtype=torch.float32, device=h.device)
    need = lf_gelu_ffn_workspace_bytes(rows, D, F, h.dtype, path) if h.dtype in DTYPE_CODE else 0
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=h.device)
    st = lib().lf_gelu_ffn_forward(_ptr(h), _ptr(W_1), _ptr(b_1), _ptr(W_2), _ptr(b_2), rows, D, F,
                                   DTYPE_CODE.get(h.dtype, 99), FFN_PATH[path], _ptr(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(stream), _ptr(out))
    _check(st, "lf_gelu_ffn_forward")
    return out


def lf_set_ffn_path(path: str):
    """The FFN path of the layer and encoder calls in this process."""
    _check(lib().lf_set_ffn_path(FFN_PATH[path]), "lf_set_ffn_path")


def lf_get_ffn_path() -> str:
    code = lib().lf_get_ffn_path()
    return {v: k for k, v in FFN_PATH.items()}[code]


def lf_encoder_layer_workspace_bytes(B: int, H: int, L: int, w: int, ffn_dim: int, dtype) -> int:
    return lib().lf_encoder_layer_workspace_bytes(B, H, L, w, ffn_dim, DTYPE_CODE[dtype])


def _layer(name, size_fn, x, local_mask, global_mask, weights, H, w, attn_scale, ln_eps, out, workspace, stream):
    B, L, D = x.shape
    ffn = weights["W_1"].shape[0]
    wt = LayerWeights(ffn, *[weights[n].data_ptr() for n in LAYER_FIELDS])
    for n in LAYER_FIELDS:
        _ptr(weights[n])
    if out is None:
        out = torch.empty_like(x)
    need = size_fn(B, H, L, w, ffn, x.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    st = getattr(lib(), name)(_ptr(x), _ptr(local_mask), _ptr(global_mask), ctypes.byref(wt), B, H, L,
                              w, attn_scale, ln_eps, DTYPE_CODE.get(x.dtype, 99), _ptr(workspace),
                              workspace.numel(), _stream(stream), _ptr(out))
    _check(st, name)
    return out


def lf_encoder_layer_forward(x, local_mask, global_mask, weights: dict, H: int, w: int, attn_scale: float = 0.125,
                             ln_eps: float = 1e-5, out=None, workspace=None, stream=None):
    """One encoder layer; x [B, L, H*64]; weights: tensors named as the
    fields of lf_layer_weights (nn.Linear layout [out, in]), LayerNorm
    parameters fp32.  Returns out [B, L, H*64]."""
    return _layer("lf_encoder_layer_forward", lf_encoder_layer_workspace_bytes, x, local_mask, global_mask,
                  weights, H, w, attn_scale, ln_eps, out, workspace, stream)


def lf_encoder_layer_any_globals_workspace_bytes(B: int, H: int, L: int, w: int, ffn_dim: int, dtype) -> int:
    return lib().lf_encoder_layer_any_globals_workspace_bytes(B, H, L, w, ffn_dim, DTYPE_CODE[dtype])


def lf_encoder_layer_forward_any_globals(x, local_mask, global_mask, weights: dict, H: int, w: int,
                                         attn_scale: float = 0.125, ln_eps: float = 1e-5, out=None, workspace=None,
                                         stream=None):
    """Same as :func:`lf_encoder_layer_forward` with the global tokens
    (global_mask == 0.0) at any positions."""
    return _layer("lf_encoder_layer_forward_any_globals", lf_encoder_layer_any_globals_workspace_bytes, x,
                  local_mask, global_mask, weights, H, w, attn_scale, ln_eps, out, workspace, stream)


def lf_encoder_workspace_bytes(n_layers: int, B: int, H: int, L: int, w: int, ffn_dim: int, dtype) -> int:
    return lib().lf_encoder_workspace_bytes(n_layers, B, H, L, w, ffn_dim, DTYPE_CODE[dtype])


def lf_encoder_forward(x, local_mask, global_mask, layers: list, H: int, w: int, attn_scale: float = 0.125,
                       ln_eps: float = 1e-5, out=None, workspace=None, stream=None):
    """The encoder: the layers in `layers` (each a weight dict as for
    lf_encoder_layer_forward, same FFN width) applied in turn to x
    [B, L, H*64].  Returns out [B, L, H*64]."""
    return _encoder("lf_encoder_forward", lf_encoder_workspace_bytes, x, local_mask, global_mask, layers, H, w,
                    attn_scale, ln_eps, out, workspace, stream)


def lf_encoder_any_globals_workspace_bytes(n_layers: int, B: int, H: int, L: int, w: int, ffn_dim: int,
                                           dtype) -> int:
    return lib().lf_encoder_any_globals_workspace_bytes(n_layers, B, H, L, w, ffn_dim, DTYPE_CODE[dtype])


def lf_encoder_forward_any_globals(x, local_mask, global_mask, layers: list, H: int, w: int,
                                   attn_scale: float = 0.125, ln_eps: float = 1e-5, out=None, workspace=None,
                                   stream=None):
    """Same as :func:`lf_encoder_forward` with the global tokens
    (global_mask == 0.0) at any positions."""
    return _encoder("lf_encoder_forward_any_globals", lf_encoder_any_globals_workspace_bytes, x, local_mask,
                    global_mask, layers, H, w, attn_scale, ln_eps, out, workspace, stream)


def _encoder(fn_name, size_fn, x, local_mask, global_mask, layers, H, w, attn_scale, ln_eps, out, workspace, stream):
    B, L, D = x.shape
    n = len(layers)
    ffn = layers[0]["W_1"].shape[0] if n else 0
    arr = (LayerWeights * max(n, 1))()
    for j, weights in enumerate(layers):
        for name in LAYER_FIELDS:
            _ptr(weights[name])
        arr[j] = LayerWeights(weights["W_1"].shape[0], *[weights[name].data_ptr() for name in LAYER_FIELDS])
    if out is None:
        out = torch.empty_like(x)
    need = size_fn(n, B, H, L, w, ffn, x.dtype) if n else 0
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    st = getattr(lib(), fn_name)(_ptr(x), _ptr(local_mask), _ptr(global_mask), arr, n, B, H, L, w, attn_scale,
                                 ln_eps, DTYPE_CODE.get(x.dtype, 99), _ptr(workspace), workspace.numel(),
                                 _stream(stream), _ptr(out))
    _check(st, fn_name)
    return out
