"""Float64 CPU oracle for Longformer banded + global self-attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the package smoke check
and by the benchmark's CPU-baseline leg, never by the product path.  It is
independent of the CUDA library: it shares no source, header, constant or
helper with it and imports nothing from the package.

"FTL" below is the page "FasterTransformer Longformer 推理加速实践：PyTorch
集成、输入约束与端到端性能解析".  Each function cites the section it follows.

Parity status per function:
  * global_partition   -- pinned (brute force + hand-written golden file).
  * attention          -- pinned (dense brute force with an explicit mask,
                          closed form at q = 0, library SDPA special cases,
                          invariants); with any_pos (global tokens at any
                          position) pinned by a hand-worked golden file,
                          dense brute force, the q = 0 closed form,
                          invariants and bit-equality with the prefix
                          definition on prefix masks.
  * encoder_layer      -- pinned per step (numpy/scipy library routines,
                          LayerNorm moments, GELU closed values).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

D = 64
SCALE = 0.125  # 1/sqrt(64): reading of FTL §PyTorch OP (attn_scaler has no value on the page)

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        ip = ctypes.POINTER(ctypes.c_int32)
        lib.lfo_num_threads.restype = ctypes.c_int
        lib.lfo_check_shape.argtypes = [ctypes.c_int] * 4
        lib.lfo_check_shape.restype = ctypes.c_int
        for fn in (lib.lfo_global_partition, lib.lfo_global_partition_any):
            fn.argtypes = [fp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ip, ip]
            fn.restype = ctypes.c_int
        for fn in (lib.lfo_attention, lib.lfo_attention_any):
            fn.argtypes = [dp] * 6 + [fp, fp] + [ctypes.c_int] * 4 + [ctypes.c_double, dp]
            fn.restype = ctypes.c_int
        lib.lfo_attention_rows.argtypes = ([dp] * 6 + [fp, fp] + [ctypes.c_int] * 4 +
                                           [ctypes.c_double, ctypes.c_int, ip, ctypes.c_longlong, dp])
        lib.lfo_attention_rows.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the C oracle runs on (OpenMP)."""
    return _load().lfo_num_threads()


def _f64(a):
    if hasattr(a, "detach"):  # torch tensor: exact widening of its stored values
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu().float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class OracleError(RuntimeError):
    def __init__(self, status: int):
        super().__init__("oracle status %d" % status)
        self.status = status


def check_shape(B: int, H: int, L: int, w: int) -> int:
    """FTL §使用前提 items 1-2: status of the shape constraints (0 = ok)."""
    return _load().lfo_check_shape(B, H, L, w)


def global_partition(global_mask, w: int, any_pos: bool = False):
    """invokeInitLongformerIdx, FTL §计算流程 / 预处理.

    Returns (global_idx int32 [B, L], global_token_nums int32 [B], status):
    flagged (global_mask == 0.0) positions ascending at the front, the others
    descending at the back; status 5 if some g_b > w, 6 if the flagged
    positions of some sample are not the prefix 0..g_b-1 (FTL §使用前提 items
    3-4; with any_pos, global tokens may lie anywhere and only item 3 is
    checked)."""
    gm = _f32(global_mask)
    B, L = gm.shape
    idx = np.zeros((B, L), dtype=np.int32)
    nums = np.zeros((B,), dtype=np.int32)
    fn = _load().lfo_global_partition_any if any_pos else _load().lfo_global_partition
    st = fn(_ptr(gm, ctypes.c_float), B, L, w, _ptr(idx, ctypes.c_int32), _ptr(nums, ctypes.c_int32))
    return idx, nums, st


def attention(q, k, v, qg, kg, vg, local_mask, global_mask, w: int, scale: float = SCALE,
              any_pos: bool = False):
    """The attention layer of FTL §计算流程 / 每个 Transformer 层 steps 3-5.

    Inputs q, k, v, qg, kg, vg are [B, H, L, 64] (their stored values are
    widened exactly to float64); masks are [B, L] float32.  Returns out
    float64 [B, L, H, 64].  Raises OracleError on a constraint failure.

    any_pos: global tokens (global_mask == 0.0) may lie anywhere, the
    HuggingFace arrangement that FTL §使用前提 item 4 sets apart from FT's
    prefix rule; a non-global row then attends its window united with every
    global token, each key once."""
    arrs = [_f64(t) for t in (q, k, v, qg, kg, vg)]
    B, H, L, d = arrs[0].shape
    assert d == D
    lm, gm = _f32(local_mask), _f32(global_mask)
    out = np.zeros((B, L, H, D), dtype=np.float64)
    fn = _load().lfo_attention_any if any_pos else _load().lfo_attention
    st = fn(*[_ptr(a, ctypes.c_double) for a in arrs],
            _ptr(lm, ctypes.c_float), _ptr(gm, ctypes.c_float),
            B, H, L, w, float(scale), _ptr(out, ctypes.c_double))
    if st != 0:
        raise OracleError(st)
    return out


def attention_rows(q, k, v, qg, kg, vg, local_mask, global_mask, w: int, rows,
                   scale: float = SCALE, any_pos: bool = False):
    """Same as :func:`attention`, for the listed rows only.

    rows: int array [n, 3] of (b, h, i).  Returns float64 [n, 64] =
    out[b, i, h, :]."""
    arrs = [_f64(t) for t in (q, k, v, qg, kg, vg)]
    B, H, L, d = arrs[0].shape
    lm, gm = _f32(local_mask), _f32(global_mask)
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    out = np.zeros((rows.shape[0], D), dtype=np.float64)
    st = _load().lfo_attention_rows(*[_ptr(a, ctypes.c_double) for a in arrs],
                                    _ptr(lm, ctypes.c_float), _ptr(gm, ctypes.c_float),
                                    B, H, L, w, float(scale), 1 if any_pos else 0,
                                    _ptr(rows, ctypes.c_int32), rows.shape[0],
                                    _ptr(out, ctypes.c_double))
    if st != 0:
        raise OracleError(st)
    return out


# ---------------------------------------------------------------------------
# One encoder layer, FTL §计算流程 / 每个 Transformer 层 steps 1-6, in numpy
# float64.  Weight convention: y = x @ W + b with W stored [in, out] (the page,
# §PyTorch OP: weights are transposed from the HF layout and concatenated, q
# k v kg vg contiguous).

def gelu(x):
    """GELU, exact erf form 0.5 x (1 + erf(x / sqrt 2)) (reading: the page
    names GELU without a formula)."""
    from scipy.special import erf
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def layer_norm(z, gamma, beta, eps):
    """LayerNorm over the last axis with the population variance."""
    mu = z.mean(axis=-1, keepdims=True)
    var = ((z - mu) ** 2).mean(axis=-1, keepdims=True)
    return gamma * (z - mu) / np.sqrt(var + eps) + beta


def gelu_ffn(h, W_1, b_1, W_2, b_2, round_stored=None):
    """Step 6 of the layer before its LayerNorm (FTL §Longformer Encoder
    计算流程 / 每个 Transformer 层 step 6, GeluFfnLayer; the FastFFN page's
    linear -> GELU -> linear): h + b_2 + GELU(h W_1 + b_1) W_2, with the
    oracle's x @ W convention (W_1 [D, F], W_2 [F, D]).  round_stored:
    optional function applied to the F-wide intermediate, which the page's
    layer stores in T.  Float64 throughout."""
    keep = round_stored or (lambda a: a)
    h = _f64(h)
    f = keep(gelu(h @ _f64(W_1) + _f64(b_1)))
    return f @ _f64(W_2) + _f64(b_2) + h


def to_heads(y, H):
    """[B, L, H*64] -> [B, H, L, 64] (AddBiasTransposeToMultiHead layout, step 2)."""
    B, L, _ = y.shape
    return np.ascontiguousarray(y.reshape(B, L, H, D).transpose(0, 2, 1, 3))


def encoder_layer(x, local_mask, global_mask, weights: dict, H: int, w: int,
                  scale: float, eps: float, round_attention_inputs=None, round_stored=None,
                  any_pos: bool = False):
    """x: [B, L, H*64]; weights: float64 arrays with keys
    W_qkv_kgvg [5, D, D], b_qkv_kgvg [5, D], W_qg [D, D], b_qg [D],
    W_o [D, D], b_o [D], ln1_gamma, ln1_beta [D], W_1 [D, F], b_1 [F],
    W_2 [F, D], b_2 [D], ln2_gamma, ln2_beta [D].

    round_attention_inputs: optional function applied to each projected
    [B, H, L, 64] tensor before attention; round_stored: optional function
    applied to the attention output, to h and to the FFN intermediate.  The
    page's LongformerEncoder<T> keeps every intermediate buffer in T (FTL
    §Longformer Encoder 计算流程), so the comparison rounds where values are
    stored; all arithmetic stays float64.  any_pos: global tokens at any
    position (as in :func:`attention`).  Returns float64 [B, L, D]."""
    x = _f64(x)
    W = {k: _f64(v) for k, v in weights.items()}
    rnd = round_attention_inputs or (lambda a: a)
    keep = round_stored or (lambda a: a)
    proj = [to_heads(x @ W["W_qkv_kgvg"][n] + W["b_qkv_kgvg"][n], H) for n in range(5)]
    q, k, v, kg, vg = [rnd(p) for p in proj]
    qg = rnd(to_heads(x @ W["W_qg"] + W["b_qg"], H))
    att = attention(q, k, v, qg, kg, vg, local_mask, global_mask, w, scale, any_pos=any_pos)
    B, L = x.shape[:2]
    att = keep(att.reshape(B, L, H * D))
    h = keep(layer_norm(att @ W["W_o"] + W["b_o"] + x, W["ln1_gamma"], W["ln1_beta"], eps))
    z = gelu_ffn(h, W["W_1"], W["b_1"], W["W_2"], W["b_2"], round_stored=keep)
    return layer_norm(z, W["ln2_gamma"], W["ln2_beta"], eps)
