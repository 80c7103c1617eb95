"""Algorithmic work counts used for the roofline numbers (host-side only).

Encoder layer (one Longformer layer, hidden D = 64 H, FFN width Fw):
    F_layer = 2 L D (5 D) + 2 g_max D D + 2 L D D + 2 L D Fw + 2 L Fw D + F
per sample: the five q k v kg vg projections, the qg projection of the
global rows, the output projection, the two FFN GEMMs and the attention.

FLOPs count the band + global work of unpadded query rows:
    F = 4 * 64 * H * sum_b [ sum_{i valid, i >= g_b} |K_i| + sum_{i valid, i < g_b} L ]
with K_i = [max(0, i - w), min(L - 1, i + w)] united with [0, g_b) (each key
once); 2 * 64 FLOPs for the score and 2 * 64 for the value update per key.
Bytes are the compulsory HBM traffic of one call: q, k, v, kg, vg read in
full, qg rows i < g_b, the two fp32 masks, and the output written once.
"""
from __future__ import annotations

import numpy as np

ELEM = {"f32": 4, "f16": 2, "bf16": 2}


def key_set_sizes(L: int, w: int, g: int) -> np.ndarray:
    i = np.arange(L)
    lo = np.maximum(0, i - w)
    hi = np.minimum(L - 1, i + w)
    return (hi - lo + 1) + np.minimum(g, lo)


def flops(B: int, H: int, L: int, w: int, g_list, pad_list) -> float:
    total = 0
    for b in range(B):
        g, pad = g_list[b], pad_list[b]
        valid = np.arange(L) < L - pad
        sizes = key_set_sizes(L, w, g)
        is_global = np.arange(L) < g
        total += int(np.where(is_global, L, sizes)[valid].sum())
    return 4.0 * 64 * H * total


def flops_masks(local_mask, global_mask, H: int, w: int) -> float:
    """F for any masks, global tokens at any position: G_b = {j : global_mask
    == 0.0}; a local row's key set is its window united with G_b (each key
    once), a global row's is all L keys; unpadded query rows only."""
    lm = np.asarray(local_mask, dtype=np.float32)
    gm = np.asarray(global_mask, dtype=np.float32)
    B, L = lm.shape
    i = np.arange(L)
    lo = np.maximum(0, i - w)
    hi = np.minimum(L - 1, i + w)
    total = 0
    for b in range(B):
        G = gm[b] == 0.0
        before = np.concatenate([[0], np.cumsum(G)])  # global tokens before each position
        in_window = before[hi + 1] - before[lo]
        sizes = (hi - lo + 1) + int(G.sum()) - in_window
        total += int(np.where(G, L, sizes)[lm[b] == 1.0].sum())
    return 4.0 * 64 * H * total


def algorithmic_bytes(B: int, H: int, L: int, w: int, g_list, dtype: str) -> float:
    e = ELEM[dtype]
    full = 5 * B * H * L * 64 * e
    qg = sum(g_list) * H * 64 * e
    masks = 2 * B * L * 4
    out = B * L * H * 64 * e
    return float(full + qg + masks + out)


def layer_flops(B: int, H: int, L: int, w: int, g_list, pad_list, ffn: int) -> float:
    D = 64 * H
    gemm = B * (2.0 * L * D * 5 * D + 2.0 * L * D * D + 4.0 * L * D * ffn)
    gemm += 2.0 * max(g_list) * D * D * B
    return gemm + flops(B, H, L, w, g_list, pad_list)
