"""Seeded synthetic inputs for the Longformer attention workloads.

This module only draws random numbers and lays out masks; it holds none of
the attention arithmetic.  Both the tests (for the oracle and the CUDA path)
and the benchmark take their inputs from here.

Workloads (all head_dim 64; values ~ N(0, 1) * 0.5 rounded to the dtype):
  1  fp32  B=1 H=2  L=512   w=64  g=8 prefix globals, no padding
  2  fp16  B=1 H=16 L=4096  w=256 g=64, last 300 positions padded
  3  bf16  B=4 H=16 L=4096  w=256 per-sample g ~ U{1..128}, padding tail
           ~ U{0..1024}, drawn in the order g_0, pad_0, g_1, pad_1, ...
  4  fp16  B=1 H=12 L=16384 w=256 g=32, no padding
  5  fp16  one encoder layer: B=1 L=4096 hidden 1024 (16 x 64) FFN 4096,
           w=256 g=64; x ~ N(0,1), weights ~ N(0, 0.02), biases 0,
           LayerNorm gamma 1 beta 0.
  6  fp16  workload 2 with its 64 global tokens at seeded random positions
           among the unpadded ones (the HuggingFace arrangement), for the
           entry point that takes global tokens at any position.
Mask conventions follow the FasterTransformer Longformer page's input list:
local_mask 1.0 = token / 0.0 = padding; global_mask 0.0 = global /
-10000.0 = not global.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

import torch

TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
NAMES = ("q", "k", "v", "qg", "kg", "vg")


@dataclass
class Workload:
    cid: int
    name: str
    dtype: str
    B: int
    H: int
    L: int
    w: int
    g: List[int] = field(default_factory=list)
    pad: List[int] = field(default_factory=list)
    seed: int = 0
    scattered: bool = False  # global tokens at random positions (masks_scattered)


def workload(cid: int) -> Workload:
    if cid == 1:
        return Workload(1, "fp32 B1 H2 L512 w64 g8", "f32", 1, 2, 512, 64, [8], [0], 1001)
    if cid == 2:
        return Workload(2, "fp16 Longformer-large B1 H16 L4096 w256 g64 pad300", "f16",
                        1, 16, 4096, 256, [64], [300], 1002)
    if cid == 3:
        gen = torch.Generator().manual_seed(1003)
        g, pad = [], []
        for _ in range(4):
            g.append(int(torch.randint(1, 129, (1,), generator=gen)))
            pad.append(int(torch.randint(0, 1025, (1,), generator=gen)))
        return Workload(3, "bf16 batched B4 H16 L4096 w256 g~U[1,128] pad~U[0,1024]", "bf16",
                        4, 16, 4096, 256, g, pad, 1003)
    if cid == 4:
        return Workload(4, "fp16 long document B1 H12 L16384 w256 g32", "f16",
                        1, 12, 16384, 256, [32], [0], 1004)
    if cid == 5:
        return Workload(5, "fp16 encoder layer B1 L4096 hidden1024 H16 w256 g64 ffn4096", "f16",
                        1, 16, 4096, 256, [64], [0], 1005)
    if cid == 6:
        return Workload(6, "fp16 B1 H16 L4096 w256 64 globals at random positions pad300", "f16",
                        1, 16, 4096, 256, [64], [300], 1006, scattered=True)
    raise ValueError("unknown workload %r" % cid)


def masks(B: int, L: int, g: List[int], pad: List[int]):
    """local_mask / global_mask [B, L] float32 for prefix globals g[b] and a
    padding tail of pad[b] positions."""
    local = torch.ones(B, L, dtype=torch.float32)
    glob = torch.full((B, L), -10000.0, dtype=torch.float32)
    for b in range(B):
        if pad[b] > 0:
            local[b, L - pad[b]:] = 0.0
        glob[b, :g[b]] = 0.0
    return local, glob


def masks_scattered(B: int, L: int, g: List[int], pad: List[int], seed: int, padded_globals: int = 0):
    """local_mask / global_mask [B, L] float32 with g[b] global tokens at
    positions drawn without replacement from the unpadded ones [0, L -
    pad[b]) (torch.Generator(seed), sample by sample), a padding tail of
    pad[b] positions, and padded_globals of each sample's global tokens also
    marked as padding."""
    gen = torch.Generator().manual_seed(seed)
    local, glob = masks(B, L, [0] * B, pad)
    for b in range(B):
        pos = torch.randperm(L - pad[b], generator=gen)[:g[b]]
        glob[b, pos] = 0.0
        if padded_globals:
            local[b, pos[:padded_globals]] = 0.0
    return local, glob


def attention_inputs(B: int, H: int, L: int, dtype: str, seed: int, scale: float = 0.5,
                     device: str = "cpu"):
    """q, k, v, qg, kg, vg: [B, H, L, 64] ~ N(0,1)*scale, rounded to dtype."""
    gen = torch.Generator().manual_seed(seed)
    out = {}
    for n in NAMES:
        t = torch.randn(B, H, L, 64, generator=gen, dtype=torch.float32) * scale
        out[n] = t.to(TORCH_DTYPES[dtype]).to(device)
    return out


def workload_inputs(cid: int, device: str = "cpu"):
    """(Workload, tensors dict, local_mask, global_mask) for workload cid."""
    wl = workload(cid)
    t = attention_inputs(wl.B, wl.H, wl.L, wl.dtype, wl.seed, device=device)
    if wl.scattered:
        lm, gm = masks_scattered(wl.B, wl.L, wl.g, wl.pad, wl.seed + 1)
    else:
        lm, gm = masks(wl.B, wl.L, wl.g, wl.pad)
    return wl, t, lm.to(device), gm.to(device)


def layer_inputs(cid: int = 5, hidden: int = 1024, ffn: int = 4096, device: str = "cpu", B=None, L=None,
                 dtype=None, g=None, pad=None, seed=None, bias_scale: float = 0.0, ln_scale: float = 0.0):
    """Encoder-layer input x [B, L, hidden] and weights in the nn.Linear
    layout [out, in] (y = x @ W.T + b; q k v kg vg weights contiguous as
    [5, hidden, hidden]).  Workload 5 by default; B, L, dtype, g, pad and
    seed override it for smaller test layers; bias_scale > 0 draws biases
    ~ N(0, bias_scale^2) and ln_scale > 0 draws gamma ~ 1 + N(0, ln_scale^2),
    beta ~ N(0, ln_scale^2) (workload 5 itself has zero biases, gamma 1,
    beta 0)."""
    wl = workload(cid)
    B = wl.B if B is None else B
    L = wl.L if L is None else L
    g = wl.g if g is None else g
    pad = wl.pad if pad is None else pad
    dt = TORCH_DTYPES[wl.dtype if dtype is None else dtype]
    gen = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    x = torch.randn(B, L, hidden, generator=gen)
    w = {}
    mats = [("W_q", (hidden, hidden)), ("W_k", (hidden, hidden)), ("W_v", (hidden, hidden)),
            ("W_kg", (hidden, hidden)), ("W_vg", (hidden, hidden)), ("W_qg", (hidden, hidden)),
            ("W_o", (hidden, hidden)), ("W_1", (ffn, hidden)), ("W_2", (hidden, ffn))]
    for n, shp in mats:
        w[n] = torch.randn(*shp, generator=gen) * 0.02
    def vec(n, scale, base=0.0):
        return base + torch.randn(n, generator=gen) * scale if scale > 0 else torch.full((n,), base)

    weights = {
        "W_qkv_kgvg": torch.stack([w["W_q"], w["W_k"], w["W_v"], w["W_kg"], w["W_vg"]]).to(dt),
        "b_qkv_kgvg": vec(5 * hidden, bias_scale).reshape(5, hidden).to(dt),
        "W_qg": w["W_qg"].to(dt), "b_qg": vec(hidden, bias_scale).to(dt),
        "W_o": w["W_o"].to(dt), "b_o": vec(hidden, bias_scale).to(dt),
        "ln1_gamma": vec(hidden, ln_scale, 1.0), "ln1_beta": vec(hidden, ln_scale),
        "W_1": w["W_1"].to(dt), "b_1": vec(ffn, bias_scale).to(dt),
        "W_2": w["W_2"].to(dt), "b_2": vec(hidden, bias_scale).to(dt),
        "ln2_gamma": vec(hidden, ln_scale, 1.0), "ln2_beta": vec(hidden, ln_scale),
    }
    lm, gm = masks(B, L, g, pad)
    return wl, x.to(dt).to(device), {k: v.to(device) for k, v in weights.items()}, lm.to(device), gm.to(device)
