"""GPU parity of the entry point for global tokens at any position
(lf_attention_forward_any_globals) against the float64 oracle with any_pos.

The global tokens are those with global_mask == 0.0 wherever they lie (the
HuggingFace arrangement that the FasterTransformer Longformer page's
§使用前提 item 4 sets apart from FT's prefix rule).  Bars as for the prefix
path: max abs error 1e-4 (fp32), 1e-2 (fp16), 2e-2 (bf16); padded rows
exactly zero.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_banded_b200 import build, inputs, lf
from tests._util import TOL

pytestmark = pytest.mark.gpu

TDT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    lf.lib()
    lf.lf_device_status(reset=True)
    yield


def _run(t, lm, gm, w):
    dev = {n: t[n].cuda() for n in inputs.NAMES}
    out = lf.lf_attention_forward_any_globals(*[dev[n] for n in inputs.NAMES], lm.cuda(), gm.cuda(), w)
    torch.cuda.synchronize()
    return out


def _compare_full(t, lm, gm, w, dtype):
    B, H, L, _ = t["q"].shape
    out = _run(t, lm, gm, w).float().cpu().numpy().reshape(B, L, H, 64)
    ref = oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, w, any_pos=True)
    err = np.abs(out - ref).max()
    assert err <= TOL[dtype], "max abs err %g" % err
    pad = (lm.numpy() != 1.0)
    assert np.all(out[pad] == 0.0)
    return out, ref


SMALL = [
    # B, H, L, w, g list, pad list, padded global tokens per sample
    (1, 2, 512, 64, [8], [0], 0),
    (2, 3, 384, 64, [0, 64], [0, 100], 0),       # g = 0 and g = w
    (1, 2, 320, 64, [17], [33], 2),              # ragged L, padded global tokens
    (2, 2, 768, 128, [128, 3], [1, 0], 1),       # g = w = 128: one full slot block
    (1, 2, 1024, 256, [200], [257], 5),          # two slot blocks, two global row tiles
    (1, 1, 288, 96, [40], [5], 0),               # w not a multiple of 128
    (1, 2, 1024, 512, [300], [0], 3),            # L = 2w, wide band
    (1, 1, 12, 3, [2], [1], 0),                  # tiny
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B%dH%dL%dw%d" % s[:4])
def test_any_globals_small_parity(dtype, shape):
    B, H, L, w, g, pad, pg = shape
    t = inputs.attention_inputs(B, H, L, dtype, seed=hash((B, H, L, w, 6)) & 0xffff)
    lm, gm = inputs.masks_scattered(B, L, g, pad, seed=L + w, padded_globals=pg)
    _compare_full(t, lm, gm, w, TDT[dtype])


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("where", ["end", "middle_block", "every_7th", "prefix"])
def test_any_globals_arrangements(dtype, where):
    """Global tokens at the end of the sequence, as one block in the middle
    (inside many rows' windows), spread evenly, and as the prefix (which
    must give the prefix definition's result)."""
    B, H, L, w = 1, 2, 1024, 128
    t = inputs.attention_inputs(B, H, L, dtype, seed=21)
    lm, gm = inputs.masks(B, L, [0], [40])
    if where == "end":
        gm[0, L - 40 - 100:L - 40] = 0.0
    elif where == "middle_block":
        gm[0, 500:600] = 0.0
    elif where == "every_7th":
        gm[0, 3:L - 40:7][:128] = 0.0
    else:
        gm[0, :77] = 0.0
    _compare_full(t, lm, gm, w, TDT[dtype])


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_any_globals_rows_sum_to_one(dtype):
    B, H, L, w = 2, 2, 1024, 256
    t = inputs.attention_inputs(B, H, L, dtype, seed=4)
    t["v"] = torch.ones_like(t["v"])
    t["vg"] = torch.ones_like(t["vg"])
    lm, gm = inputs.masks_scattered(B, L, [50, 256], [77, 0], seed=9, padded_globals=3)
    out = _run(t, lm, gm, w).float().cpu().numpy().reshape(B, L, H, 64)
    valid = lm.numpy() == 1.0
    assert np.abs(out[valid] - 1.0).max() <= TOL[TDT[dtype]]
    assert np.all(out[~valid] == 0.0)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_any_globals_bitwise_invariant_outside_set(dtype):
    """Keys outside a local row's set (outside its window and not global)
    do not change the row at all."""
    B, H, L, w = 1, 1, 1024, 128
    t = inputs.attention_inputs(B, H, L, dtype, seed=5)
    lm, gm = inputs.masks_scattered(B, L, [30], [0], seed=11)
    G = set(np.flatnonzero(gm[0].numpy() == 0.0).tolist())
    i = next(i for i in range(600, L) if i not in G)
    base = _run(t, lm, gm, w).cpu()
    outside = [j for j in range(L) if abs(i - j) > w and j not in G]
    t2 = dict(t)
    for n in ("k", "v"):
        x = t[n].clone()
        x[0, 0, outside] = (torch.randn(len(outside), 64) * 3).to(x.dtype)
        t2[n] = x
    pert = _run(t2, lm, gm, w).cpu()
    assert torch.equal(pert[0, i], base[0, i])


def test_any_globals_device_status():
    B, H, L, w = 2, 1, 512, 64
    t = inputs.attention_inputs(B, H, L, "f16", seed=6)
    lm, gm = inputs.masks_scattered(B, L, [3, 20], [0, 0], seed=2)
    lf.lf_device_status(reset=True)
    _run(t, lm, gm, w)
    assert lf.lf_device_status(reset=True) == 0  # scattered globals are not an error here
    gm_bad = gm.clone()
    gm_bad[1, ::7] = 0.0  # sample 1: 74 > w global tokens
    out = _run(t, lm, gm_bad, w)
    assert lf.lf_device_status(reset=True) == 5
    assert torch.all(out[1] == 0)
    ref = oracle.attention(*[t[n][:1] for n in inputs.NAMES], lm[:1], gm[:1], w, any_pos=True)
    got = out[:1].float().cpu().numpy().reshape(1, L, H, 64)
    assert np.abs(got - ref).max() <= TOL[torch.float16]


def test_any_globals_repeated_calls_identical():
    wl, t, lm, gm = inputs.workload_inputs(6)
    dev = {n: t[n].cuda() for n in inputs.NAMES}
    lmc, gmc = lm.cuda(), gm.cuda()
    a = lf.lf_attention_forward_any_globals(*[dev[n] for n in inputs.NAMES], lmc, gmc, wl.w)
    for _ in range(3):
        b = lf.lf_attention_forward_any_globals(*[dev[n] for n in inputs.NAMES], lmc, gmc, wl.w)
        assert torch.equal(a, b)


def test_any_globals_workload_full_parity():
    """Workload 6 at full size (workload 2 with its 64 global tokens at random
    positions): every element against the oracle."""
    wl, t, lm, gm = inputs.workload_inputs(6)
    out = _run(t, lm, gm, wl.w).float().cpu().numpy().reshape(wl.B, wl.L, wl.H, 64)
    ref = oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, wl.w, any_pos=True)
    err = float(np.abs(out - ref).max())
    print("workload 6: max abs err %.3e over %d elements" % (err, out.size))
    assert err <= TOL[torch.float16], "max abs err %g" % err
    assert np.all(out[lm.numpy() != 1.0] == 0.0)


def test_scratch_reuse_across_shapes_and_dtypes():
    """Calls of other shapes and dtypes between two identical calls leave the
    result unchanged: the scheduler and split counters at the head of the
    shared scratch are cleared whenever a call of another layout wrote there
    (here an fp32 call, whose partition outputs start at the scratch's first
    byte, and a small shape whose split partials cover a larger shape's
    counters)."""
    def call(fn, B, H, L, w, g, pad, dtype, seed, scattered):
        t = inputs.attention_inputs(B, H, L, dtype, seed=seed)
        if scattered:
            lm, gm = inputs.masks_scattered(B, L, g, pad, seed=seed + 1)
        else:
            lm, gm = inputs.masks(B, L, g, pad)
        dev = [t[n].cuda() for n in inputs.NAMES]
        out = torch.full((B, L, H * 64), 3.0, dtype=dev[0].dtype, device="cuda")
        fn(*dev, lm.cuda(), gm.cuda(), w, out=out)
        torch.cuda.synchronize()
        return out.cpu()

    big = (1, 16, 2048, 256, [64], [0], "f16", 31)
    small = (2, 1, 512, 64, [3, 2], [0, 0], "f16", 32)
    anyf = lf.lf_attention_forward_any_globals
    pre = lf.lf_attention_forward
    ref_any = call(anyf, *big, True)
    ref_pre = call(pre, *big, False)
    call(anyf, *small[:6], "f32", 33, True)          # fp32: partition at the scratch start
    assert torch.equal(call(anyf, *big, True), ref_any)
    call(pre, *small, False)                          # partials over the larger shape's counters
    assert torch.equal(call(pre, *big, False), ref_pre)
    call(anyf, *small, True)
    assert torch.equal(call(pre, *big, False), ref_pre)
    call(anyf, *small[:6], "f32", 34, True)
    assert torch.equal(call(pre, *big, False), ref_pre)
    assert lf.lf_device_status(reset=True) == 0


def _full(wl_shape, g, pad, dtype, seed, pg=0):
    """Global tokens at random positions (pg of them padded per sample) on a
    full-size shape: every element against the oracle."""
    B, H, L, w = wl_shape
    t = inputs.attention_inputs(B, H, L, dtype, seed=seed)
    lm, gm = inputs.masks_scattered(B, L, g, pad, seed=seed + 1, padded_globals=pg)
    out = _run(t, lm, gm, w).float().cpu().numpy().reshape(B, L, H, 64)
    ref = oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, w, any_pos=True)
    err = float(np.abs(out - ref).max())
    print("B%d H%d L%d w%d %s: max abs err %.3e over %d elements" % (B, H, L, w, dtype, err, out.size))
    assert err <= TOL[TDT[dtype]], "max abs err %g" % err
    assert np.all(out[lm.numpy() != 1.0] == 0.0)


def test_any_globals_batched_bf16_full():
    """Workload 3's shape (bf16, four samples) with each sample's global
    tokens at random positions, some of them padded."""
    wl = inputs.workload(3)
    _full((wl.B, wl.H, wl.L, wl.w), wl.g, wl.pad, "bf16", seed=3003, pg=2)


def test_any_globals_long_sequence_full():
    """Workload 4's shape (16384 tokens) with 32 global tokens at random positions."""
    wl = inputs.workload(4)
    _full((wl.B, wl.H, wl.L, wl.w), wl.g, wl.pad, "f16", seed=3004)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_any_globals_g_equals_w_odd_band(dtype):
    """g = w = 192 (a band that is not a multiple of 128, two slot blocks,
    two global row tiles, the second one partial) at 3072 tokens."""
    _full((1, 4, 3072, 192), [192], [77], dtype, seed=3005, pg=4)
