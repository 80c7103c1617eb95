"""GPU parity of liblf.so against the float64 oracle, through the C ABI.

Bars: bit-exact for the global-index partition; max abs error 1e-4 (fp32),
1e-2 (fp16), 2e-2 (bf16) for attention outputs; padded rows exactly zero.
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
    out = lf.lf_attention_forward(*[dev[n] for n in inputs.NAMES], lm.cuda(), gm.cuda(), w)
    torch.cuda.synchronize()
    return out


def _compare_full(t, lm, gm, w, dtype):
    B, H, L, _ = t["q"].shape
    out = _run(t, lm, gm, w).float().cpu().numpy().reshape(B, L, H, 64)
    ref = oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, w)
    err = np.abs(out - ref).max()
    assert err <= TOL[dtype], "max abs err %g" % err
    pad = (lm.numpy() != 1.0)
    assert np.all(out[pad] == 0.0)
    return out, ref


# ---------------------------------------------------------------- partition

@pytest.mark.parametrize("seed", range(6))
def test_global_idx_bit_exact(seed):
    rng = np.random.default_rng(seed)
    B, w = int(rng.integers(1, 6)), int(rng.choice([3, 64, 256]))
    L = w * int(rng.integers(2, 40))
    gm = np.full((B, L), -10000.0, np.float32)
    for b in range(B):
        gm[b, : int(rng.integers(0, w + 1))] = 0.0
    idx, nums, mx = lf.lf_init_global_idx(torch.from_numpy(gm).cuda(), w)
    e_idx, e_nums, st = oracle.global_partition(gm, w)
    assert st == 0
    assert np.array_equal(idx.cpu().numpy(), e_idx)
    assert np.array_equal(nums.cpu().numpy(), e_nums)
    assert mx == int(e_nums.max())


@pytest.mark.parametrize("case", ["not_prefix", "too_many", "scatter"])
def test_global_idx_content_errors(case):
    B, L, w = 3, 1024, 128
    gm = np.full((B, L), -10000.0, np.float32)
    gm[0, :5] = 0.0
    if case == "not_prefix":
        gm[1, 700] = 0.0
    elif case == "too_many":
        gm[1, :w + 1] = 0.0
    else:
        gm[2, ::7] = 0.0
    e_idx, e_nums, st = oracle.global_partition(gm, w)
    g = torch.from_numpy(gm).cuda()
    with pytest.raises(lf.LFError) as e:
        lf.lf_init_global_idx(g, w)
    assert e.value.status == st
    # asynchronous mode: outputs still bit-exact, error in the status word
    lf.lf_device_status(reset=True)
    idx, nums, _ = lf.lf_init_global_idx(g, w, sync=False)
    assert lf.lf_device_status(reset=True) == st
    assert np.array_equal(idx.cpu().numpy(), e_idx)
    assert np.array_equal(nums.cpu().numpy(), e_nums)


# ---------------------------------------------------------------- attention, small shapes

SMALL = [
    # B, H, L, w, g list, pad list
    (1, 2, 512, 64, [8], [0]),
    (2, 3, 384, 64, [0, 64], [0, 100]),       # g = 0 and g = w
    (1, 2, 320, 64, [17], [33]),              # ragged: L not a multiple of 128
    (2, 2, 768, 128, [128, 3], [1, 0]),       # g = w = 128
    (1, 2, 1024, 256, [200], [257]),          # g > 128: two global row tiles
    (1, 1, 288, 96, [40], [5]),               # w not a multiple of 128, ragged L
    (1, 2, 1024, 512, [300], [0]),            # L = 2w, wide band
    (2, 1, 1536, 192, [1, 191], [1536 - 7, 0]),  # almost fully padded sample
    (1, 1, 12, 3, [2], [1]),                  # tiny
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B%dH%dL%dw%d" % s[:4])
def test_attention_small_parity(dtype, shape):
    B, H, L, w, g, pad = shape
    t = inputs.attention_inputs(B, H, L, dtype, seed=hash((B, H, L, w)) & 0xffff)
    lm, gm = inputs.masks(B, L, g, pad)
    _compare_full(t, lm, gm, w, TDT[dtype])


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_attention_fully_padded_sample(dtype):
    B, H, L, w = 2, 2, 512, 128
    t = inputs.attention_inputs(B, H, L, dtype, seed=3)
    lm, gm = inputs.masks(B, L, [4, 0], [L, 0])
    out, _ = _compare_full(t, lm, gm, w, TDT[dtype])
    assert np.all(out[0] == 0.0)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_attention_rows_sum_to_one(dtype):
    B, H, L, w = 1, 2, 1024, 256
    t = inputs.attention_inputs(B, H, L, dtype, seed=4)
    t["v"] = torch.ones_like(t["v"])
    t["vg"] = torch.ones_like(t["vg"])
    lm, gm = inputs.masks(B, L, [50], [77])
    out = _run(t, lm, gm, w).float().cpu().numpy().reshape(B, L, H, 64)
    valid = lm.numpy() == 1.0
    assert np.abs(out[valid] - 1.0).max() <= TOL[TDT[dtype]]
    assert np.all(out[~valid] == 0.0)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_attention_bitwise_invariant_outside_window(dtype):
    """Keys outside row i's set (finite values) do not change row i at all."""
    B, H, L, w = 1, 1, 1024, 128
    t = inputs.attention_inputs(B, H, L, dtype, seed=5)
    lm, gm = inputs.masks(B, L, [10], [0])
    base = _run(t, lm, gm, w).cpu()
    i = 700
    outside = [j for j in range(L) if abs(i - j) > w and j >= 10]
    t2 = dict(t)
    for n in ("k", "v"):
        x = t[n].clone()
        x[0, 0, outside] = (torch.randn(len(outside), 64) * 3).to(x.dtype)
        t2[n] = x
    pert = _run(t2, lm, gm, w).cpu()
    assert torch.equal(pert[0, i], base[0, i])


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_attention_growing_scores_rescale(dtype):
    """Scores that grow along the sequence, so the running row max rises by
    far more than 2^8 between key blocks: exercises the accumulator
    rescaling of the tensor-core path."""
    B, H, L, w = 1, 2, 2048, 256
    t = inputs.attention_inputs(B, H, L, dtype, seed=8)
    direction = torch.ones(64) / 8.0
    ramp = torch.linspace(0, 24, L)[:, None] * direction[None, :]
    for n in ("q", "qg"):
        t[n] = (t[n].float() + direction * 8).to(t[n].dtype)
    for n in ("k", "kg"):
        t[n] = (t[n].float() + ramp).to(t[n].dtype)
    lm, gm = inputs.masks(B, L, [40], [100])
    _compare_full(t, lm, gm, w, TDT[dtype])


def test_attention_device_status_errors():
    B, H, L, w = 2, 1, 512, 64
    t = inputs.attention_inputs(B, H, L, "f16", seed=6)
    lm, gm = inputs.masks(B, L, [3, 2], [0, 0])
    lf.lf_device_status(reset=True)
    gm_bad = gm.clone()
    gm_bad[1, :w + 1] = 0.0  # sample 1: more than w leading globals
    out = _run(t, lm, gm_bad, w)
    assert lf.lf_device_status(reset=True) == 5
    assert torch.all(out[1] == 0)
    gm_bad = gm.clone()
    gm_bad[0, 300] = 0.0     # sample 0: a global token after the prefix
    _run(t, lm, gm_bad, w)
    assert lf.lf_device_status(reset=True) == 6
    _run(t, lm, gm, w)
    assert lf.lf_device_status(reset=True) == 0


def test_attention_repeated_calls_identical():
    """The split-KV counters are left clean: repeated calls give the same bits."""
    wl, t, lm, gm = inputs.workload_inputs(2)
    dev = {n: t[n].cuda() for n in inputs.NAMES}
    lmc, gmc = lm.cuda(), gm.cuda()
    a = lf.lf_attention_forward(*[dev[n] for n in inputs.NAMES], lmc, gmc, wl.w)
    for _ in range(3):
        b = lf.lf_attention_forward(*[dev[n] for n in inputs.NAMES], lmc, gmc, wl.w)
        assert torch.equal(a, b)


# ---------------------------------------------------------------- partition and attention in one call

def _run_idx(t, lm, gm, w):
    dev = {n: t[n].cuda() for n in inputs.NAMES}
    out, idx, nums = lf.lf_attention_forward_idx(*[dev[n] for n in inputs.NAMES], lm.cuda(), gm.cuda(), w)
    torch.cuda.synchronize()
    return out, idx, nums


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B%dH%dL%dw%d" % s[:4])
def test_attention_idx_small(dtype, shape):
    """lf_attention_forward_idx: the same output bits as lf_attention_forward
    and the partition bit-exact against the oracle (for fp16 / bf16 the
    partition is computed inside the attention kernel's launch)."""
    B, H, L, w, g, pad = shape
    t = inputs.attention_inputs(B, H, L, dtype, seed=31 + L)
    lm, gm = inputs.masks(B, L, g, pad)
    lf.lf_device_status(reset=True)
    out, idx, nums = _run_idx(t, lm, gm, w)
    assert lf.lf_device_status(reset=True) == 0
    assert torch.equal(out, _run(t, lm, gm, w))
    e_idx, e_nums, st = oracle.global_partition(gm.numpy(), w)
    assert st == 0
    assert np.array_equal(idx.cpu().numpy(), e_idx)
    assert np.array_equal(nums.cpu().numpy(), e_nums)


@pytest.mark.parametrize("dtype", ["f32", "f16"])
@pytest.mark.parametrize("seed", range(6))
def test_attention_idx_partition_bit_exact(seed, dtype):
    """Random prefix lengths (0..w), batch sizes and window widths, among them
    L not a multiple of 4: the in-kernel partition against the oracle."""
    rng = np.random.default_rng(100 + seed)
    B, w = int(rng.integers(1, 6)), int(rng.choice([3, 64, 256]))
    L = w * int(rng.integers(2, 12))
    gm = np.full((B, L), -10000.0, np.float32)
    for b in range(B):
        gm[b, : int(rng.integers(0, w + 1))] = 0.0
    t = inputs.attention_inputs(B, 1, L, dtype, seed=seed)
    lm = torch.ones(B, L, dtype=torch.float32)
    lf.lf_device_status(reset=True)
    _, idx, nums = _run_idx(t, lm, torch.from_numpy(gm), w)
    assert lf.lf_device_status(reset=True) == 0
    e_idx, e_nums, st = oracle.global_partition(gm, w)
    assert np.array_equal(idx.cpu().numpy(), e_idx)
    assert np.array_equal(nums.cpu().numpy(), e_nums)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("case", ["not_prefix", "too_many", "scatter"])
def test_attention_idx_content_errors(case, dtype):
    """Masks that break the prefix rules: the combined call records the same
    status as lf_init_global_idx followed by lf_attention_forward, writes the
    oracle's partition and the same output."""
    B, H, L, w = 3, 2, 1024, 128
    gm = np.full((B, L), -10000.0, np.float32)
    gm[0, :5] = 0.0
    if case == "not_prefix":
        gm[1, 700] = 0.0
    elif case == "too_many":
        gm[1, :w + 1] = 0.0
    else:
        gm[2, ::7] = 0.0
    t = inputs.attention_inputs(B, H, L, dtype, seed=8)
    lm = torch.ones(B, L, dtype=torch.float32)
    g = torch.from_numpy(gm)
    lf.lf_device_status(reset=True)
    lf.lf_init_global_idx(g.cuda(), w, sync=False)
    ref_out = _run(t, lm, g, w)
    st_sep = lf.lf_device_status(reset=True)
    out, idx, nums = _run_idx(t, lm, g, w)
    st = lf.lf_device_status(reset=True)
    e_idx, e_nums, e_st = oracle.global_partition(gm, w)
    assert st == st_sep and st != 0
    assert np.array_equal(idx.cpu().numpy(), e_idx)
    assert np.array_equal(nums.cpu().numpy(), e_nums)
    assert torch.equal(out, ref_out)


def test_attention_idx_workload2():
    """The benchmark's step (workload 2): one launch gives the attention
    output of lf_attention_forward bit for bit and the oracle's partition."""
    wl, t, lm, gm = inputs.workload_inputs(2)
    out, idx, nums = _run_idx(t, lm, gm, wl.w)
    assert lf.lf_device_status(reset=True) == 0
    assert torch.equal(out, _run(t, lm, gm, wl.w))
    e_idx, e_nums, _ = oracle.global_partition(gm.numpy(), wl.w)
    assert np.array_equal(idx.cpu().numpy(), e_idx)
    assert np.array_equal(nums.cpu().numpy(), e_nums)


# ---------------------------------------------------------------- the five workloads

def test_workload1_full_parity():
    wl, t, lm, gm = inputs.workload_inputs(1)
    _compare_full(t, lm, gm, wl.w, TDT[wl.dtype])


@pytest.mark.parametrize("cid", [2, 3, 4])
def test_workload_full_parity(cid):
    """Workloads 2 (fp16, 4096 tokens, 300 padded), 3 (bf16, four samples
    with their own g and padding) and 4 (fp16, 16384 tokens) at full size:
    every element of the output against the oracle, in the launch
    configuration the benchmark times."""
    wl, t, lm, gm = inputs.workload_inputs(cid)
    out = _run(t, lm, gm, wl.w).float().cpu().numpy().reshape(wl.B, wl.L, wl.H, 64)
    ref = oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, wl.w)
    err = float(np.abs(out - ref).max())
    print("workload %d: max abs err %.3e over %d elements" % (cid, err, out.size))
    assert err <= TOL[TDT[wl.dtype]], "max abs err %g" % err
    pad = lm.numpy() != 1.0
    assert np.all(out[pad] == 0.0)
