"""Pins of the float64 oracle against facts that do not come from the oracle.

"FTL" = the page "FasterTransformer Longformer 推理加速实践：PyTorch 集成、
输入约束与端到端性能解析".

Each pin targets a plausible mistake:
  * hand-worked golden files          -> key-set membership, duplicate global
                                         keys, padding bias, scale, partition order
  * dense L x L brute force           -> any index/sign/transposition slip over
                                         many random shapes, padding and g
  * q = 0 closed form                 -> the key set of every row (means)
  * library SDPA special cases        -> scale, softmax, operand order, and that
                                         global rows use qg/kg/vg
  * invariants                        -> rows sum to one, padded rows zero,
                                         no dependence on keys outside the set
  * layer pieces vs torch/scipy       -> LayerNorm, GELU, residual wiring
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import softmax
from scipy.stats import norm

import oracle
from sparse_attention_banded_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden_cases(name):
    cases, cur = [], None
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0] == "case":
                cur = {"name": tok[1], "samples": []}
                for kv in tok[2:]:
                    k, v = kv.split("=")
                    cur[k] = int(v)
                cases.append(cur)
            elif tok[0] == "mask":
                cur["samples"].append({"mask": [float(x) for x in tok[1:]]})
            elif tok[0] == "idx":
                cur["samples"][-1]["idx"] = [int(x) for x in tok[1:]]
            elif tok[0] == "num":
                cur["samples"][-1]["num"] = int(tok[1])
            elif tok[0] == "status":
                cur["status"] = int(tok[1])
    return cases


def _golden_kv(name):
    d = {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            d[tok[0]] = [float(x) for x in tok[1:]]
    return d


# ---------------------------------------------------------------- partition

@pytest.mark.parametrize("case", _golden_cases("global_partition.txt"), ids=lambda c: c["name"])
def test_partition_golden(case):
    gm = np.array([s["mask"] for s in case["samples"]], dtype=np.float32)
    idx, nums, st = oracle.global_partition(gm, case["w"])
    assert st == case["status"]
    for b, s in enumerate(case["samples"]):
        assert idx[b].tolist() == s["idx"]
        assert nums[b] == s["num"]


def _partition_brute(gm_row):
    sel = [j for j, x in enumerate(gm_row) if x == 0.0]
    rej = [j for j, x in enumerate(gm_row) if x != 0.0]
    return sel + rej[::-1], len(sel)


@pytest.mark.parametrize("seed", range(20))
def test_partition_brute_force(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 5))
    w = int(rng.integers(1, 9))
    L = w * int(rng.integers(2, 6))
    gm = np.full((B, L), -10000.0, np.float32)
    expect_status = 0
    for b in range(B):
        kind = rng.integers(0, 3)
        if kind == 0:  # valid prefix
            gm[b, : int(rng.integers(0, w + 1))] = 0.0
        elif kind == 1:  # random scatter
            gm[b, rng.random(L) < 0.3] = 0.0
        else:  # prefix longer than w
            gm[b, : min(L, w + 1 + int(rng.integers(0, 3)))] = 0.0
    for b in range(B):
        g = int((gm[b] == 0.0).sum())
        prefix = all(gm[b, :g] == 0.0)
        st = 6 if not prefix else (5 if g > w else 0)
        if st and not expect_status:
            expect_status = st
    idx, nums, st = oracle.global_partition(gm, w)
    assert st == expect_status
    for b in range(B):
        e_idx, e_num = _partition_brute(gm[b].tolist())
        assert idx[b].tolist() == e_idx and nums[b] == e_num


# ---------------------------------------------------------------- attention

def _golden_attention(path, build):
    g = _golden_kv(path)
    L, w = int(g["L"][0]), int(g["w"][0])
    t, lm, gm = build(L, g)
    out = oracle.attention(*t, lm, gm, w)
    np.testing.assert_allclose(out[0, :, 0, 0], np.array(g["out0"]), rtol=0, atol=1e-12)
    assert np.all(out[0, :, 0, 1:] == 0.0)


def test_attention_golden_uniform():
    def build(L, g):
        gcount, pad = int(g["g"][0]), int(g["pad"][0])
        z = np.zeros((1, 1, L, 64))
        v = np.zeros((1, 1, L, 64))
        v[0, 0, :, 0] = np.arange(L) + 1
        lm, gm = inputs.masks(1, L, [gcount], [pad])
        return (z, z, v, z, z, v.copy()), lm, gm
    _golden_attention("attention_uniform.txt", build)


def test_attention_golden_weighted():
    def build(L, g):
        q = np.zeros((1, 1, L, 64)); q[0, 0, :, 0] = 8.0
        k = np.zeros((1, 1, L, 64)); k[0, 0, :, 0] = np.log(np.arange(L) + 1.0)
        v = np.zeros((1, 1, L, 64)); v[0, 0, :, 0] = np.arange(L)
        lm, gm = inputs.masks(1, L, [0], [0])
        return (q, k, v, q.copy(), k.copy(), v.copy()), lm, gm
    _golden_attention("attention_weighted.txt", build)


def dense_reference(t, lm, gm, w, scale=0.125):
    """Dense L x L attention with an explicit -inf mask built row by row from
    the set definition; softmax from scipy.  Returns [B, L, H, 64]."""
    q, k, v, qg, kg, vg = [np.asarray(x, dtype=np.float64) for x in t]
    B, H, L, _ = q.shape
    out = np.zeros((B, L, H, 64))
    for b in range(B):
        is_global = (gm[b] == 0.0)
        lb = np.where(lm[b] == 1.0, 0.0, -10000.0)
        allowed = np.zeros((L, L), dtype=bool)
        for i in range(L):
            for j in range(L):
                allowed[i, j] = abs(i - j) <= w or is_global[j]
        colbias = np.where(is_global, gm[b].astype(np.float64), 0.0)
        for h in range(H):
            s_loc = scale * q[b, h] @ k[b, h].T + lb[None, :] + colbias[None, :]
            s_loc = np.where(allowed, s_loc, -np.inf)
            o_loc = softmax(s_loc, axis=1) @ v[b, h]
            s_glb = scale * qg[b, h] @ kg[b, h].T + lb[None, :]
            o_glb = softmax(s_glb, axis=1) @ vg[b, h]
            rows = np.where(is_global[:, None], o_glb, o_loc)
            rows[lb != 0.0] = 0.0
            out[b, :, h, :] = rows
    return out


def _random_case(rng, dtype="f32"):
    w = int(rng.choice([2, 4, 8, 16, 32]))
    L = w * int(rng.integers(2, max(3, 64 // w) + 1))
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
    g = [int(rng.integers(0, w + 1)) for _ in range(B)]
    pad = [int(rng.integers(0, L // 2)) for _ in range(B)]
    t = inputs.attention_inputs(B, H, L, dtype, int(rng.integers(1 << 30)))
    lm, gm = inputs.masks(B, L, g, pad)
    return [t[n] for n in inputs.NAMES], lm.numpy(), gm.numpy(), w


@pytest.mark.parametrize("seed", range(30))
def test_attention_matches_dense_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    t, lm, gm, w = _random_case(rng)
    got = oracle.attention(*t, lm, gm, w)
    want = dense_reference(t, lm, gm, w)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(10))
def test_attention_q_zero_closed_form(seed):
    """q = qg = 0: every score is its padding bias, so an unpadded row is the
    mean of v over its unpadded key set -- computed here with Python sets."""
    rng = np.random.default_rng(200 + seed)
    t, lm, gm, w = _random_case(rng)
    q, k, v, qg, kg, vg = [x.double().numpy() for x in t]
    q[:] = 0; qg[:] = 0
    out = oracle.attention(q, k, v, qg, kg, vg, lm, gm, w)
    B, H, L, _ = q.shape
    for b in range(B):
        g = int((gm[b] == 0).sum())
        valid = {j for j in range(L) if lm[b, j] == 1.0}
        for i in range(L):
            if i not in valid:
                assert np.all(out[b, i] == 0.0)
                continue
            if i < g:
                keys, vals = set(range(L)), vg
            else:
                keys = set(range(max(0, i - w), min(L - 1, i + w) + 1)) | set(range(g))
                vals = v
            keys = sorted(keys & valid)
            for h in range(H):
                np.testing.assert_allclose(out[b, i, h], vals[b, h, keys].mean(axis=0), atol=1e-12)


def test_attention_special_case_matches_library_sdpa():
    """L = 2w, g = 0, no padding: row w sees every key, so it equals plain
    dense attention (torch SDPA, default scale 1/sqrt(64)); with g > 0 the
    global rows equal unmasked SDPA on qg/kg/vg."""
    B, H, w = 1, 2, 16
    L = 2 * w
    t = inputs.attention_inputs(B, H, L, "f32", 7)
    lm, gm = inputs.masks(B, L, [0], [0])
    args = [t[n] for n in inputs.NAMES]
    out = oracle.attention(*args, lm, gm, w)
    sd = torch.nn.functional.scaled_dot_product_attention(
        t["q"].double(), t["k"].double(), t["v"].double())
    np.testing.assert_allclose(out[0, w], sd[0, :, w].numpy(), atol=1e-12)
    lm, gm = inputs.masks(B, L, [5], [0])
    out = oracle.attention(*args, lm, gm, w)
    sdg = torch.nn.functional.scaled_dot_product_attention(
        t["qg"].double(), t["kg"].double(), t["vg"].double())
    for i in range(5):
        np.testing.assert_allclose(out[0, i], sdg[0, :, i].numpy(), atol=1e-12)
    # and a local row that sees everything (row w) still uses q/k/v
    np.testing.assert_allclose(out[0, w], sd[0, :, w].numpy(), atol=1e-12)


@pytest.mark.parametrize("seed", range(5))
def test_attention_invariants(seed):
    rng = np.random.default_rng(300 + seed)
    t, lm, gm, w = _random_case(rng)
    q, k, v, qg, kg, vg = [x.double().numpy() for x in t]
    ones = np.ones_like(v)
    out = oracle.attention(q, k, ones, qg, kg, ones, lm, gm, w)
    B, H, L, _ = q.shape
    for b in range(B):
        for i in range(L):
            if lm[b, i] == 1.0:
                np.testing.assert_allclose(out[b, i], 1.0, atol=1e-12)
            else:
                assert np.all(out[b, i] == 0.0)
    # keys outside a row's set do not matter: perturb one row's outside keys
    base = oracle.attention(q, k, v, qg, kg, vg, lm, gm, w)
    b, h = 0, 0
    g = int((gm[b] == 0).sum())
    i = L - 1
    if i >= g:
        outside = [j for j in range(L) if abs(i - j) > w and j >= g]
        k2, v2 = k.copy(), v.copy()
        k2[b, h, outside] += rng.normal(size=(len(outside), 64))
        v2[b, h, outside] += rng.normal(size=(len(outside), 64))
        pert = oracle.attention(q, k2, v2, qg, kg, vg, lm, gm, w)
        assert np.array_equal(pert[b, i, h], base[b, i, h])


def test_attention_rows_matches_full():
    rng = np.random.default_rng(5)
    t, lm, gm, w = _random_case(rng)
    full = oracle.attention(*t, lm, gm, w)
    B, L, H, _ = full.shape
    rows = np.array([[b, h, i] for b in range(B) for h in range(H) for i in range(0, L, 3)])
    sub = oracle.attention_rows(*t, lm, gm, w, rows)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(sub[r], full[b, i, h])


@pytest.mark.parametrize("B,H,L,w,status", [
    (1, 1, 10, 4, 3), (1, 1, 4, 4, 4), (0, 1, 8, 4, 2), (1, 1, 8, 0, 2)])
def test_oracle_shape_errors(B, H, L, w, status):
    assert oracle.check_shape(B, H, L, w) == status


def test_oracle_rejects_bad_globals():
    t = inputs.attention_inputs(1, 1, 16, "f32", 1)
    lm, gm = inputs.masks(1, 16, [0], [0])
    gm[0, 3] = 0.0
    with pytest.raises(oracle.OracleError) as e:
        oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, 4)
    assert e.value.status == 6
    lm, gm = inputs.masks(1, 16, [5], [0])
    with pytest.raises(oracle.OracleError) as e:
        oracle.attention(*[t[n] for n in inputs.NAMES], lm, gm, 4)
    assert e.value.status == 5


# ------------------------------------------------- global tokens at any position

def _scattered_masks(rng, B, L, w, pad_global=True):
    """Masks with g_b <= w global tokens at random positions (the HuggingFace
    arrangement of FTL §使用前提 item 4) and random padded positions, some of
    them on global tokens."""
    lm = np.ones((B, L), np.float32)
    gm = np.full((B, L), -10000.0, np.float32)
    for b in range(B):
        g = int(rng.integers(0, w + 1))
        gm[b, rng.choice(L, size=g, replace=False)] = 0.0
        pad = int(rng.integers(0, L // 2))
        if pad:
            lm[b, L - pad:] = 0.0
        if pad_global and rng.random() < 0.5:
            lm[b, rng.integers(0, L)] = 0.0
    return lm, gm


def test_any_globals_golden():
    g = _golden_kv("attention_any_globals.txt")
    L, w = int(g["L"][0]), int(g["w"][0])
    z = np.zeros((1, 1, L, 64))
    v = np.zeros((1, 1, L, 64)); v[0, 0, :, 0] = np.arange(L) + 1
    vg = np.zeros((1, 1, L, 64)); vg[0, 0, :, 0] = np.arange(L) + 101
    for case in ("a", "b"):
        lm = np.ones((1, L), np.float32)
        gm = np.full((1, L), -10000.0, np.float32)
        gm[0, [int(x) for x in g[case + "_globals"]]] = 0.0
        lm[0, [int(x) for x in g[case + "_padded"]]] = 0.0
        out = oracle.attention(z, z, v, z, z, vg, lm, gm, w, any_pos=True)
        np.testing.assert_allclose(out[0, :, 0, 0], np.array(g[case + "_out0"]), rtol=0, atol=1e-12)
        assert np.all(out[0, :, 0, 1:] == 0.0)


@pytest.mark.parametrize("seed", range(30))
def test_any_globals_match_dense_brute_force(seed):
    rng = np.random.default_rng(700 + seed)
    w = int(rng.choice([2, 4, 8, 16, 32]))
    L = w * int(rng.integers(2, max(3, 64 // w) + 1))
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
    lm, gm = _scattered_masks(rng, B, L, w)
    t = inputs.attention_inputs(B, H, L, "f32", int(rng.integers(1 << 30)))
    t = [t[n] for n in inputs.NAMES]
    got = oracle.attention(*t, lm, gm, w, any_pos=True)
    want = dense_reference(t, lm, gm, w)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_any_globals_q_zero_closed_form(seed):
    """q = qg = 0: an unpadded row is the mean of v (vg for a global row)
    over its unpadded key set, the sets built here with Python set algebra."""
    rng = np.random.default_rng(800 + seed)
    w = int(rng.choice([4, 8, 16]))
    L = w * int(rng.integers(2, 5))
    B, H = 2, 2
    lm, gm = _scattered_masks(rng, B, L, w)
    t = inputs.attention_inputs(B, H, L, "f32", seed)
    q, k, v, qg, kg, vg = [t[n].double().numpy() for n in inputs.NAMES]
    q[:] = 0; qg[:] = 0
    out = oracle.attention(q, k, v, qg, kg, vg, lm, gm, w, any_pos=True)
    for b in range(B):
        G = {j for j in range(L) if gm[b, j] == 0.0}
        valid = {j for j in range(L) if lm[b, j] == 1.0}
        for i in range(L):
            if i not in valid:
                assert np.all(out[b, i] == 0.0)
                continue
            if i in G:
                keys, vals = set(range(L)), vg
            else:
                keys, vals = set(range(max(0, i - w), min(L - 1, i + w) + 1)) | G, v
            keys = sorted(keys & valid)
            for h in range(H):
                np.testing.assert_allclose(out[b, i, h], vals[b, h, keys].mean(axis=0), atol=1e-12)


@pytest.mark.parametrize("seed", range(5))
def test_any_globals_prefix_case_is_the_prefix_oracle(seed):
    """With the global tokens at the front both definitions are the same
    computation, bit for bit."""
    rng = np.random.default_rng(900 + seed)
    t, lm, gm, w = _random_case(rng)
    a = oracle.attention(*t, lm, gm, w)
    b = oracle.attention(*t, lm, gm, w, any_pos=True)
    assert np.array_equal(a, b)


def test_any_globals_invariants_and_errors():
    rng = np.random.default_rng(11)
    B, H, L, w = 2, 2, 48, 8
    lm, gm = _scattered_masks(rng, B, L, w)
    t = inputs.attention_inputs(B, H, L, "f32", 3)
    q, k, v, qg, kg, vg = [t[n].double().numpy() for n in inputs.NAMES]
    ones = np.ones_like(v)
    out = oracle.attention(q, k, ones, qg, kg, ones, lm, gm, w, any_pos=True)
    for b in range(B):
        for i in range(L):
            if lm[b, i] == 1.0:
                np.testing.assert_allclose(out[b, i], 1.0, atol=1e-12)
            else:
                assert np.all(out[b, i] == 0.0)
    # keys outside a local row's set (outside the window and not global) do not matter
    base = oracle.attention(q, k, v, qg, kg, vg, lm, gm, w, any_pos=True)
    b, h = 0, 1
    G = set(np.flatnonzero(gm[b] == 0.0).tolist())
    i = next(i for i in range(L) if i not in G)
    outside = [j for j in range(L) if abs(i - j) > w and j not in G]
    k2, v2 = k.copy(), v.copy()
    k2[b, h, outside] += rng.normal(size=(len(outside), 64))
    v2[b, h, outside] += rng.normal(size=(len(outside), 64))
    pert = oracle.attention(q, k2, v2, qg, kg, vg, lm, gm, w, any_pos=True)
    assert np.array_equal(pert[b, i, h], base[b, i, h])
    # more than w global tokens is still an error; scattered ones are not
    gm2 = np.full((1, 16), -10000.0, np.float32); gm2[0, [3, 9, 14]] = 0.0
    t1 = inputs.attention_inputs(1, 1, 16, "f32", 1)
    args = [t1[n] for n in inputs.NAMES]
    oracle.attention(*args, np.ones((1, 16), np.float32), gm2, 4, any_pos=True)
    gm2[0, [1, 5]] = 0.0
    with pytest.raises(oracle.OracleError) as e:
        oracle.attention(*args, np.ones((1, 16), np.float32), gm2, 4, any_pos=True)
    assert e.value.status == 5


@pytest.mark.parametrize("seed", range(10))
def test_any_globals_partition_brute_force(seed):
    rng = np.random.default_rng(1000 + seed)
    B, w = 3, int(rng.integers(1, 9))
    L = w * int(rng.integers(2, 6))
    gm = np.full((B, L), -10000.0, np.float32)
    for b in range(B):
        gm[b, rng.random(L) < rng.random() * 0.5] = 0.0
    idx, nums, st = oracle.global_partition(gm, w, any_pos=True)
    expect = 0
    for b in range(B):
        e_idx, e_num = _partition_brute(gm[b].tolist())
        assert idx[b].tolist() == e_idx and nums[b] == e_num
        if e_num > w and not expect:
            expect = 5
    assert st == expect


def test_any_globals_rows_match_full():
    rng = np.random.default_rng(12)
    lm, gm = _scattered_masks(rng, 2, 32, 8)
    t = inputs.attention_inputs(2, 2, 32, "f32", 4)
    t = [t[n] for n in inputs.NAMES]
    full = oracle.attention(*t, lm, gm, 8, any_pos=True)
    rows = np.array([[b, h, i] for b in range(2) for h in range(2) for i in range(32)])
    sub = oracle.attention_rows(*t, lm, gm, 8, rows, any_pos=True)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(sub[r], full[b, i, h])


# ---------------------------------------------------------------- encoder layer

def test_gelu_closed_values():
    x = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(oracle.gelu(x), x * norm.cdf(x), atol=1e-14)
    assert oracle.gelu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(oracle.gelu(np.array([1.0]))[0], 0.8413447460685429, atol=1e-15)
    np.testing.assert_allclose(oracle.gelu(x) - oracle.gelu(-x), x, atol=1e-14)


def test_layer_norm_moments_and_library():
    rng = np.random.default_rng(0)
    z = rng.normal(size=(7, 64)) * 3 + 1
    y = oracle.layer_norm(z, np.ones(64), np.zeros(64), 1e-5)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=1), 1 - 1e-5 / (z.var(axis=1) + 1e-5), atol=1e-9)
    gam, bet = rng.normal(size=64), rng.normal(size=64)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(z), (64,), torch.from_numpy(gam),
                                         torch.from_numpy(bet), 1e-5).numpy()
    np.testing.assert_allclose(oracle.layer_norm(z, gam, bet, 1e-5), ref, atol=1e-12)


def test_encoder_layer_matches_torch_composition():
    """Small layer (H=2, hidden 128, FFN 256): the oracle's wiring of
    projections, attention, out-proj + residual + LN and GELU-FFN + residual +
    LN against torch float64 library ops (linear, layer_norm, gelu)."""
    rng = np.random.default_rng(1)
    B, H, L, w, D, F = 1, 2, 32, 8, 128, 256
    x = rng.normal(size=(B, L, D))
    W = {"W_qkv_kgvg": rng.normal(size=(5, D, D)) * 0.05, "b_qkv_kgvg": rng.normal(size=(5, D)) * 0.1,
         "W_qg": rng.normal(size=(D, D)) * 0.05, "b_qg": rng.normal(size=D) * 0.1,
         "W_o": rng.normal(size=(D, D)) * 0.05, "b_o": rng.normal(size=D) * 0.1,
         "ln1_gamma": 1 + rng.normal(size=D) * 0.1, "ln1_beta": rng.normal(size=D) * 0.1,
         "W_1": rng.normal(size=(D, F)) * 0.05, "b_1": rng.normal(size=F) * 0.1,
         "W_2": rng.normal(size=(F, D)) * 0.05, "b_2": rng.normal(size=D) * 0.1,
         "ln2_gamma": 1 + rng.normal(size=D) * 0.1, "ln2_beta": rng.normal(size=D) * 0.1}
    lm, gm = inputs.masks(B, L, [3], [4])
    got = oracle.encoder_layer(x, lm, gm, W, H, w, 0.125, 1e-5)

    T = {k: torch.from_numpy(np.asarray(v)) for k, v in W.items()}
    X = torch.from_numpy(x)
    F_ = torch.nn.functional

    def heads(y):
        return y.view(B, L, H, 64).permute(0, 2, 1, 3).contiguous()
    proj = [heads(F_.linear(X, T["W_qkv_kgvg"][n].T, T["b_qkv_kgvg"][n])) for n in range(5)]
    qg = heads(F_.linear(X, T["W_qg"].T, T["b_qg"]))
    att = oracle.attention(proj[0], proj[1], proj[2], qg, proj[3], proj[4], lm, gm, w)
    att = torch.from_numpy(att).reshape(B, L, D)
    h = F_.layer_norm(F_.linear(att, T["W_o"].T, T["b_o"]) + X, (D,), T["ln1_gamma"], T["ln1_beta"], 1e-5)
    f = F_.gelu(F_.linear(h, T["W_1"].T, T["b_1"]), approximate="none")
    y = F_.layer_norm(F_.linear(f, T["W_2"].T, T["b_2"]) + h, (D,), T["ln2_gamma"], T["ln2_beta"], 1e-5)
    np.testing.assert_allclose(got, y.numpy(), atol=1e-10)


def test_gelu_ffn_matches_torch_and_rounds_only_the_intermediate():
    """The FFN oracle (step 6 before LN) against torch float64 library ops
    (linear, gelu with its own erf), and its rounding hook: applied to the
    intermediate only (rounding to fp16 changes the result, and equals
    rounding that intermediate by hand)."""
    rng = np.random.default_rng(5)
    M, D, F = 37, 128, 384
    h = rng.normal(size=(M, D))
    W1, b1 = rng.normal(size=(D, F)) * 0.05, rng.normal(size=F) * 0.1
    W2, b2 = rng.normal(size=(F, D)) * 0.05, rng.normal(size=D) * 0.1
    got = oracle.gelu_ffn(h, W1, b1, W2, b2)
    F_ = torch.nn.functional
    T = [torch.from_numpy(a) for a in (h, W1, b1, W2, b2)]
    ref = F_.linear(F_.gelu(F_.linear(T[0], T[1].T, T[2]), approximate="none"), T[3].T, T[4]) + T[0]
    np.testing.assert_allclose(got, ref.numpy(), atol=1e-12)

    def r16(a):
        return torch.from_numpy(np.ascontiguousarray(a)).half().double().numpy()
    rounded = oracle.gelu_ffn(h, W1, b1, W2, b2, round_stored=r16)
    f = r16(oracle.gelu(h @ W1 + b1))
    np.testing.assert_allclose(rounded, f @ W2 + b2 + h, atol=1e-12)
    assert np.abs(rounded - got).max() > 1e-6


def test_encoder_layer_any_pos_wiring():
    """The layer oracle with global tokens at any position: on prefix masks
    the same bits as the prefix definition, and on scattered masks the same
    composition around oracle.attention(any_pos=True)."""
    rng = np.random.default_rng(2)
    B, H, L, w, D, F = 1, 2, 32, 8, 128, 256
    x = rng.normal(size=(B, L, D))
    W = {"W_qkv_kgvg": rng.normal(size=(5, D, D)) * 0.05, "b_qkv_kgvg": rng.normal(size=(5, D)) * 0.1,
         "W_qg": rng.normal(size=(D, D)) * 0.05, "b_qg": rng.normal(size=D) * 0.1,
         "W_o": rng.normal(size=(D, D)) * 0.05, "b_o": rng.normal(size=D) * 0.1,
         "ln1_gamma": np.ones(D), "ln1_beta": np.zeros(D),
         "W_1": rng.normal(size=(D, F)) * 0.05, "b_1": rng.normal(size=F) * 0.1,
         "W_2": rng.normal(size=(F, D)) * 0.05, "b_2": rng.normal(size=D) * 0.1,
         "ln2_gamma": np.ones(D), "ln2_beta": np.zeros(D)}
    lm, gm = inputs.masks(B, L, [3], [4])
    a = oracle.encoder_layer(x, lm, gm, W, H, w, 0.125, 1e-5)
    b = oracle.encoder_layer(x, lm, gm, W, H, w, 0.125, 1e-5, any_pos=True)
    assert np.array_equal(a, b)
    lm2, gm2 = inputs.masks_scattered(B, L, [5], [4], seed=9, padded_globals=1)
    got = oracle.encoder_layer(x, lm2, gm2, W, H, w, 0.125, 1e-5, any_pos=True)
    proj = [oracle.to_heads(x @ W["W_qkv_kgvg"][n] + W["b_qkv_kgvg"][n], H) for n in range(5)]
    qg = oracle.to_heads(x @ W["W_qg"] + W["b_qg"], H)
    att = oracle.attention(proj[0], proj[1], proj[2], qg, proj[3], proj[4], lm2, gm2, w, any_pos=True)
    h = oracle.layer_norm(att.reshape(B, L, D) @ W["W_o"] + W["b_o"] + x, W["ln1_gamma"], W["ln1_beta"], 1e-5)
    y = oracle.layer_norm(oracle.gelu(h @ W["W_1"] + W["b_1"]) @ W["W_2"] + W["b_2"] + h,
                          W["ln2_gamma"], W["ln2_beta"], 1e-5)
    np.testing.assert_allclose(got, y, atol=1e-12)
    # and it differs from treating the same mask as a prefix would (that is an error there)
    with pytest.raises(oracle.OracleError):
        oracle.encoder_layer(x, lm2, gm2, W, H, w, 0.125, 1e-5)


def test_workload_draws_are_stable():
    wl = inputs.workload(3)
    assert len(wl.g) == 4 and all(1 <= g <= 128 for g in wl.g)
    assert all(0 <= p <= 1024 for p in wl.pad)
    assert inputs.workload(3).g == wl.g


# ---------------------------------------------------------------- work counts (host side)

@pytest.mark.parametrize("seed", range(4))
def test_flops_from_masks_brute_force(seed):
    """The benchmark's FLOP count for any masks equals 4*64*H times the sizes
    of the key sets built with Python set algebra, and the prefix formula on
    prefix masks."""
    from sparse_attention_banded_b200 import metrics
    rng = np.random.default_rng(1200 + seed)
    B, H, w = 2, 3, int(rng.choice([4, 8, 16]))
    L = w * int(rng.integers(2, 6))
    lm, gm = _scattered_masks(rng, B, L, w)
    total = 0
    for b in range(B):
        G = {j for j in range(L) if gm[b, j] == 0.0}
        for i in range(L):
            if lm[b, i] != 1.0:
                continue
            total += L if i in G else len(set(range(max(0, i - w), min(L - 1, i + w) + 1)) | G)
    assert metrics.flops_masks(lm, gm, H, w) == 4.0 * 64 * H * total
    g = [int(rng.integers(0, w + 1)) for _ in range(B)]
    pad = [int(rng.integers(0, L)) for _ in range(B)]
    lm2, gm2 = inputs.masks(B, L, g, pad)
    assert metrics.flops_masks(lm2.numpy(), gm2.numpy(), H, w) == metrics.flops(B, H, L, w, g, pad)


def test_scattered_masks_generator():
    lm, gm = inputs.masks_scattered(3, 256, [0, 10, 64], [0, 50, 100], seed=5, padded_globals=2)
    for b, (g, pad) in enumerate([(0, 0), (10, 50), (64, 100)]):
        G = np.flatnonzero(gm[b].numpy() == 0.0)
        assert len(G) == g and (G < 256 - pad).all()
        assert set(np.unique(gm[b].numpy())) <= {0.0, -10000.0}
        assert (lm[b, 256 - pad:] == 0.0).all()
        assert int((lm[b, :256 - pad] == 0.0).sum()) == min(2, g)
