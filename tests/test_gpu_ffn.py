"""GPU parity of the GELU FFN (step 6 of the layer before its LayerNorm)
through lf_gelu_ffn_forward: the fused kernel (intermediate kept on chip,
clusters of 1, 2 and 4 CTAs) and the two-GEMM path, each against the float64
oracle, and against each other bit for bit (both sum over D and over F in
the same order); the layer with either path selected; error cases."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_banded_b200 import build, inputs, lf
from tests._util import TOL

pytestmark = pytest.mark.gpu

TDT = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    lf.lib()
    lf.lf_device_status(reset=True)
    yield
    lf.lf_set_ffn_path("auto")


def _round_to(dtype):
    def rnd(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).double().numpy()
    return rnd


def _ffn_inputs(M, D, F, dtype, seed):
    """h ~ N(0, 1) (a LayerNorm output), weights ~ N(0, 0.02^2) as the layer
    inputs, biases ~ N(0, 0.1^2)."""
    gen = torch.Generator().manual_seed(seed)
    dt = TDT[dtype]
    h = torch.randn(M, D, generator=gen).to(dt)
    W1 = (torch.randn(F, D, generator=gen) * 0.02).to(dt)
    b1 = (torch.randn(F, generator=gen) * 0.1).to(dt)
    W2 = (torch.randn(D, F, generator=gen) * 0.02).to(dt)
    b2 = (torch.randn(D, generator=gen) * 0.1).to(dt)
    return h, W1, b1, W2, b2


def _oracle(h, W1, b1, W2, b2, dtype):
    return oracle.gelu_ffn(h, W1.double().numpy().T, b1, W2.double().numpy().T, b2,
                           round_stored=_round_to(TDT[dtype]))


# (rows, D, F): clusters of 1 (D <= 256), 2 (D <= 512) and 4 CTAs, output
# quarters of 160 / 192 / 224 / 256 columns, ragged last row tiles, and a
# two-GEMM launch whose last partial round of tiles is split in halves
SHAPES = [
    (300, 128, 256),
    (200, 256, 512),
    (257, 384, 512),
    (384, 512, 1024),
    (130, 640, 512),
    (260, 768, 1024),
    (129, 896, 512),
    (513, 1024, 2048),
    (8192, 640, 512),   # the second GEMM's 192 tiles: its last 44 run as 128-wide halves, ragged last N tile among them
]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("M,D,F", SHAPES)
def test_ffn_parity_both_paths(dtype, M, D, F):
    h, W1, b1, W2, b2 = _ffn_inputs(M, D, F, dtype, seed=M + D + F)
    dev = [t.cuda() for t in (h, W1, b1, W2, b2)]
    zf = lf.lf_gelu_ffn_forward(*dev, path="fused")
    zu = lf.lf_gelu_ffn_forward(*dev, path="unfused")
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
    ref = _oracle(h, W1, b1, W2, b2, dtype)
    for name, z in (("fused", zf), ("unfused", zu)):
        got = z.cpu().double().numpy()
        assert np.isfinite(got).all()
        err = float(np.abs(got - ref).max())
        print("ffn %s %s M%d D%d F%d: max abs err %.3e" % (name, dtype, M, D, F, err))
        assert err <= TOL[TDT[dtype]], (name, err)
    assert torch.equal(zf, zu), "fused and unfused differ: max %g" % (zf - zu).abs().max().item()


def test_ffn_workload5_full_parity():
    """The FFN of the headline encoder layer (4096 rows, D 1024, F 4096; the
    layer's own weights), every element against the oracle."""
    wl, x, W, lm, gm = inputs.layer_inputs(5)
    gen = torch.Generator().manual_seed(505)
    h = torch.randn(4096, 1024, generator=gen).to(torch.float16)
    dev = [t.cuda() for t in (h, W["W_1"], W["b_1"], W["W_2"], W["b_2"])]
    zf = lf.lf_gelu_ffn_forward(*dev, path="fused")
    zu = lf.lf_gelu_ffn_forward(*dev, path="unfused")
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
    ref = _oracle(h, W["W_1"], W["b_1"], W["W_2"], W["b_2"], "f16")
    err = float(np.abs(zf.cpu().double().numpy() - ref).max())
    print("ffn workload 5 fused: max abs err %.3e" % err)
    assert err <= TOL[torch.float16]
    assert torch.equal(zf, zu)


@pytest.mark.parametrize("dtype,hidden,ffn,L", [("f16", 512, 1024, 1024), ("bf16", 512, 1024, 1024),
                                                 ("f16", 1024, 4096, 4096)])
def test_layer_ffn_paths(dtype, hidden, ffn, L):
    """The encoder layer (a 512-wide one, and workload 5's shape) with either
    FFN path selected matches the layer oracle; auto takes the two GEMMs at
    these widths.  (With the two GEMMs the LayerNorm runs in the second
    GEMM's epilogue, with the fused FFN in its own kernel, so the two paths
    round differently.)"""
    wl, x, W, lm, gm = inputs.layer_inputs(5, hidden=hidden, ffn=ffn, B=1, L=L, dtype=dtype, g=[64], pad=[17],
                                           seed=91, bias_scale=0.1, ln_scale=0.1)
    dev = {k: v.cuda() for k, v in W.items()}
    outs = {}
    for path in ("unfused", "fused", "auto"):
        lf.lf_set_ffn_path(path)
        assert lf.lf_get_ffn_path() == path
        outs[path] = lf.lf_encoder_layer_forward(x.cuda(), lm.cuda(), gm.cuda(), dev, hidden // 64, 256, 0.125,
                                                 1e-5)
    lf.lf_set_ffn_path("auto")
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
    assert torch.equal(outs["auto"], outs["unfused"])
    o = {k: np.swapaxes(v.double().numpy(), -1, -2) if k in ("W_qkv_kgvg", "W_qg", "W_o", "W_1", "W_2")
         else v.double().numpy() for k, v in W.items()}
    ref = oracle.encoder_layer(x, lm, gm, o, hidden // 64, 256, 0.125, 1e-5,
                               round_attention_inputs=_round_to(TDT[dtype]), round_stored=_round_to(TDT[dtype]))
    for path in ("unfused", "fused"):
        got = outs[path].float().cpu().numpy()
        err = float((np.abs(got - ref) / np.maximum(1.0, np.abs(ref))).max())
        print("layer %s ffn=%s: max scaled err %.3e" % (dtype, path, err))
        assert err <= TOL[TDT[dtype]], (path, err)


def test_ffn_errors():
    h, W1, b1, W2, b2 = [t.cuda() for t in _ffn_inputs(256, 1024, 640, "f16", seed=3)]
    # F = 640 is not a multiple of 4 * 128: the fused path does not take it
    with pytest.raises(lf.LFError) as e:
        lf.lf_gelu_ffn_forward(h, W1, b1, W2, b2, path="fused")
    assert e.value.status == 2
    # ... while auto runs it unfused (and needs the workspace for that)
    assert lf.lf_gelu_ffn_workspace_bytes(256, 1024, 640, torch.float16, "auto") == 256 * 640 * 2
    z = lf.lf_gelu_ffn_forward(h, W1, b1, W2, b2, path="auto")
    ref = _oracle(h.cpu(), W1.cpu(), b1.cpu(), W2.cpu(), b2.cpu(), "f16")
    assert float(np.abs(z.cpu().double().numpy() - ref).max()) <= TOL[torch.float16]
    small = torch.empty(256 * 640 * 2 - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(lf.LFError) as e:
        lf.lf_gelu_ffn_forward(h, W1, b1, W2, b2, path="unfused", workspace=small)
    assert e.value.status == 12
    # the fused path needs no workspace
    h2, W12, b12, W22, b22 = [t.cuda() for t in _ffn_inputs(256, 1024, 2048, "f16", seed=4)]
    assert lf.lf_gelu_ffn_workspace_bytes(256, 1024, 2048, torch.float16, "fused") == 0
    lf.lf_gelu_ffn_forward(h2, W12, b12, W22, b22, path="fused")
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
