"""GPU parity of the encoder layer (projections, attention, output
projection + residual + LayerNorm, GELU FFN + residual + LayerNorm) against
the float64 oracle, through lf_encoder_layer_forward."""
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


def _oracle_weights(W):
    """nn.Linear layout [out, in] -> the oracle's x @ W convention."""
    o = {k: v.double().cpu().numpy() for k, v in W.items()}
    for k in ("W_qkv_kgvg", "W_qg", "W_o", "W_1", "W_2"):
        o[k] = np.swapaxes(o[k], -1, -2)
    return o


def _round_to(dtype):
    def rnd(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).double().numpy()
    return rnd


def _run_and_compare(x, W, lm, gm, H, w, dtype, rows=None):
    dev = {k: v.cuda() for k, v in W.items()}
    out = lf.lf_encoder_layer_forward(x.cuda(), lm.cuda(), gm.cuda(), dev, H, w, 0.125, 1e-5)
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
    got = out.float().cpu().numpy()
    ref = oracle.encoder_layer(x, lm, gm, _oracle_weights(W), H, w, 0.125, 1e-5,
                               round_attention_inputs=_round_to(dtype), round_stored=_round_to(dtype))
    # The stated bounds (1e-2 fp16, 2e-2 bf16) are for unit-scale outputs; the
    # layer's LayerNorm outputs reach |y| ~ 5, where one bf16 ulp is 0.0156.
    # Bound: |got - ref| <= tol * max(1, |ref|) per element (~5 bf16 or ~10
    # fp16 ulps of the output's magnitude).
    assert np.isfinite(got).all()
    scaled = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
    err = scaled.max()
    assert err <= TOL[dtype], "max scaled err %g (max abs %g)" % (err, np.abs(got - ref).max())
    return err


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("B,H,L,w,ffn,g,pad", [
    (1, 2, 512, 64, 256, [8], [0]),
    (2, 2, 640, 128, 384, [5, 100], [0, 33]),   # ragged last M tile, padding, two samples
    (1, 4, 1024, 256, 512, [64], [17]),
])
def test_layer_small_parity(dtype, B, H, L, w, ffn, g, pad):
    wl, x, W, lm, gm = inputs.layer_inputs(5, hidden=H * 64, ffn=ffn, B=B, L=L, dtype=dtype, g=g, pad=pad,
                                           seed=77 + L, bias_scale=0.1, ln_scale=0.1)
    _run_and_compare(x, W, lm, gm, H, w, TDT[dtype])


def test_workload5_full_parity():
    wl, x, W, lm, gm = inputs.layer_inputs(5)
    _run_and_compare(x, W, lm, gm, wl.H, wl.w, TDT[wl.dtype])


def test_layer_workspace_errors():
    wl, x, W, lm, gm = inputs.layer_inputs(5, hidden=128, ffn=256, B=1, L=512, dtype="f16", g=[4], pad=[0])
    dev = {k: v.cuda() for k, v in W.items()}
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(lf.LFError) as e:
        lf.lf_encoder_layer_forward(x.cuda(), lm.cuda(), gm.cuda(), dev, 2, 64, workspace=small)
    assert e.value.status == 12


# ---------------------------------------------------------------- the encoder stack

def _stack_weights(n, H, ffn, dtype, seed):
    return [inputs.layer_inputs(5, hidden=H * 64, ffn=ffn, B=1, L=512, dtype=dtype, g=[4], pad=[0],
                                seed=seed + j, bias_scale=0.1, ln_scale=0.1)[2] for j in range(n)]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_encoder_stack_equals_chained_layers(dtype):
    """lf_encoder_forward over three layers gives exactly the bits of three
    chained lf_encoder_layer_forward calls."""
    B, H, L, w, ffn = 2, 2, 640, 128, 256
    wl, x, _, lm, gm = inputs.layer_inputs(5, hidden=H * 64, ffn=ffn, B=B, L=L, dtype=dtype, g=[5, 70], pad=[0, 41],
                                           seed=91)
    layers = [{k: v.cuda() for k, v in W.items()} for W in _stack_weights(3, H, ffn, dtype, 300)]
    xd, lmd, gmd = x.cuda(), lm.cuda(), gm.cuda()
    got = lf.lf_encoder_forward(xd, lmd, gmd, layers, H, w)
    ref = xd
    for W in layers:
        ref = lf.lf_encoder_layer_forward(ref, lmd, gmd, W, H, w)
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
    assert torch.equal(got, ref)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_encoder_stack_two_layer_parity(dtype):
    """Two layers against the float64 oracle applied twice, the activation
    between them rounded to the dtype as the kernels store it."""
    B, H, L, w, ffn = 1, 2, 512, 64, 256
    wl, x, _, lm, gm = inputs.layer_inputs(5, hidden=H * 64, ffn=ffn, B=B, L=L, dtype=dtype, g=[8], pad=[19], seed=92)
    Ws = _stack_weights(2, H, ffn, dtype, 400)
    out = lf.lf_encoder_forward(x.cuda(), lm.cuda(), gm.cuda(), [{k: v.cuda() for k, v in W.items()} for W in Ws],
                                H, w)
    torch.cuda.synchronize()
    assert lf.lf_device_status(reset=True) == 0
    got = out.float().cpu().numpy()
    rnd = _round_to(TDT[dtype])
    h = x
    for W in Ws:
        y = oracle.encoder_layer(h, lm, gm, _oracle_weights(W), H, w, 0.125, 1e-5,
                                 round_attention_inputs=rnd, round_stored=rnd)
        h = torch.from_numpy(np.ascontiguousarray(y)).to(TDT[dtype])
    ref = h.double().numpy()
    assert np.isfinite(got).all()
    scaled = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
    assert scaled.max() <= TOL[TDT[dtype]], "max scaled err %g" % scaled.max()
