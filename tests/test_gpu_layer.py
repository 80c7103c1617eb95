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
