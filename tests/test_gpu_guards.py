"""Guard canaries around output buffers.

Every entry point writes its output through a view into a larger buffer:
256-byte guard bands before and after it hold 7.0 and must come back
untouched (no write past either end), and the output itself starts as NaN
and must come back finite everywhere (every element written, padded rows
included).
"""
import pytest
import torch

from sparse_attention_banded_b200 import build, inputs, lf

pytestmark = pytest.mark.gpu

TDT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    lf.lib()
    lf.lf_device_status(reset=True)
    yield


def _guarded(shape, dtype):
    n = 1
    for s in shape:
        n *= s
    guard = 256 // torch.tensor([], dtype=dtype).element_size()
    buf = torch.full((n + 2 * guard,), 7.0, dtype=dtype, device="cuda")
    buf[guard:guard + n] = float("nan")
    return buf, buf[guard:guard + n].view(*shape), guard, n


def _check(buf, out, guard, n):
    torch.cuda.synchronize()
    assert torch.all(buf[:guard] == 7.0), "write before the output"
    assert torch.all(buf[guard + n:] == 7.0), "write past the output"
    assert torch.isfinite(out.float()).all(), "output element not written"


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("any_globals", [False, True])
def test_attention_output_guards(dtype, any_globals):
    B, H, L, w = 2, 2, 320, 64  # ragged last tile
    t = inputs.attention_inputs(B, H, L, dtype, seed=41)
    if any_globals:
        lm, gm = inputs.masks_scattered(B, L, [17, 0], [33, 0], seed=42, padded_globals=1)
    else:
        lm, gm = inputs.masks(B, L, [17, 0], [33, 0])
    buf, out, guard, n = _guarded((B, L, H * 64), TDT[dtype])
    fn = lf.lf_attention_forward_any_globals if any_globals else lf.lf_attention_forward
    fn(*[t[k].cuda() for k in inputs.NAMES], lm.cuda(), gm.cuda(), w, out=out)
    _check(buf, out, guard, n)
    assert lf.lf_device_status(reset=True) == 0


@pytest.mark.parametrize("any_globals", [False, True])
def test_layer_output_guards(any_globals):
    B, H, L, w, ffn = 1, 2, 640, 128, 256
    wl, x, W, lm, gm = inputs.layer_inputs(5, hidden=H * 64, ffn=ffn, B=B, L=L, dtype="f16", g=[5], pad=[41],
                                           seed=43, bias_scale=0.1, ln_scale=0.1)
    if any_globals:
        lm, gm = inputs.masks_scattered(B, L, [5], [41], seed=44)
    dev = {k: v.cuda() for k, v in W.items()}
    buf, out, guard, n = _guarded((B, L, H * 64), torch.float16)
    fn = lf.lf_encoder_layer_forward_any_globals if any_globals else lf.lf_encoder_layer_forward
    fn(x.cuda(), lm.cuda(), gm.cuda(), dev, H, w, out=out)
    _check(buf, out, guard, n)
    assert lf.lf_device_status(reset=True) == 0
