"""GPU parity of the fused p4 MLP block at the edges of the fp16 range.

A stack of two fp16 EQ-Linear layers with GELU between gives a finite result
whenever its input, weights, hidden activation h and output y are finite fp16
numbers; the fused block must match it there, although its fp16 operand planes
hold sums of four values (bin 0 of x, of the weights and of GELU(h)).  Each
case puts one operand in [1.6e4, 6e4] (or the hidden activation up to about
5e4) with the others scaled so that h and y stay finite, and checks that the
unscaled planes would have left the fp16 range; a last case puts x near the
subnormals.  Metric and bound as in test_mlp_gpu.py: max|err| / max|ref| <= 5e-3.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import make_mlp_range_inputs
from oracle import feql_mlp_oracle as M

pytestmark = pytest.mark.gpu

TOL = 5e-3
FP16 = F.FEQL_FP16
FP16_MAX = 65504.0
BIG = (1.6e4, 6.0e4)
BIG_RMS = float(np.sqrt((BIG[1] ** 3 - BIG[0] ** 3) / 3 / (BIG[1] - BIG[0])))
TARGET = 3.0e3

# resident weights (Swin stage-1 block, ragged tail) and streamed weights (ViT-S block)
SHAPES = [(300, 24, 96, 24), (400, 96, 384, 96)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from group_dft_structured_b200 import build
    build.build()
    F.load()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy().astype(np.float64)


def f64(inp):
    return {k: v.astype(np.float64) for k, v in inp.items()}


def bin0_overflows(a):
    """True when a fibre's unscaled bin 0 (or first-stage pair sum) leaves the fp16 range."""
    v = a.astype(np.float64)
    return bool(np.any(np.abs(v.sum(axis=-1)) > FP16_MAX)
                or np.any(np.abs(v[..., 0] + v[..., 2]) > FP16_MAX)
                or np.any(np.abs(v[..., 1] + v[..., 3]) > FP16_MAX))


def check(inp):
    r = f64(inp)
    ref = M.forward(r["x"], r["W1"], r["b1"], r["W2"], r["b2"])
    h = M.hidden(r["x"], r["W1"], r["b1"])
    assert np.abs(h).max() < FP16_MAX and np.abs(ref).max() < FP16_MAX / 2
    H, Co = inp["W1"].shape[0], inp["W2"].shape[0]
    What = Lyr.mlp_weight_fft(dev(inp["W1"]), dev(inp["W2"]), FP16)
    y = Lyr.mlp_forward(dev(inp["x"]), What, dev(inp["b1"]), dev(inp["b2"]), H, Co, FP16)
    assert F.feql_device_status() == F.FEQL_OK
    err = M.rel_err(host(y), ref)
    assert err <= TOL, err
    return r, h


@pytest.mark.parametrize("N,C,H,Co", SHAPES)
def test_large_x(N, C, H, Co):
    inp = make_mlp_range_inputs(60, N, C, H, Co, BIG, TARGET / (BIG_RMS * np.sqrt(4 * C)),
                                1.0 / np.sqrt(4 * H))
    assert bin0_overflows(inp["x"])
    check(inp)


@pytest.mark.parametrize("N,C,H,Co", SHAPES)
def test_large_hidden_activation(N, C, H, Co):
    """h of rms about 7e3 and up to 5e4: the four-value sums of GELU(h) exceed the fp16 range."""
    inp = make_mlp_range_inputs(61, N, C, H, Co, 1.0, 1e4 / np.sqrt(4 * C),
                                TARGET / (1e4 * np.sqrt(2 * H)), b1_std=20.0)
    _, h = check(inp)
    assert bin0_overflows(M.gelu(h))


@pytest.mark.parametrize("N,C,H,Co", SHAPES)
def test_large_w1(N, C, H, Co):
    inp = make_mlp_range_inputs(62, N, C, H, Co, (1e-3, 3e-3), BIG, 1.0 / np.sqrt(4 * H))
    assert bin0_overflows(inp["W1"])
    check(inp)


@pytest.mark.parametrize("N,C,H,Co", SHAPES)
def test_large_w2(N, C, H, Co):
    inp = make_mlp_range_inputs(63, N, C, H, Co, 1.0, 4e-3 / np.sqrt(4 * C), BIG, b1_std=4e-4)
    assert bin0_overflows(inp["W2"])
    check(inp)


@pytest.mark.parametrize("N,C,H,Co", SHAPES)
def test_small_x_near_the_subnormals(N, C, H, Co):
    """|x| in [1e-4, 1e-3]: h / 8, the scale of the hidden planes, is largely
    below the smallest normal fp16."""
    inp = make_mlp_range_inputs(64, N, C, H, Co, (1e-4, 1e-3), 1.0 / np.sqrt(4 * C),
                                1.0 / np.sqrt(4 * H), b1_std=1e-5, b2_std=1e-6)
    check(inp)
