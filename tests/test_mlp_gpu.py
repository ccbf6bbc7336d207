"""GPU parity of the fused p4-equivariant MLP block (fc1 -> GELU -> fc2) against
the float64 oracle.

Every test calls the library through the C ABI (ctypes); the oracle consumes
the same fp16-rounded inputs and evaluates the exact GELU.  Tolerance:
max|err| / max|ref| <= 5e-3 (the kernel's fp16 hidden activations and its tanh
form of GELU stay an order of magnitude inside it).
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import WORKLOADS, make_mlp_inputs
from oracle import feql_mlp_oracle as M

pytestmark = pytest.mark.gpu

TOL = 5e-3
FP16 = F.FEQL_FP16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from group_dft_structured_b200 import build
    build.build()
    F.load()


def dev(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy().astype(np.float64)


def run_mlp(inp, with_bias=True):
    x, W1, W2 = dev(inp["x"]), dev(inp["W1"]), dev(inp["W2"])
    b1 = dev(inp["b1"]) if with_bias else None
    b2 = dev(inp["b2"]) if with_bias else None
    H, Co = W1.shape[0], W2.shape[0]
    What = Lyr.mlp_weight_fft(W1, W2, FP16)
    y = Lyr.mlp_forward(x, What, b1, b2, H, Co, FP16)
    assert F.feql_device_status() == F.FEQL_OK
    return host(y)


def ref_mlp(inp, with_bias=True, rows=None):
    x = inp["x"].astype(np.float64)
    if rows is not None:
        x = x[rows]
    b1 = inp["b1"].astype(np.float64) if with_bias else None
    b2 = inp["b2"].astype(np.float64) if with_bias else None
    return M.forward(x, inp["W1"].astype(np.float64), b1, inp["W2"].astype(np.float64), b2)


# (N, C, H, Co): the Swin stage-1 block with a ragged tail, tiny, single hidden slice,
# padded hidden and output channels, many slices, one x tile buffer (wide C, Co = 64);
# streamed weights: the ViT-Ti and ViT-S blocks, padded output channels (Co = 80)
SHAPES = [(300, 24, 96, 24), (1, 8, 16, 8), (1000, 16, 64, 16), (129, 6, 40, 10),
          (517, 32, 128, 32), (2000, 48, 64, 64), (333, 2, 16, 2),
          (1000, 48, 192, 48), (400, 96, 384, 96), (300, 64, 256, 80), (260, 24, 96, 80)]


@pytest.mark.parametrize("N,C,H,Co", SHAPES)
def test_mlp_matches_oracle(N, C, H, Co):
    inp = make_mlp_inputs(41, N, C, H, Co, "fp16")
    err = M.rel_err(run_mlp(inp), ref_mlp(inp))
    assert err <= TOL, err


def test_mlp_without_biases():
    inp = make_mlp_inputs(42, 300, 24, 96, 24, "fp16")
    assert M.rel_err(run_mlp(inp, False), ref_mlp(inp, False)) <= TOL


@pytest.mark.parametrize("r", [1, 2])
def test_mlp_rotation_equivariance(r):
    inp = make_mlp_inputs(43, 600, 24, 96, 24, "fp16")
    y = run_mlp(inp)
    rot = dict(inp, x=np.ascontiguousarray(np.roll(inp["x"], r, axis=2)))
    assert M.rel_err(run_mlp(rot), np.roll(y, r, axis=2)) < 2e-3


def test_mlp_zero_tokens_and_output_stays_in_its_buffer():
    C, H, Co = 24, 96, 24
    inp = make_mlp_inputs(44, 777, C, H, Co, "fp16")
    x, W1, W2, b1, b2 = (dev(inp[k]) for k in ("x", "W1", "W2", "b1", "b2"))
    What = Lyr.mlp_weight_fft(W1, W2, FP16)
    y = torch.full((1, Co, 4), 7.0, dtype=torch.float16, device="cuda")
    F.feql_mlp_forward(x, What, b1, b2, y, 0, C, H, Co, FP16)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    N, guard = 777, 4096
    n = N * Co * 4
    buf = torch.full((n + 2 * guard,), -3.0, dtype=torch.float16, device="cuda")
    F.feql_mlp_forward(x, What, b1, b2, buf[guard:guard + n], N, C, H, Co, FP16)
    torch.cuda.synchronize()
    assert torch.all(buf[:guard] == -3.0) and torch.all(buf[guard + n:] == -3.0)
    out = host(buf[guard:guard + n]).reshape(N, Co, 4)
    assert M.rel_err(out, ref_mlp(inp)) <= TOL


def test_mlp_unsupported_shapes_and_modes():
    assert F.feql_mlp_weight_fft_bytes(24, 96, 112, FP16) == 0      # Co > 96
    assert F.feql_mlp_weight_fft_bytes(192, 768, 96, FP16) == 0     # x tile does not fit
    assert F.feql_mlp_weight_fft_bytes(48, 192, 48, FP16) > 0       # streamed weights
    assert F.feql_mlp_weight_fft_bytes(24, 96, 24, F.FEQL_FP32) == 0
    assert F.feql_mlp_weight_fft_bytes(24, 96, 24, FP16) > 0
    x = torch.zeros((16, 5, 4), dtype=torch.float16, device="cuda")
    y = torch.empty((16, 8, 4), dtype=torch.float16, device="cuda")
    W = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(F.FeqlError) as e:
        F.feql_mlp_forward(x, W, None, None, y, 16, 5, 16, 8, FP16)  # odd C
    assert e.value.status == F.FEQL_ERR_UNSUPPORTED


@pytest.mark.slow
def test_mlp_workload_full_size():
    w = WORKLOADS[7]
    inp = make_mlp_inputs(7, w.N, w.C, w.D, w.C, w.dtype)
    y = run_mlp(inp)
    rows = np.r_[0:4096, w.N // 2:w.N // 2 + 1024, w.N - 4096:w.N]  # sampled token rows
    assert M.rel_err(y[rows], ref_mlp(inp, rows=rows)) <= TOL
