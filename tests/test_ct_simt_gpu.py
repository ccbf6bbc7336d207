"""GPU parity of the CUDA-core kernels of the cyclic group C_T (any order 2..16)
against the float64 C_T oracle.

Every test calls the library through the C ABI (ctypes).  Orders with
non-dyadic twiddles (T = 3, 5, 6, 7, 12) and mixed radices (6 = 2 x 3,
12 = 4 x 3) run here, as do the fp32 modes of T = 8.  Tolerances:
max|err| / max|ref| <= 1e-5 for fp32 data, 5e-3 for fp16 data (fp32 arithmetic).
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import make_inputs
from oracle import feql_ct_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-5, "fp16": 5e-3}
MODE = {"fp32": F.FEQL_FP32, "fp16": F.FEQL_FP16_SIMT}


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


def run_and_check(T, dtype, N, C, D, seed=51):
    inp = make_inputs(seed, N, C, D, dtype, T=T)
    mode = MODE[dtype]
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    What = Lyr.ct_weight_fft(W, mode)
    y = Lyr.ct_forward(x, What, b, D, mode)
    dx = Lyr.ct_backward_dx(dy, What, C, mode)
    dW, db = Lyr.ct_backward_dw(x, dy, mode)
    assert F.feql_device_status() == F.FEQL_OK
    f64 = {k: v.astype(np.float64) for k, v in inp.items()}
    rdW, rdb = O.backward_dw(f64["x"], f64["dy"])
    errs = {"y": O.rel_err(host(y), O.forward(f64["x"], f64["W"], f64["b"])),
            "dx": O.rel_err(host(dx), O.backward_dx(f64["dy"], f64["W"])),
            "dW": O.rel_err(host(dW), rdW), "db": O.rel_err(host(db), rdb)}
    for k, e in errs.items():
        assert e <= TOL[dtype], (T, dtype, k, e)


@pytest.mark.parametrize("T", [2, 3, 5, 6, 7, 8, 12, 16])
@pytest.mark.parametrize("dtype", ["fp32", "fp16"])
def test_ct_cuda_cores_match_oracle(T, dtype):
    # several 32 x 32 tiles with ragged tails in tokens, channels and outputs
    run_and_check(T, dtype, 300, 12, 40)


@pytest.mark.parametrize("N,C,D", [(1, 1, 1), (33, 35, 9), (1000, 64, 64)])
def test_ct_cuda_cores_shapes(N, C, D):
    run_and_check(6, "fp32", N, C, D, seed=52)


def test_ct_cuda_cores_rotation_equivariance():
    T, N, C, D = 6, 200, 10, 14
    inp = make_inputs(53, N, C, D, "fp32", T=T)
    mode = F.FEQL_FP32
    x, W, b = dev(inp["x"]), dev(inp["W"]), dev(inp["b"])
    What = Lyr.ct_weight_fft(W, mode)
    y = host(Lyr.ct_forward(x, What, b, D, mode))
    yr = host(Lyr.ct_forward(torch.roll(x, 1, dims=2).contiguous(), What, b, D, mode))
    assert O.rel_err(yr, np.roll(y, 1, axis=2)) < 1e-5


def test_ct_cuda_cores_zero_tokens():
    T, C, D = 12, 6, 10
    W = dev(make_inputs(54, 4, C, D, "fp32", T=T)["W"])
    What = Lyr.ct_weight_fft(W, F.FEQL_FP32)
    x = torch.empty((0, C, T), dtype=torch.float32, device="cuda")
    dy = torch.empty((0, D, T), dtype=torch.float32, device="cuda")
    y = torch.full((1, D, T), 7.0, dtype=torch.float32, device="cuda")
    F.feql_ct_forward(T, x, What, None, y, 0, C, D, F.FEQL_FP32)
    dW, db = Lyr.ct_backward_dw(x, dy, F.FEQL_FP32)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0) and torch.all(dW == 0) and torch.all(db == 0)
