"""GPU parity: the CUDA path through the C ABI against the float64 oracle on
the same seeded, dtype-rounded inputs.

Metric: max|got - ref| / max|ref| per output tensor.  Bounds: 5e-3 for the
fp16 modes (fp32 accumulation), 1e-5 for the fp32 modes.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import WORKLOADS, make_inputs, workload_inputs
from oracle import feql_oracle as O

pytestmark = pytest.mark.gpu

TOL = {F.FEQL_FP16: 5e-3, F.FEQL_FP16_SIMT: 5e-3, F.FEQL_FP32: 1e-5, F.FEQL_FP32_SIMT: 1e-5,
       F.FEQL_FP32_3XTF32: 1e-5}
NAME = {F.FEQL_FP16: "fp16", F.FEQL_FP16_SIMT: "fp16", F.FEQL_FP32: "fp32",
        F.FEQL_FP32_SIMT: "fp32", F.FEQL_FP32_3XTF32: "fp32"}


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


def run_all(inp, mode, passes=("fwd", "dx", "dw"), with_bias=True):
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    N, C, _ = x.shape
    D = W.shape[0]
    What = Lyr.weight_fft(W, mode)
    out = {}
    if "fwd" in passes:
        out["y"] = host(Lyr.forward(x, What, b if with_bias else None, D, mode))
    if "dx" in passes:
        out["dx"] = host(Lyr.backward_dx(dy, What, C, mode))
    if "dw" in passes:
        dW, db = Lyr.backward_dw(x, dy, mode)
        out["dW"], out["db"] = host(dW), host(db)
    assert F.feql_device_status() == F.FEQL_OK
    return out


def check(out, inp, mode, with_bias=True):
    x, W, b, dy = (inp[k].astype(np.float64) for k in ("x", "W", "b", "dy"))
    errs = {}
    if "y" in out:
        errs["y"] = O.rel_err(out["y"], O.forward(x, W, b if with_bias else None))
    if "dx" in out:
        errs["dx"] = O.rel_err(out["dx"], O.backward_dx(dy, W))
    if "dW" in out:
        dW, db = O.backward_dw(x, dy)
        errs["dW"] = O.rel_err(out["dW"], dW)
        errs["db"] = O.rel_err(out["db"], db)
    for k, e in errs.items():
        assert e <= TOL[mode], (k, e)
    return errs


SMALL = [(300, 16, 16), (1000, 48, 192), (517, 24, 96), (260, 192, 192), (257, 256, 256),
         (1, 24, 96), (129, 6, 40), (384, 2, 2), (128, 34, 130)]


@pytest.mark.parametrize("mode", [F.FEQL_FP16, F.FEQL_FP16_SIMT, F.FEQL_FP32_SIMT,
                                  F.FEQL_FP32_3XTF32])
@pytest.mark.parametrize("N,C,D", SMALL)
def test_small_shapes_all_passes(mode, N, C, D):
    inp = make_inputs(9, N, C, D, NAME[mode])
    check(run_all(inp, mode), inp, mode)


@pytest.mark.parametrize("mode", [F.FEQL_FP16, F.FEQL_FP32])
def test_forward_without_bias(mode):
    inp = make_inputs(8, 333, 24, 96, NAME[mode])
    check(run_all(inp, mode, passes=("fwd",), with_bias=False), inp, mode, with_bias=False)


@pytest.mark.parametrize("mode", [F.FEQL_FP32, F.FEQL_FP32_3XTF32])
@pytest.mark.parametrize("C,D", [(3, 5), (17, 9), (1, 1), (33, 130)])
def test_fp32_odd_channels(mode, C, D):
    inp = make_inputs(7, 200, C, D, "fp32")
    check(run_all(inp, mode), inp, mode)


def test_split_tf32_deep_contraction():
    """Split TF32 keeps the fp32 bound over a 512-channel contraction per bin (the
    unrolled layer is 2048 deep), where a single tf32 product (about 2^-11
    relative) would miss it by an order of magnitude."""
    inp = make_inputs(17, 640, 512, 64, "fp32")
    check(run_all(inp, F.FEQL_FP32_3XTF32, passes=("fwd", "dx")), inp, F.FEQL_FP32_3XTF32)


def test_zero_tokens_is_a_noop_and_zeroes_dw():
    mode = F.FEQL_FP16
    inp = make_inputs(6, 4, 16, 32, "fp16")
    W = dev(inp["W"])
    What = Lyr.weight_fft(W, mode)
    x = torch.empty((0, 16, 4), dtype=torch.float16, device="cuda")
    dy = torch.empty((0, 32, 4), dtype=torch.float16, device="cuda")
    y = torch.full((1, 32, 4), 7.0, dtype=torch.float16, device="cuda")
    F.feql_forward(x, What, None, y, 0, 16, 32, mode)
    dW = torch.full((32, 16, 4), 7.0, dtype=torch.float16, device="cuda")
    db = torch.full((32,), 7.0, dtype=torch.float16, device="cuda")
    ws = Lyr.dw_workspace(0, 16, 32, mode, "cuda")
    F.feql_backward_dw(x, dy, dW, db, ws, ws.numel(), 0, 16, 32, mode)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    assert torch.all(dW == 0) and torch.all(db == 0)


@pytest.mark.parametrize("mode", [F.FEQL_FP16, F.FEQL_FP32])
def test_outputs_stay_inside_their_buffers(mode):
    N, C, D = 300, 24, 40
    inp = make_inputs(5, N, C, D, NAME[mode])
    dt = Lyr.torch_dtype(mode)
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    What = Lyr.weight_fft(W, mode)
    guard = 4096
    for shape, fn in [((N, D, 4), lambda o: F.feql_forward(x, What, b, o, N, C, D, mode)),
                      ((N, C, 4), lambda o: F.feql_backward_dx(dy, What, o, N, C, D, mode))]:
        n = int(np.prod(shape))
        buf = torch.full((n + 2 * guard,), -3.0, dtype=dt, device="cuda")
        fn(buf[guard:guard + n].view(shape))
        torch.cuda.synchronize()
        assert torch.all(buf[:guard] == -3.0) and torch.all(buf[guard + n:] == -3.0)


def test_dw_is_deterministic():
    inp = make_inputs(4, 5000, 48, 64, "fp16")
    x, dy = dev(inp["x"]), dev(inp["dy"])
    a = Lyr.backward_dw(x, dy, F.FEQL_FP16)
    b = Lyr.backward_dw(x, dy, F.FEQL_FP16)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("r", [1, 2, 3])
def test_rotation_equivariance_on_gpu(r):
    mode = F.FEQL_FP16
    inp = make_inputs(3, 700, 48, 64, "fp16")
    x, W, b = dev(inp["x"]), dev(inp["W"]), dev(inp["b"])
    What = Lyr.weight_fft(W, mode)
    y = Lyr.forward(x, What, b, 64, mode)
    yr = Lyr.forward(torch.roll(x, r, dims=2).contiguous(), What, b, 64, mode)
    err = O.rel_err(host(yr), np.roll(host(y), r, axis=2))
    assert err < 2e-3


def test_fp16_tensor_core_matches_fp16_simt_closely():
    inp = make_inputs(2, 2000, 64, 96, "fp16")
    a = run_all(inp, F.FEQL_FP16)
    b = run_all(inp, F.FEQL_FP16_SIMT)
    for k in a:
        assert O.rel_err(a[k], b[k]) < 2e-3, k


# ----------------------------------------------------------- fused backward

FUSED = [(517, 24, 96), (300, 16, 16), (1000, 48, 64), (129, 6, 40), (64, 24, 96), (1, 8, 8),
         (4097, 16, 112)]
SEPARATE = [(257, 256, 256), (300, 96, 24), (700, 32, 112)]


@pytest.mark.parametrize("N,C,D", FUSED + SEPARATE)
def test_fused_backward_matches_oracle(N, C, D):
    mode = F.FEQL_FP16
    inp = make_inputs(12, N, C, D, "fp16")
    x, W, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["dy"])
    What = Lyr.weight_fft(W, mode)
    dx, dW, db = Lyr.backward(x, dy, What, mode)
    assert F.feql_device_status() == F.FEQL_OK
    out = {"dx": host(dx), "dW": host(dW), "db": host(db)}
    check(out, inp, mode)
    # same results as the two separate passes, within rounding
    sep_dx = host(Lyr.backward_dx(dy, What, C, mode))
    sep_dW, sep_db = (host(t) for t in Lyr.backward_dw(x, dy, mode))
    assert O.rel_err(out["dx"], sep_dx) < 2e-3
    assert O.rel_err(out["dW"], sep_dW) < 2e-3 and O.rel_err(out["db"], sep_db) < 2e-3


def test_fused_backward_is_deterministic_and_stays_in_bounds():
    mode = F.FEQL_FP16
    N, C, D = 3000, 24, 96
    inp = make_inputs(13, N, C, D, "fp16")
    x, W, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["dy"])
    What = Lyr.weight_fft(W, mode)
    guard = 4096
    n = N * C * 4
    buf = torch.full((n + 2 * guard,), -3.0, dtype=torch.float16, device="cuda")
    dx = buf[guard:guard + n].view(N, C, 4)
    dW1 = torch.empty((D, C, 4), dtype=torch.float16, device="cuda")
    db1 = torch.empty((D,), dtype=torch.float16, device="cuda")
    ws = Lyr.dw_workspace(N, C, D, mode, "cuda")
    F.feql_backward(x, dy, What, dx, dW1, db1, ws, ws.numel(), N, C, D, mode)
    dW2, db2 = torch.empty_like(dW1), torch.empty_like(db1)
    F.feql_backward(x, dy, What, dx, dW2, db2, ws, ws.numel(), N, C, D, mode)
    torch.cuda.synchronize()
    assert torch.all(buf[:guard] == -3.0) and torch.all(buf[guard + n:] == -3.0)
    assert torch.equal(dW1, dW2) and torch.equal(db1, db2)


# ---------------------------------------------------------------- full sizes

@pytest.mark.parametrize("wid,mode", [(1, F.FEQL_FP32), (2, F.FEQL_FP16), (3, F.FEQL_FP16),
                                      (3, F.FEQL_FP32), (4, F.FEQL_FP16), (5, F.FEQL_FP16),
                                      (1, F.FEQL_FP32_3XTF32), (3, F.FEQL_FP32_3XTF32)])
def test_workload_full_size(wid, mode):
    w = WORKLOADS[wid]
    inp = workload_inputs(wid, dtype=NAME[mode])
    errs = check(run_all(inp, mode, passes=w.passes), inp, mode)
    print(w.name, NAME[mode], errs)


@pytest.mark.parametrize("wid", [4, 5])
def test_workload_full_size_fused_backward(wid):
    mode = F.FEQL_FP16
    inp = workload_inputs(wid, dtype="fp16")
    x, W, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["dy"])
    What = Lyr.weight_fft(W, mode)
    dx, dW, db = Lyr.backward(x, dy, What, mode)
    assert F.feql_device_status() == F.FEQL_OK
    errs = check({"dx": host(dx), "dW": host(dW), "db": host(db)}, inp, mode)
    print(WORKLOADS[wid].name, "fused backward", errs)
