"""GPU parity of the cyclic-group tensor-core kernels (C_8, and C_6 with its
non-dyadic twiddles and 12-byte fibres) against the float64 C_T oracle.

Every test calls the library through the C ABI (ctypes); the oracle consumes
the same dtype-rounded inputs.  Tolerance: max|err| / max|ref| <= 5e-3 (fp16
data, fp32 accumulation).
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import WORKLOADS, make_inputs, workload_inputs
from oracle import feql_ct_oracle as O

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
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy().astype(np.float64)


def run_c8(inp):
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    N, C, _ = x.shape
    D = W.shape[0]
    What = Lyr.ct_weight_fft(W, FP16)
    y = Lyr.ct_forward(x, What, b, D, FP16)
    dx = Lyr.ct_backward_dx(dy, What, C, FP16)
    dW, db = Lyr.ct_backward_dw(x, dy, FP16)
    assert F.feql_device_status() == F.FEQL_OK
    return {"y": host(y), "dx": host(dx), "dW": host(dW), "db": host(db)}


def check_c8(out, inp):
    x, W, b, dy = (inp[k].astype(np.float64) for k in ("x", "W", "b", "dy"))
    ref = {"y": O.forward(x, W, b), "dx": O.backward_dx(dy, W)}
    ref["dW"], ref["db"] = O.backward_dw(x, dy)
    errs = {k: O.rel_err(out[k], ref[k]) for k in ref}
    for k, e in errs.items():
        assert e <= TOL, (k, e)
    return errs


# several tiles and ragged tails: forward tiles of <= 64 output channels,
# 16-channel chunks, 128-token tiles; dW tiles of 128 d x 16/32 c, 32-token chunks
SHAPES = [(300, 12, 48), (1, 8, 8), (129, 6, 40), (1000, 16, 64), (517, 32, 24), (257, 40, 130),
          (70, 64, 16)]


@pytest.mark.parametrize("N,C,D", SHAPES)
def test_c8_matches_oracle(N, C, D):
    inp = make_inputs(21, N, C, D, "fp16", T=8)
    check_c8(run_c8(inp), inp)


def test_c8_without_bias():
    N, C, D = 200, 12, 48
    inp = make_inputs(22, N, C, D, "fp16", T=8)
    x, W = dev(inp["x"]), dev(inp["W"])
    y = Lyr.ct_forward(x, Lyr.ct_weight_fft(W, FP16), None, D, FP16)
    ref = O.forward(inp["x"].astype(np.float64), inp["W"].astype(np.float64), None)
    assert O.rel_err(host(y), ref) <= TOL


def test_c8_zero_tokens_is_a_noop_and_zeroes_dw():
    C, D = 12, 48
    W = dev(make_inputs(23, 4, C, D, "fp16", T=8)["W"])
    What = Lyr.ct_weight_fft(W, FP16)
    x = torch.empty((0, C, 8), dtype=torch.float16, device="cuda")
    dy = torch.empty((0, D, 8), dtype=torch.float16, device="cuda")
    y = torch.full((1, D, 8), 7.0, dtype=torch.float16, device="cuda")
    F.feql_ct_forward(8, x, What, None, y, 0, C, D, FP16)
    dW, db = Lyr.ct_backward_dw(x, dy, FP16)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    assert torch.all(dW == 0) and torch.all(db == 0)


@pytest.mark.parametrize("r", [1, 3])
def test_c8_rotation_equivariance(r):
    N, C, D = 500, 16, 32
    inp = make_inputs(24, N, C, D, "fp16", T=8)
    x, W, b = dev(inp["x"]), dev(inp["W"]), dev(inp["b"])
    What = Lyr.ct_weight_fft(W, FP16)
    y = host(Lyr.ct_forward(x, What, b, D, FP16))
    yr = host(Lyr.ct_forward(torch.roll(x, r, dims=2).contiguous(), What, b, D, FP16))
    assert O.rel_err(yr, np.roll(y, r, axis=2)) < 2e-3


def test_c8_dw_is_deterministic_and_outputs_stay_in_their_buffers():
    N, C, D = 3000, 12, 48
    inp = make_inputs(25, N, C, D, "fp16", T=8)
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    a = Lyr.ct_backward_dw(x, dy, FP16)
    c = Lyr.ct_backward_dw(x, dy, FP16)
    torch.cuda.synchronize()
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])
    What = Lyr.ct_weight_fft(W, FP16)
    guard = 4096
    for shape, fn in [((N, D, 8), lambda o: F.feql_ct_forward(8, x, What, b, o, N, C, D, FP16)),
                      ((N, C, 8), lambda o: F.feql_ct_backward_dx(8, dy, What, o, N, C, D, FP16))]:
        n = int(np.prod(shape))
        buf = torch.full((n + 2 * guard,), -3.0, dtype=torch.float16, device="cuda")
        fn(buf[guard:guard + n].view(shape))
        torch.cuda.synchronize()
        assert torch.all(buf[:guard] == -3.0) and torch.all(buf[guard + n:] == -3.0)


def test_ct_order_4_is_the_p4_path():
    N, C, D = 300, 24, 96
    inp = make_inputs(26, N, C, D, "fp16")
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    What = Lyr.weight_fft(W, FP16)
    assert torch.equal(Lyr.ct_weight_fft(W, FP16), What)
    assert torch.equal(Lyr.ct_forward(x, What, b, D, FP16), Lyr.forward(x, What, b, D, FP16))
    assert torch.equal(Lyr.ct_backward_dx(dy, What, C, FP16), Lyr.backward_dx(dy, What, C, FP16))


def test_ct_unsupported_orders_and_modes():
    # orders outside 2..16 and the split-TF32 mode (p4 only) are rejected before any launch
    assert F.feql_ct_weight_fft_bytes(17, 4, 4, FP16) == 0
    assert F.feql_ct_weight_fft_bytes(1, 4, 4, FP16) == 0
    assert F.feql_ct_weight_fft_bytes(8, 4, 4, F.FEQL_FP32_3XTF32) == 0
    # the CUDA-core orders size their buffer as fp32 planes of both directions
    assert F.feql_ct_weight_fft_bytes(6, 6, 6, FP16) == 2 * 6 * 6 * 6 * 4
    assert F.feql_ct_weight_fft_bytes(3, 4, 4, FP16) == 2 * 3 * 4 * 4 * 4
    x = torch.zeros((16, 4, 17), dtype=torch.float16, device="cuda")
    W = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    y = torch.empty((16, 4, 17), dtype=torch.float16, device="cuda")
    with pytest.raises(F.FeqlError) as e:
        F.feql_ct_forward(17, x, W, None, y, 16, 4, 4, FP16)
    assert e.value.status == F.FEQL_ERR_UNSUPPORTED


@pytest.mark.slow
def test_c8_workload_full_size():
    w = WORKLOADS[6]
    inp = workload_inputs(6)
    out = run_c8(inp)
    x, W, b, dy = (inp[k].astype(np.float64) for k in ("x", "W", "b", "dy"))
    rows = np.r_[0:2048, w.N - 2048:w.N]  # sampled token rows for y and dx
    assert O.rel_err(out["y"][rows], O.forward(x[rows], W, b)) <= TOL
    assert O.rel_err(out["dx"][rows], O.backward_dx(dy[rows], W)) <= TOL
    dW, db = O.backward_dw(x, dy)  # every token
    assert O.rel_err(out["dW"], dW) <= TOL and O.rel_err(out["db"], db) <= TOL


# C_6 on the tensor cores (C and D multiples of 4): forward tiles of <= 64 output
# channels, 16-channel chunks with a ragged second box, ragged token tiles, dW tiles
# of 128 d x 16/32 c; D = 132 and 20 take one TMA load per 8-channel box (no box stack)
C6_SHAPES = [(300, 12, 48), (1, 8, 8), (129, 4, 40), (1000, 16, 64), (517, 32, 24),
             (257, 40, 132), (70, 64, 16), (333, 20, 20)]


@pytest.mark.parametrize("N,C,D", C6_SHAPES)
def test_c6_tensor_cores_match_oracle(N, C, D):
    inp = make_inputs(31, N, C, D, "fp16", T=6)
    check_c8(run_c8(inp), inp)


@pytest.mark.parametrize("C,D", [(6, 40), (12, 10)])
def test_c6_other_channel_counts_take_the_cuda_cores(C, D):
    # C or D not a multiple of 4: the 12-byte fibres' row strides would not be
    # 16-byte multiples for the tensor maps; the CUDA-core kernels serve them
    assert F.feql_ct_weight_fft_bytes(6, C, D, FP16) == 2 * 6 * C * D * 4
    inp = make_inputs(32, 200, C, D, "fp16", T=6)
    check_c8(run_c8(inp), inp)


def test_c6_without_bias_and_zero_tokens():
    N, C, D = 200, 12, 48
    inp = make_inputs(33, N, C, D, "fp16", T=6)
    x, W = dev(inp["x"]), dev(inp["W"])
    What = Lyr.ct_weight_fft(W, FP16)
    y = Lyr.ct_forward(x, What, None, D, FP16)
    ref = O.forward(inp["x"].astype(np.float64), inp["W"].astype(np.float64), None)
    assert O.rel_err(host(y), ref) <= TOL
    x0 = torch.empty((0, C, 6), dtype=torch.float16, device="cuda")
    dy0 = torch.empty((0, D, 6), dtype=torch.float16, device="cuda")
    y0 = torch.full((1, D, 6), 7.0, dtype=torch.float16, device="cuda")
    F.feql_ct_forward(6, x0, What, None, y0, 0, C, D, FP16)
    dW, db = Lyr.ct_backward_dw(x0, dy0, FP16)
    torch.cuda.synchronize()
    assert torch.all(y0 == 7.0) and torch.all(dW == 0) and torch.all(db == 0)


@pytest.mark.parametrize("r", [1, 2, 3])
def test_c6_rotation_equivariance(r):
    N, C, D = 500, 16, 32
    inp = make_inputs(34, N, C, D, "fp16", T=6)
    x, W, b = dev(inp["x"]), dev(inp["W"]), dev(inp["b"])
    What = Lyr.ct_weight_fft(W, FP16)
    y = host(Lyr.ct_forward(x, What, b, D, FP16))
    yr = host(Lyr.ct_forward(torch.roll(x, r, dims=2).contiguous(), What, b, D, FP16))
    assert O.rel_err(yr, np.roll(y, r, axis=2)) < 2e-3


def test_c6_dw_is_deterministic_and_outputs_stay_in_their_buffers():
    N, C, D = 3000, 12, 48
    inp = make_inputs(35, N, C, D, "fp16", T=6)
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    a = Lyr.ct_backward_dw(x, dy, FP16)
    c = Lyr.ct_backward_dw(x, dy, FP16)
    torch.cuda.synchronize()
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])
    What = Lyr.ct_weight_fft(W, FP16)
    guard = 4096
    for shape, fn in [((N, D, 6), lambda o: F.feql_ct_forward(6, x, What, b, o, N, C, D, FP16)),
                      ((N, C, 6), lambda o: F.feql_ct_backward_dx(6, dy, What, o, N, C, D, FP16))]:
        n = int(np.prod(shape))
        buf = torch.full((n + 2 * guard,), -3.0, dtype=torch.float16, device="cuda")
        fn(buf[guard:guard + n].view(shape))
        torch.cuda.synchronize()
        assert torch.all(buf[:guard] == -3.0) and torch.all(buf[guard + n:] == -3.0)


@pytest.mark.slow
def test_c6_workload_full_size():
    w = WORKLOADS[10]
    inp = workload_inputs(10)
    out = run_c8(inp)
    x, W, b, dy = (inp[k].astype(np.float64) for k in ("x", "W", "b", "dy"))
    rows = np.r_[0:2048, w.N - 2048:w.N]  # sampled token rows for y and dx
    assert O.rel_err(out["y"][rows], O.forward(x[rows], W, b)) <= TOL
    assert O.rel_err(out["dx"][rows], O.backward_dx(dy[rows], W)) <= TOL
    dW, db = O.backward_dw(x, dy)  # every token
    assert O.rel_err(out["dW"], dW) <= TOL and O.rel_err(out["db"], db) <= TOL
