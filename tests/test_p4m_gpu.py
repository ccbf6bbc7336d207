"""GPU parity of the p4m (point group D4) kernels against the float64 p4m oracle.

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
from oracle import feql_p4m_oracle as O

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


def run_p4m(inp):
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    N, C, _ = x.shape
    D = W.shape[0]
    What = Lyr.p4m_weight_fft(W, FP16)
    y = Lyr.p4m_forward(x, What, b, D, FP16)
    dx = Lyr.p4m_backward_dx(dy, What, C, FP16)
    dW, db = Lyr.p4m_backward_dw(x, dy, FP16)
    assert F.feql_device_status() == F.FEQL_OK
    return {"y": host(y), "dx": host(dx), "dW": host(dW), "db": host(db)}


def check_p4m(out, inp):
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
def test_p4m_matches_oracle(N, C, D):
    inp = make_inputs(21, N, C, D, "fp16", T=8)
    check_p4m(run_p4m(inp), inp)


def test_p4m_without_bias():
    N, C, D = 200, 12, 48
    inp = make_inputs(22, N, C, D, "fp16", T=8)
    x, W = dev(inp["x"]), dev(inp["W"])
    y = Lyr.p4m_forward(x, Lyr.p4m_weight_fft(W, FP16), None, D, FP16)
    ref = O.forward(inp["x"].astype(np.float64), inp["W"].astype(np.float64), None)
    assert O.rel_err(host(y), ref) <= TOL


def test_p4m_zero_tokens_is_a_noop_and_zeroes_dw():
    C, D = 12, 48
    W = dev(make_inputs(23, 4, C, D, "fp16", T=8)["W"])
    What = Lyr.p4m_weight_fft(W, FP16)
    x = torch.empty((0, C, 8), dtype=torch.float16, device="cuda")
    dy = torch.empty((0, D, 8), dtype=torch.float16, device="cuda")
    y = torch.full((1, D, 8), 7.0, dtype=torch.float16, device="cuda")
    F.feql_p4m_forward(x, What, None, y, 0, C, D, FP16)
    dW, db = Lyr.p4m_backward_dw(x, dy, FP16)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    assert torch.all(dW == 0) and torch.all(db == 0)


@pytest.mark.parametrize("u", [O.index(1, 0), O.index(0, 1), O.index(3, 1)])
def test_p4m_equivariance(u):
    # (L_u v)(h) = v(u^-1 h): acting on the input acts the same way on the output
    N, C, D = 500, 16, 32
    inp = make_inputs(24, N, C, D, "fp16", T=8)
    x, W, b = dev(inp["x"]), dev(inp["W"]), dev(inp["b"])
    What = Lyr.p4m_weight_fft(W, FP16)
    perm = [O.mul(O.inv(u), h) for h in range(8)]
    y = host(Lyr.p4m_forward(x, What, b, D, FP16))
    yu = host(Lyr.p4m_forward(x[:, :, perm].contiguous(), What, b, D, FP16))
    assert O.rel_err(yu, y[:, :, perm]) < 2e-3


def test_p4m_rotation_only_case_agrees_with_the_p4_kernels():
    N, C, D = 700, 24, 40
    inp = make_inputs(27, N, C, D, "fp16", T=8)
    x, W, b = (torch.from_numpy(inp[k].copy()) for k in ("x", "W", "b"))
    x[:, :, 4:] = 0
    W[:, :, 4:] = 0
    x, W, b = x.cuda(), W.cuda(), b.cuda()
    y8 = host(Lyr.p4m_forward(x, Lyr.p4m_weight_fft(W, FP16), b, D, FP16))
    x4, W4 = x[:, :, :4].contiguous(), W[:, :, :4].contiguous()
    y4 = host(Lyr.forward(x4, Lyr.weight_fft(W4, FP16), b, D, FP16))
    assert O.rel_err(y8[:, :, :4], y4) < 2e-3
    assert O.rel_err(y8[:, :, 4:], np.broadcast_to(inp["b"].astype(np.float64)[None, :, None],
                                                     (N, D, 4))) < 2e-3


def test_p4m_dw_is_deterministic_and_outputs_stay_in_their_buffers():
    N, C, D = 3000, 12, 48
    inp = make_inputs(25, N, C, D, "fp16", T=8)
    x, W, b, dy = dev(inp["x"]), dev(inp["W"]), dev(inp["b"]), dev(inp["dy"])
    a = Lyr.p4m_backward_dw(x, dy, FP16)
    c = Lyr.p4m_backward_dw(x, dy, FP16)
    torch.cuda.synchronize()
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])
    What = Lyr.p4m_weight_fft(W, FP16)
    guard = 4096
    for shape, fn in [((N, D, 8), lambda o: F.feql_p4m_forward(x, What, b, o, N, C, D, FP16)),
                      ((N, C, 8), lambda o: F.feql_p4m_backward_dx(dy, What, o, N, C, D, FP16))]:
        n = int(np.prod(shape))
        buf = torch.full((n + 2 * guard,), -3.0, dtype=torch.float16, device="cuda")
        fn(buf[guard:guard + n].view(shape))
        torch.cuda.synchronize()
        assert torch.all(buf[:guard] == -3.0) and torch.all(buf[guard + n:] == -3.0)


def test_p4m_unsupported_modes():
    assert F.feql_p4m_weight_fft_bytes(4, 4, F.FEQL_FP32) == 0
    assert F.feql_p4m_weight_fft_bytes(4, 4, FP16) > 0
    x = torch.zeros((16, 4, 8), dtype=torch.float32, device="cuda")
    W = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    y = torch.empty((16, 4, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(F.FeqlError) as e:
        F.feql_p4m_forward(x, W, None, y, 16, 4, 4, F.FEQL_FP32)
    assert e.value.status == F.FEQL_ERR_UNSUPPORTED


@pytest.mark.slow
def test_p4m_workload_full_size():
    w = WORKLOADS[8]
    inp = workload_inputs(8)
    out = run_p4m(inp)
    x, W, b, dy = (inp[k].astype(np.float64) for k in ("x", "W", "b", "dy"))
    rows = np.r_[0:2048, w.N - 2048:w.N]  # sampled token rows for y and dx
    assert O.rel_err(out["y"][rows], O.forward(x[rows], W, b)) <= TOL
    assert O.rel_err(out["dx"][rows], O.backward_dx(dy[rows], W)) <= TOL
    dW, db = O.backward_dw(x, dy)  # every token
    assert O.rel_err(out["dW"], dW) <= TOL and O.rel_err(out["db"], db) <= TOL
