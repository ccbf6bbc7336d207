"""GPU parity at the edges of the fp16 range (p4 layer, FEQL_FP16).

The layer is exact ("Garanzie Teoriche" of the technical summary: the Fourier
route equals the dense layer up to floating-point rounding), so the fp16 path
must give the oracle's result for every finite fp16 input whose outputs are
representable.  The group-axis sums of the transform reach 4 max|v| (bin 0 of
four equal values), which leaves the fp16 range for |v| above 16376; these
cases put |x| or |dy| in [1.6e4, 6e4] with the other operand and the weights
scaled so that y, dx, dW and db stay finite, and a second set puts the inputs
near the subnormals.  Metric and bound as in test_parity_gpu.py:
max|got - ref| / max|ref| <= 5e-3.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import make_range_inputs
from oracle import feql_oracle as O

pytestmark = pytest.mark.gpu

TOL = 5e-3
MODE = F.FEQL_FP16
FP16_MAX = 65504.0
BIG = (1.6e4, 6.0e4)
# rms of |v| uniform in BIG
BIG_RMS = float(np.sqrt((BIG[1] ** 3 - BIG[0] ** 3) / 3 / (BIG[1] - BIG[0])))
TARGET = 3.0e3  # rms of the outputs the scalings aim for (max about 4x that)

# fused-kernel shape, wide separate shapes, a ragged tail, tiny channel counts
SHAPES = [(517, 24, 96), (260, 192, 192), (257, 256, 256), (129, 6, 40), (300, 16, 112)]


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


def w_std(C):
    """Weights that bring |x| ~ BIG down to outputs of rms TARGET."""
    return TARGET / (BIG_RMS * np.sqrt(4 * C))


def small_range(N):
    """|dy| (or |x|) range that brings dW = sum over 4N products with a BIG
    operand down to rms TARGET."""
    s = TARGET / (BIG_RMS * np.sqrt(4 * N))
    return (0.5 * s, 1.5 * s)


def overflows_unscaled(a):
    """True when some group-axis fibre's bin-0 sum leaves the fp16 range, i.e.
    when unscaled fp16 operand planes would hold inf."""
    v = a.astype(np.float64)
    return bool(np.any(np.abs(v.sum(axis=-1)) > FP16_MAX)
                or np.any(np.abs(v[..., 0] + v[..., 2]) > FP16_MAX))


@pytest.mark.parametrize("N,C,D", SHAPES)
def test_forward_and_dx_with_large_inputs(N, C, D):
    inp = make_range_inputs(40, N, C, D, BIG, BIG, min(w_std(C), w_std(D)), b_std=20.0)
    assert overflows_unscaled(inp["x"]) and overflows_unscaled(inp["dy"])
    r = f64(inp)
    ref_y, ref_dx = O.forward(r["x"], r["W"], r["b"]), O.backward_dx(r["dy"], r["W"])
    assert np.abs(ref_y).max() < FP16_MAX / 2 and np.abs(ref_dx).max() < FP16_MAX / 2
    What = Lyr.weight_fft(dev(inp["W"]), MODE)
    y = Lyr.forward(dev(inp["x"]), What, dev(inp["b"]), D, MODE)
    dx = Lyr.backward_dx(dev(inp["dy"]), What, C, MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert O.rel_err(host(y), ref_y) <= TOL
    assert O.rel_err(host(dx), ref_dx) <= TOL


@pytest.mark.parametrize("N,C,D", SHAPES)
def test_dw_with_large_x(N, C, D):
    inp = make_range_inputs(41, N, C, D, BIG, small_range(N), w_std(C))
    assert overflows_unscaled(inp["x"])
    r = f64(inp)
    ref_dW, ref_db = O.backward_dw(r["x"], r["dy"])
    assert np.abs(ref_dW).max() < FP16_MAX / 2
    dW, db = Lyr.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert O.rel_err(host(dW), ref_dW) <= TOL
    assert O.rel_err(host(db), ref_db) <= TOL


@pytest.mark.parametrize("N,C,D", SHAPES)
def test_dw_with_large_dy(N, C, D):
    # db = sum of dy leaves the fp16 range for |dy| ~ BIG, so it is not requested
    inp = make_range_inputs(42, N, C, D, small_range(N), BIG, w_std(C))
    assert overflows_unscaled(inp["dy"])
    r = f64(inp)
    ref_dW, _ = O.backward_dw(r["x"], r["dy"])
    assert np.abs(ref_dW).max() < FP16_MAX / 2
    dW, db = Lyr.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE, with_db=False)
    assert db is None
    assert F.feql_device_status() == F.FEQL_OK
    assert O.rel_err(host(dW), ref_dW) <= TOL


@pytest.mark.parametrize("large", ["x", "dy"])
@pytest.mark.parametrize("N,C,D", [(517, 24, 96), (4097, 16, 112), (257, 256, 256)])
def test_fused_backward_with_large_inputs(large, N, C, D):
    if large == "x":
        inp = make_range_inputs(43, N, C, D, BIG, small_range(N), w_std(D))
    else:
        inp = make_range_inputs(44, N, C, D, small_range(N), BIG, w_std(D))
    assert overflows_unscaled(inp[large])
    r = f64(inp)
    ref_dx = O.backward_dx(r["dy"], r["W"])
    ref_dW, ref_db = O.backward_dw(r["x"], r["dy"])
    What = Lyr.weight_fft(dev(inp["W"]), MODE)
    dx, dW, db = Lyr.backward(dev(inp["x"]), dev(inp["dy"]), What, MODE,
                              with_db=(large == "x"))
    assert F.feql_device_status() == F.FEQL_OK
    assert O.rel_err(host(dx), ref_dx) <= TOL
    assert O.rel_err(host(dW), ref_dW) <= TOL
    if large == "x":
        assert O.rel_err(host(db), ref_db) <= TOL


# signs along the group axis: the first-stage pairs (0, 2) and (1, 3) add equal
# signs, so both double |dy|, while bin 0 (their sum) nearly cancels
PATTERN = np.array([1, -1, 1, -1], dtype=np.float64)
U16 = 2.0 ** -11  # unit roundoff of fp16


def db_plane_bound(dy, ref_db):
    """Error bound of db taken from the fp16 bin-0 planes: the two butterfly
    stages round once each (unit roundoff u) at magnitudes of at most
    sum_t |dy[n, d, t]| / 4, the 1/4 is exact and the fp32 sums add O(u^2), so
    |db - ref| <= 2 u sum_n sum_t |dy[n, d, t]| + u |ref| (the final fp16 rounding)."""
    return 2 * U16 * np.abs(dy).sum(axis=(0, 2)) + U16 * np.abs(ref_db) + 1e-6


@pytest.mark.parametrize("N,C,D", [(16, 24, 96), (48, 256, 256)])
def test_db_with_large_cancelling_dy(N, C, D):
    """|dy| in [3.4e4, 3.6e4] with the sign pattern above: the unscaled
    first-stage sums would overflow, yet dW (for small x) and db are ordinary
    fp16 numbers.  dx and dW meet the parity bound; db, whose fibre sums cancel
    to a few percent of sum |dy|, meets the bound of the fp16 bin-0 planes it
    is computed from (db_plane_bound), in the separate and the fused backward."""
    inp = make_range_inputs(49, N, C, D, (5e-3, 1.5e-2), (3.4e4, 3.6e4), 0.5 / np.sqrt(4 * D * 16))
    dy = inp["dy"].astype(np.float64)
    sign = np.sign(dy[..., :1])  # one random sign per (token, output channel)
    inp["dy"] = (sign * PATTERN * np.abs(dy)).astype(np.float16)
    assert overflows_unscaled(inp["dy"])
    r = f64(inp)
    ref_dx = O.backward_dx(r["dy"], r["W"])
    ref_dW, ref_db = O.backward_dw(r["x"], r["dy"])
    assert np.abs(ref_db).max() < FP16_MAX / 2 and np.abs(ref_dW).max() < FP16_MAX / 2
    assert np.abs(ref_dx).max() < FP16_MAX / 2
    What = Lyr.weight_fft(dev(inp["W"]), MODE)
    bound = db_plane_bound(r["dy"], ref_db)
    for dx, dW, db in ((None,) + Lyr.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE),
                       Lyr.backward(dev(inp["x"]), dev(inp["dy"]), What, MODE)):
        assert F.feql_device_status() == F.FEQL_OK
        if dx is not None:
            assert O.rel_err(host(dx), ref_dx) <= TOL
        assert O.rel_err(host(dW), ref_dW) <= TOL
        err = np.abs(host(db) - ref_db)
        assert np.all(err <= bound), err.max()


def test_large_weights():
    """Weights up to 3e4 (bin 0 of a fibre then exceeds the fp16 range) with small x."""
    N, C, D = 300, 24, 96
    inp = make_range_inputs(45, N, C, D, (1e-3, 3e-3), BIG, 1.0)
    W = make_range_inputs(46, 1, C, D, BIG, BIG, 1.0)["x"]  # any [.., 4] array of BIG values
    W = np.resize(W, (D, C, 4)).astype(np.float16)
    assert overflows_unscaled(W)
    r = f64(inp)
    ref_y = O.forward(r["x"], W.astype(np.float64), r["b"])
    assert np.abs(ref_y).max() < FP16_MAX / 2
    What = Lyr.weight_fft(dev(W), MODE)
    y = Lyr.forward(dev(inp["x"]), What, dev(inp["b"]), D, MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert O.rel_err(host(y), ref_y) <= TOL


@pytest.mark.parametrize("N,C,D", [(517, 24, 96), (257, 256, 256)])
def test_small_inputs_near_the_subnormals(N, C, D):
    """|x|, |dy| in [1e-4, 1e-3]: a quarter of them lie below 4x the smallest
    normal fp16, so their quarter-scaled bins are subnormal.  y and dx stay in
    the normal range; for the weight gradient dy is O(1), so that dW and db are
    normal fp16 numbers too."""
    tiny = (1e-4, 1e-3)
    inp = make_range_inputs(47, N, C, D, tiny, tiny, 1.0 / np.sqrt(4 * C), b_std=1e-5)
    r = f64(inp)
    What = Lyr.weight_fft(dev(inp["W"]), MODE)
    y = Lyr.forward(dev(inp["x"]), What, dev(inp["b"]), D, MODE)
    dx = Lyr.backward_dx(dev(inp["dy"]), What, C, MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert O.rel_err(host(y), O.forward(r["x"], r["W"], r["b"])) <= TOL
    assert O.rel_err(host(dx), O.backward_dx(r["dy"], r["W"])) <= TOL

    inp = make_range_inputs(48, N, C, D, tiny, (0.5, 2.0), 1.0 / np.sqrt(4 * C))
    r = f64(inp)
    What = Lyr.weight_fft(dev(inp["W"]), MODE)
    ref_dW, ref_db = O.backward_dw(r["x"], r["dy"])
    for dW, db in (Lyr.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE),
                   Lyr.backward(dev(inp["x"]), dev(inp["dy"]), What, MODE)[1:]):
        assert F.feql_device_status() == F.FEQL_OK
        assert O.rel_err(host(dW), ref_dW) <= TOL
        assert O.rel_err(host(db), ref_db) <= TOL
