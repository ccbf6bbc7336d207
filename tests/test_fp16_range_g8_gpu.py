"""GPU parity at the edges of the fp16 range for the tensor-core groups of
order 6 and 8 (C_6, C_8 and p4m, FEQL_FP16).

The layers are exact ("Garanzie Teoriche" of the technical summary: the
Fourier route equals the dense layer up to floating-point rounding), so every
finite fp16 input whose outputs are representable must give the oracle's
result.  Bin 0 of an order-8 (order-6) transform sums eight (six) values and
its first butterfly stage sums two, so unscaled fp16 planes leave the range
for |v| above 8188 (10917) and for any pair above 32752; these cases put |x| or |dy| in
[1.6e4, 6e4] with the other operand and the weights scaled so that y, dx, dW
and db stay finite, a weight case puts W itself in that range, and a last set
puts the inputs near the subnormals.  Metric and bound as in the other parity
tests: max|got - ref| / max|ref| <= 5e-3.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200 import layer as Lyr
from group_dft_structured_b200.workloads import make_range_inputs
from oracle import feql_ct_oracle as OC
from oracle import feql_p4m_oracle as OM

pytestmark = pytest.mark.gpu

TOL = 5e-3
MODE = F.FEQL_FP16
FP16_MAX = 65504.0
BIG = (1.6e4, 6.0e4)
BIG_RMS = float(np.sqrt((BIG[1] ** 3 - BIG[0] ** 3) / 3 / (BIG[1] - BIG[0])))
TARGET = 3.0e3  # rms of the outputs the scalings aim for

# several forward tiles and 16-channel chunks, ragged tails, a tiny channel count
# (C_6 takes the shapes with C and D multiples of 4, those it runs on the tensor cores)
SHAPES = [(517, 24, 96), (257, 40, 130), (300, 64, 64), (129, 6, 40)]


class Cyclic8:
    O = OC
    T = 8
    PAIRS = [(t, t + 4) for t in range(4)]  # first butterfly stage
    weight_fft = staticmethod(Lyr.ct_weight_fft)
    forward = staticmethod(Lyr.ct_forward)
    backward_dx = staticmethod(Lyr.ct_backward_dx)
    backward_dw = staticmethod(Lyr.ct_backward_dw)


class P4m:
    O = OM
    T = 8
    PAIRS = [(0, 2), (1, 3), (4, 6), (5, 7)]
    weight_fft = staticmethod(Lyr.p4m_weight_fft)
    forward = staticmethod(Lyr.p4m_forward)
    backward_dx = staticmethod(Lyr.p4m_backward_dx)
    backward_dw = staticmethod(Lyr.p4m_backward_dw)


class Cyclic6(Cyclic8):
    T = 6
    PAIRS = [(t, t + 3) for t in range(3)]


GROUPS = {"C8": Cyclic8, "p4m": P4m, "C6": Cyclic6}


def cases(shapes):
    """(group, N, C, D) for every group, C_6 on its tensor-core shapes only."""
    return [(g, N, C, D) for g in sorted(GROUPS) for (N, C, D) in shapes
            if g != "C6" or (C % 4 == 0 and D % 4 == 0)]


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


def inputs(G, wid, N, C, D, x_range, dy_range, w_std, b_std=0.02):
    return make_range_inputs(wid, N, C, D, x_range, dy_range, w_std, b_std=b_std, T=G.T)


def w_std(G, C):
    return TARGET / (BIG_RMS * np.sqrt(G.T * C))


def small_range(G, N):
    s = TARGET / (BIG_RMS * np.sqrt(G.T * N))
    return (0.5 * s, 1.5 * s)


def overflows_unscaled(G, a):
    """True when an unscaled butterfly of the group's transform would leave the
    fp16 range: a fibre's sum of all values, or a sum or difference of a
    first-stage pair."""
    v = a.astype(np.float64)
    firsts = [v[..., s] + sg * v[..., t] for s, t in G.PAIRS for sg in (1, -1)]
    return bool(np.any(np.abs(v.sum(axis=-1)) > FP16_MAX)
                or any(np.any(np.abs(p) > FP16_MAX) for p in firsts))


@pytest.mark.parametrize("group,N,C,D", cases(SHAPES))
def test_forward_and_dx_with_large_inputs(group, N, C, D):
    G = GROUPS[group]
    inp = inputs(G, 50, N, C, D, BIG, BIG, min(w_std(G, C), w_std(G, D)), b_std=20.0)
    assert overflows_unscaled(G, inp["x"]) and overflows_unscaled(G, inp["dy"])
    r = f64(inp)
    ref_y, ref_dx = G.O.forward(r["x"], r["W"], r["b"]), G.O.backward_dx(r["dy"], r["W"])
    assert np.abs(ref_y).max() < FP16_MAX / 2 and np.abs(ref_dx).max() < FP16_MAX / 2
    What = G.weight_fft(dev(inp["W"]), MODE)
    y = G.forward(dev(inp["x"]), What, dev(inp["b"]), D, MODE)
    dx = G.backward_dx(dev(inp["dy"]), What, C, MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert G.O.rel_err(host(y), ref_y) <= TOL
    assert G.O.rel_err(host(dx), ref_dx) <= TOL


@pytest.mark.parametrize("group,N,C,D", cases(SHAPES))
def test_dw_with_large_x(group, N, C, D):
    G = GROUPS[group]
    inp = inputs(G, 51, N, C, D, BIG, small_range(G, N), w_std(G, C))
    assert overflows_unscaled(G, inp["x"])
    r = f64(inp)
    ref_dW, ref_db = G.O.backward_dw(r["x"], r["dy"])
    assert np.abs(ref_dW).max() < FP16_MAX / 2
    dW, db = G.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert G.O.rel_err(host(dW), ref_dW) <= TOL
    assert G.O.rel_err(host(db), ref_db) <= TOL


@pytest.mark.parametrize("group,N,C,D", cases(SHAPES))
def test_dw_with_large_dy(group, N, C, D):
    # db = sum of dy leaves the fp16 range for |dy| ~ BIG, so it is not requested
    G = GROUPS[group]
    inp = inputs(G, 52, N, C, D, small_range(G, N), BIG, w_std(G, C))
    assert overflows_unscaled(G, inp["dy"])
    r = f64(inp)
    ref_dW, _ = G.O.backward_dw(r["x"], r["dy"])
    assert np.abs(ref_dW).max() < FP16_MAX / 2
    dW, db = G.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE, with_db=False)
    assert db is None
    assert F.feql_device_status() == F.FEQL_OK
    assert G.O.rel_err(host(dW), ref_dW) <= TOL


# signs along the group axis: C_8's first-stage pairs (t, t + 4) add equal signs and
# D4's (t, t + 2) subtract opposite ones, so both double |dy|, while the eight
# values of a fibre nearly cancel and db stays finite; C_6's pairs (t, t + 3) carry
# opposite signs, doubling the first-stage differences while the six values cancel
PATTERN = {8: np.array([1, 1, -1, -1, 1, 1, -1, -1], dtype=np.float64),
           6: np.array([1, 1, -1, -1, -1, 1], dtype=np.float64)}
U16 = 2.0 ** -11  # unit roundoff of fp16


def db_plane_bound(dy, ref_db):
    """Error bound of db taken from the fp16 bin-0 planes: the three butterfly
    stages round once each (unit roundoff u) at magnitudes of at most
    sum_t |dy[n, d, t]| / 8, the 1/8 is exact and the fp32 sums add O(u^2), so
    |db - ref| <= 3 u sum_n sum_t |dy[n, d, t]| + u |ref| (the final fp16 rounding)."""
    return 3 * U16 * np.abs(dy).sum(axis=(0, 2)) + U16 * np.abs(ref_db) + 1e-6


@pytest.mark.parametrize("group", sorted(GROUPS))
def test_db_with_large_cancelling_dy(group):
    """|dy| in [3.4e4, 3.6e4] with the sign pattern above: every first-stage
    butterfly of an unscaled transform would overflow, yet dW (for small x)
    and db are ordinary fp16 numbers.  dW meets the parity bound; db, whose
    fibre sums cancel to a few percent of sum |dy|, meets the bound of the
    fp16 bin-0 planes it is computed from (db_plane_bound)."""
    G = GROUPS[group]
    N, C, D = 16, 24, 96
    inp = inputs(G, 53, N, C, D, (5e-3, 1.5e-2), (3.4e4, 3.6e4), 1.0)
    dy = inp["dy"].astype(np.float64)
    sign = np.sign(dy[..., :1])  # one random sign per (token, output channel)
    inp["dy"] = (sign * PATTERN[G.T] * np.abs(dy)).astype(np.float16)
    assert overflows_unscaled(G, inp["dy"])
    r = f64(inp)
    ref_dW, ref_db = G.O.backward_dw(r["x"], r["dy"])
    assert np.abs(ref_db).max() < FP16_MAX / 2 and np.abs(ref_dW).max() < FP16_MAX / 2
    dW, db = G.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert G.O.rel_err(host(dW), ref_dW) <= TOL
    err = np.abs(host(db) - ref_db)
    assert np.all(err <= db_plane_bound(r["dy"], ref_db)), err.max()


@pytest.mark.parametrize("group", sorted(GROUPS))
def test_large_weights(group):
    """Weights in [1.6e4, 6e4] (a fibre's unscaled Fourier planes leave the
    fp16 range) with small x and dy."""
    G = GROUPS[group]
    N, C, D = 300, 24, 96
    inp = inputs(G, 54, N, C, D, (1e-3, 3e-3), (1e-3, 3e-3), 1.0)
    W = inputs(G, 55, D, C, 1, BIG, BIG, 1.0)["x"]  # [D, C, T] of BIG magnitudes
    assert overflows_unscaled(G, W)
    r = f64(inp)
    ref_y = G.O.forward(r["x"], W.astype(np.float64), r["b"])
    ref_dx = G.O.backward_dx(r["dy"], W.astype(np.float64))
    assert np.abs(ref_y).max() < FP16_MAX / 2 and np.abs(ref_dx).max() < FP16_MAX / 2
    What = G.weight_fft(dev(W), MODE)
    y = G.forward(dev(inp["x"]), What, dev(inp["b"]), D, MODE)
    dx = G.backward_dx(dev(inp["dy"]), What, C, MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert G.O.rel_err(host(y), ref_y) <= TOL
    assert G.O.rel_err(host(dx), ref_dx) <= TOL


@pytest.mark.parametrize("group,N,C,D", cases([(517, 24, 96), (300, 64, 64)]))
def test_small_inputs_near_the_subnormals(group, N, C, D):
    """|x|, |dy| in [1e-4, 1e-3]: most eighth-scaled planes of them lie near or
    below the smallest normal fp16.  y and dx stay in the normal range; for the
    weight gradient dy is O(1), so that dW and db are normal fp16 numbers too."""
    G = GROUPS[group]
    tiny = (1e-4, 1e-3)
    inp = inputs(G, 56, N, C, D, tiny, tiny, 1.0 / np.sqrt(G.T * C), b_std=1e-5)
    r = f64(inp)
    What = G.weight_fft(dev(inp["W"]), MODE)
    y = G.forward(dev(inp["x"]), What, dev(inp["b"]), D, MODE)
    dx = G.backward_dx(dev(inp["dy"]), What, C, MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert G.O.rel_err(host(y), G.O.forward(r["x"], r["W"], r["b"])) <= TOL
    assert G.O.rel_err(host(dx), G.O.backward_dx(r["dy"], r["W"])) <= TOL

    inp = inputs(G, 57, N, C, D, tiny, (0.5, 2.0), 1.0 / np.sqrt(G.T * C))
    r = f64(inp)
    ref_dW, ref_db = G.O.backward_dw(r["x"], r["dy"])
    dW, db = G.backward_dw(dev(inp["x"]), dev(inp["dy"]), MODE)
    assert F.feql_device_status() == F.FEQL_OK
    assert G.O.rel_err(host(dW), ref_dW) <= TOL
    assert G.O.rel_err(host(db), ref_db) <= TOL
