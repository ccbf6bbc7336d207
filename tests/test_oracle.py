"""Pins of the float64 oracle to the mathematics and to the pages' figures.

None of these compares the oracle with itself: each check is a literal
definition, a closed form, a library routine (numpy.fft, plain matmul per
group element), an invariant, or a number printed on the pages.  The last
block plants mistakes in copies of the oracle and shows that a pin fails.
"""

import json
import os

import numpy as np
import pytest

from oracle import feql_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_cost_claims.json")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- forward ---

@pytest.mark.parametrize("N,C,D", [(1, 1, 1), (3, 2, 3), (2, 3, 2), (4, 1, 5)])
def test_forward_equals_literal_sum(N, C, D):
    x, W, b = rnd((N, C, 4), 1), rnd((D, C, 4), 2), rnd((D,), 3)
    y = O.forward(x, W, b)
    ref = O.forward_bruteforce(x, W, b)
    assert np.allclose(y, ref, rtol=0, atol=1e-13)


def test_identity_weight_returns_x():
    N, C = 7, 5
    x = rnd((N, C, 4), 4)
    W = np.zeros((C, C, 4))
    W[np.arange(C), np.arange(C), 0] = 1.0
    assert np.array_equal(O.forward(x, W, None), x)


def test_shift_weight_rolls_group_axis():
    # W[d,c,1] = delta_dc gives y_t = x_{t-1}: the convolution index (t - s).
    N, C = 6, 4
    x = rnd((N, C, 4), 5)
    W = np.zeros((C, C, 4))
    W[np.arange(C), np.arange(C), 1] = 1.0
    assert np.array_equal(O.forward(x, W, None), np.roll(x, 1, axis=2))


def test_weight_only_at_t0_is_four_plain_gemms():
    N, C, D = 9, 6, 5
    x, b = rnd((N, C, 4), 6), rnd((D,), 7)
    W = np.zeros((D, C, 4))
    W[:, :, 0] = rnd((D, C), 8)
    y = O.forward(x, W, b)
    for t in range(4):
        ref = np.matmul(x[:, :, t], W[:, :, 0].T) + b
        assert np.allclose(y[:, :, t], ref, rtol=0, atol=1e-13)


def test_weight_constant_in_t_gives_equal_outputs():
    N, C, D = 5, 3, 4
    x, b = rnd((N, C, 4), 9), rnd((D,), 10)
    Wc = rnd((D, C), 11)
    W = np.repeat(Wc[:, :, None], 4, axis=2)
    y = O.forward(x, W, b)
    ref = np.matmul(x.sum(axis=2), Wc.T) + b
    for t in range(4):
        assert np.allclose(y[:, :, t], ref, rtol=0, atol=1e-13)


def test_bias_only():
    x = rnd((3, 2, 4), 12)
    b = rnd((5,), 13)
    y = O.forward(x, np.zeros((5, 2, 4)), b)
    assert np.array_equal(y, np.broadcast_to(b[None, :, None], (3, 5, 4)))


@pytest.mark.parametrize("r", [1, 2, 3])
def test_rotation_equivariance(r):
    x, W, b = rnd((6, 3, 4), 14), rnd((4, 3, 4), 15), rnd((4,), 16)
    y = O.forward(x, W, b)
    yr = O.forward(np.roll(x, r, axis=2), W, b)
    assert np.allclose(yr, np.roll(y, r, axis=2), rtol=0, atol=1e-13)


# --------------------------------------------------- Fourier restatement ---

def test_rdft4_matches_numpy_fft():
    v = rnd((11, 4), 17)
    V0, V2, V1r, V1i = O.rdft4(v)
    F = np.fft.fft(v, axis=-1)           # F_k = sum_s v_s exp(-2 pi i s k / 4)
    assert np.allclose(V0, F[:, 0].real, atol=1e-14) and np.allclose(F[:, 0].imag, 0, atol=1e-14)
    assert np.allclose(V2, F[:, 2].real, atol=1e-14) and np.allclose(F[:, 2].imag, 0, atol=1e-14)
    assert np.allclose(V1r, F[:, 1].real, atol=1e-14)
    assert np.allclose(V1i, F[:, 1].imag, atol=1e-14)
    assert np.allclose(F[:, 3], np.conj(F[:, 1]), atol=1e-14)   # conjugate symmetry


def test_irdft4_is_exact_inverse_on_dyadic_values():
    v = np.random.default_rng(18).integers(-64, 64, size=(50, 4)).astype(np.float64) / 8
    assert np.array_equal(O.irdft4(*O.rdft4(v)), v)
    w = rnd((9, 4), 19)
    assert np.allclose(O.irdft4(*O.rdft4(w)), np.fft.ifft(np.fft.fft(w)).real, atol=1e-14)


@pytest.mark.parametrize("N,C,D", [(5, 3, 7), (16, 8, 8), (33, 24, 96)])
def test_fourier_path_equals_dense_and_counts_six_of_sixteen(N, C, D):
    x, W, b = rnd((N, C, 4), 20), rnd((D, C, 4), 21), rnd((D,), 22)
    yd, macs_dense = O.dense_forward_counted(x, W, b)
    yf, macs_fourier = O.fourier_forward_counted(x, W, b)
    assert O.rel_err(yf, yd) < 1e-13
    assert macs_dense == 16 * N * D * C
    assert macs_fourier == 6 * N * D * C


def test_paper_cost_figures():
    g = json.load(open(GOLDEN))
    T = g["group_order_T"]["value"]
    x, W = rnd((4, 2, 4), 23), rnd((3, 2, 4), 24)
    _, md = O.dense_forward_counted(x, W, None)
    _, mf = O.fourier_forward_counted(x, W, None)
    assert mf / md == 2 * (T - 1) / T ** 2                                   # abstract
    assert md // (4 * 2 * 3) == 16 and mf // (4 * 2 * 3) == g["p4_real_matmuls"]["value"]
    assert round(md / mf, 2) == g["p4_theoretical_speedup"]["approx"]
    # the measured FLOP reduction (0.134 G -> 0.052 G) sits just below 16/6:
    # transforms and bias add a little work on top of the six products.
    r = g["flops_naive_G"]["value"] / g["flops_flash_G"]["value"]
    assert abs(r - g["flops_reduction_approx"]["value"]) < 0.05 and r < md / mf
    # DFT/IDFT entries of the p4 transform are dyadic: 0, +-1 forward, 1/4 and
    # 1/2 on the inverse (product of the pages' +-1/2 radix-2 stages).
    E = np.eye(4)
    fwd = np.stack(O.rdft4(E), axis=0)
    assert set(np.unique(fwd)).issubset({-1.0, 0.0, 1.0})
    inv = O.irdft4(*[E[:, k] for k in range(4)])
    assert set(np.unique(np.abs(inv))).issubset({0.0, 0.25, 0.5})


def test_fp32_discrepancy_scale():
    # The pages report ~1e-7 relative discrepancy in FP32 between the Fourier
    # method and the dense one; the same order is reproduced here in float32.
    g = json.load(open(GOLDEN))
    x, W, b = rnd((256, 16, 4), 25), rnd((16, 16, 4), 26) / 8, rnd((16,), 27) * 0.02
    x32, W32, b32 = (a.astype(np.float32) for a in (x, W, b))
    X = [v.astype(np.float32) for v in O.rdft4(x32)]
    Wk = [v.astype(np.float32) for v in O.rdft4(W32)]
    Y0, Y2 = X[0] @ Wk[0].T, X[1] @ Wk[1].T
    Y1r = X[2] @ Wk[2].T - X[3] @ Wk[3].T
    Y1i = X[2] @ Wk[3].T + X[3] @ Wk[2].T
    y32 = O.irdft4(Y0, Y2, Y1r, Y1i) + b32[None, :, None]
    ref = O.forward(x32.astype(np.float64), W32.astype(np.float64), b32.astype(np.float64))
    err = O.rel_err(y32, ref)
    assert err < 10 * g["fp32_discrepancy"]["value"]


# --------------------------------------------------------------- backward ---

def test_adjoint_identity():
    N, C, D = 7, 3, 5
    x, W, dy = rnd((N, C, 4), 30), rnd((D, C, 4), 31), rnd((N, D, 4), 32)
    lhs = np.sum(O.forward(x, W, None) * dy)
    rhs = np.sum(x * O.backward_dx(dy, W))
    assert abs(lhs - rhs) < 1e-12 * max(1.0, abs(lhs))


def test_dx_literal_sum():
    N, C, D = 2, 3, 2
    W, dy = rnd((D, C, 4), 33), rnd((N, D, 4), 34)
    dx = O.backward_dx(dy, W)
    for n in range(N):
        for c in range(C):
            for s in range(4):
                ref = sum(W[d, c, (t - s) % 4] * dy[n, d, t] for d in range(D) for t in range(4))
                assert abs(dx[n, c, s] - ref) < 1e-13


def test_dw_db_are_exact_directional_derivatives():
    # y - b is linear in W, so <dy, y(W=E, b=0)> = <dW, E> for every E.
    N, C, D = 4, 2, 3
    x, dy = rnd((N, C, 4), 35), rnd((N, D, 4), 36)
    dW, db = O.backward_dw(x, dy)
    for d in range(D):
        for c in range(C):
            for u in range(4):
                E = np.zeros((D, C, 4))
                E[d, c, u] = 1.0
                assert abs(np.sum(dy * O.forward_bruteforce(x, E, None)) - dW[d, c, u]) < 1e-12
        e = np.zeros(D)
        e[d] = 1.0
        assert abs(np.sum(dy * O.forward_bruteforce(x, np.zeros((D, C, 4)), e)) - db[d]) < 1e-12


def test_dw_literal_sum():
    N, C, D = 3, 2, 2
    x, dy = rnd((N, C, 4), 37), rnd((N, D, 4), 38)
    dW, _ = O.backward_dw(x, dy)
    for d in range(D):
        for c in range(C):
            for u in range(4):
                ref = sum(dy[n, d, t] * x[n, c, (t - u) % 4] for n in range(N) for t in range(4))
                assert abs(dW[d, c, u] - ref) < 1e-13


@pytest.mark.parametrize("r", [1, 2, 3])
def test_backward_equivariance(r):
    x, W, dy = rnd((5, 3, 4), 39), rnd((2, 3, 4), 40), rnd((5, 2, 4), 41)
    dx = O.backward_dx(dy, W)
    assert np.allclose(O.backward_dx(np.roll(dy, r, axis=2), W), np.roll(dx, r, axis=2), atol=1e-13)
    dW, db = O.backward_dw(x, dy)
    dWr, dbr = O.backward_dw(np.roll(x, r, axis=2), np.roll(dy, r, axis=2))
    assert np.allclose(dW, dWr, atol=1e-13) and np.allclose(db, dbr, atol=1e-13)


def test_rel_err_metric():
    assert O.rel_err(np.array([1.0, -2.0]), np.array([1.0, -2.5])) == 0.5 / 2.5
    assert O.rel_err(np.zeros(0), np.zeros(0)) == 0.0


# ------------------------------------------------------- planted mistakes ---

def _circulant_with(index_fn):
    def A(W):
        D, C, _ = W.shape
        M = np.empty((4 * D, 4 * C))
        for t in range(4):
            for s in range(4):
                M[t::4, s::4] = index_fn(W, t, s)
        return M
    return A


@pytest.mark.parametrize("mutant", ["correlation", "transposed", "dropped_term"])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    fns = {
        "correlation": lambda W, t, s: W[:, :, (s - t) % 4],      # wrong sign of the index
        "transposed": lambda W, t, s: W.transpose(1, 0, 2)[:, :, (t - s) % 4],  # d and c swapped
        "dropped_term": lambda W, t, s: W[:, :, (t - s) % 4] * ((t - s) % 4 != 3),
    }
    monkeypatch.setattr(O, "unrolled_circulant", _circulant_with(fns[mutant]))
    caught = []
    # shift pin
    x = rnd((3, 3, 4), 50)
    Wsh = np.zeros((3, 3, 4))
    Wsh[np.arange(3), np.arange(3), 1] = 1.0
    caught.append(not np.array_equal(O.forward(x, Wsh, None), np.roll(x, 1, axis=2)))
    # literal-sum pin on a square, non-symmetric weight
    W, b = rnd((3, 3, 4), 51), rnd((3,), 52)
    caught.append(not np.allclose(O.forward(x, W, b), O.forward_bruteforce(x, W, b), atol=1e-12))
    assert any(caught)
