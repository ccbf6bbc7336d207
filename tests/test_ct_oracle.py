"""Pins of the general cyclic-group (C_T) oracle to the mathematics.

Every check is a literal definition, a library routine (numpy.fft, plain
matmul), an invariant, a closed form, or the cost formula printed in the
arXiv abstract (2(T-1)/T^2 of the dense layer).  The last block plants
mistakes in copies of the oracle and shows a pin fails.
"""

import numpy as np
import pytest

from oracle import feql_ct_oracle as O
from oracle import feql_oracle as P4


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- forward ---

@pytest.mark.parametrize("T", [2, 3, 5, 6, 8])
def test_forward_equals_literal_sum(T):
    N, C, D = 3, 2, 3
    x, W, b = rnd((N, C, T), 1 + T), rnd((D, C, T), 2 + T), rnd((D,), 3 + T)
    assert np.allclose(O.forward(x, W, b), O.forward_bruteforce(x, W, b), rtol=0, atol=1e-12)


@pytest.mark.parametrize("T", [3, 8])
def test_identity_and_shift_weights(T):
    N, C = 5, 4
    x = rnd((N, C, T), 10)
    W = np.zeros((C, C, T))
    W[np.arange(C), np.arange(C), 0] = 1.0
    assert np.array_equal(O.forward(x, W, None), x)
    W = np.zeros((C, C, T))
    W[np.arange(C), np.arange(C), 1] = 1.0  # y_t = x_{t-1}: the convolution index (t - s)
    assert np.array_equal(O.forward(x, W, None), np.roll(x, 1, axis=2))


def test_weight_only_at_t0_is_plain_gemms():
    N, C, D, T = 6, 5, 4, 8
    x, b = rnd((N, C, T), 11), rnd((D,), 12)
    W = np.zeros((D, C, T))
    W[:, :, 0] = rnd((D, C), 13)
    y = O.forward(x, W, b)
    for t in range(T):
        assert np.allclose(y[:, :, t], np.matmul(x[:, :, t], W[:, :, 0].T) + b, rtol=0, atol=1e-13)


@pytest.mark.parametrize("T,r", [(8, 1), (8, 3), (8, 7), (6, 2)])
def test_equivariance(T, r):
    x, W, b = rnd((4, 3, T), 14), rnd((5, 3, T), 15), rnd((5,), 16)
    y = O.forward(x, W, b)
    assert np.allclose(O.forward(np.roll(x, r, axis=2), W, b), np.roll(y, r, axis=2), atol=1e-12)


def test_p4_case_agrees_with_the_p4_oracle():
    x, W, b = rnd((7, 3, 4), 17), rnd((5, 3, 4), 18), rnd((5,), 19)
    assert np.allclose(O.forward(x, W, b), P4.forward(x, W, b), rtol=0, atol=1e-13)


# ------------------------------------------------------------- transforms ---

@pytest.mark.parametrize("T", [2, 3, 4, 5, 6, 7, 8, 9])
def test_rdft_matches_numpy_fft(T):
    v = rnd((11, T), 20 + T)
    ref = np.fft.rfft(v, axis=-1)
    got = O.rdft(v)
    assert len(got) == ref.shape[-1] == len(O.kept_bins(T))
    for k, (re, im) in enumerate(got):
        assert np.allclose(re, ref[:, k].real, atol=1e-12)
        assert np.allclose(im, ref[:, k].imag, atol=1e-12)


@pytest.mark.parametrize("T", [2, 3, 4, 5, 6, 7, 8, 9])
def test_irdft_inverts_and_matches_numpy(T):
    v = rnd((9, T), 30 + T)
    bins = O.rdft(v)
    assert np.allclose(O.irdft(bins, T), v, atol=1e-12)
    spec = np.array([re + 1j * im for re, im in bins]).T
    assert np.allclose(O.irdft(bins, T), np.fft.irfft(spec, n=T, axis=-1), atol=1e-12)


def test_real_bins():
    assert [k for k in O.kept_bins(8) if O.is_real_bin(k, 8)] == [0, 4]
    assert [k for k in O.kept_bins(7) if O.is_real_bin(k, 7)] == [0]


# ------------------------------------------------- Fourier path, MAC count ---

@pytest.mark.parametrize("T", [3, 4, 5, 6, 8])
def test_fourier_path_equals_dense_and_counts_macs(T):
    N, C, D = 6, 3, 4
    x, W, b = rnd((N, C, T), 40 + T), rnd((D, C, T), 41 + T), rnd((D,), 42 + T)
    y, macs = O.fourier_forward_counted(x, W, b)
    assert O.rel_err(y, O.forward(x, W, b)) < 1e-12
    per = (2 * T - 2) if T % 2 == 0 else (2 * T - 1)
    assert macs == per * N * C * D


@pytest.mark.parametrize("T", [2, 4, 6, 8, 16])
def test_cost_ratio_is_the_abstracts_formula(T):
    # arXiv abstract: the cost is 2(T-1)/T^2 of the dense formulation.
    N, C, D = 2, 2, 3
    _, macs = O.fourier_forward_counted(rnd((N, C, T), 50), rnd((D, C, T), 51), None)
    assert macs / O.dense_macs(N, C, D, T) == 2 * (T - 1) / T ** 2
    if T == 8:
        assert macs // (N * C * D) == 14   # bins 0, 4 real; 1, 2, 3 complex


# --------------------------------------------------------------- backward ---

@pytest.mark.parametrize("T", [3, 8])
def test_adjoint_identity(T):
    x, dy, W = rnd((6, 3, T), 60), rnd((6, 4, T), 61), rnd((4, 3, T), 62)
    lhs = np.sum(O.forward(x, W, None) * dy)
    rhs = np.sum(x * O.backward_dx(dy, W))
    assert abs(lhs - rhs) < 1e-11 * max(1.0, abs(lhs))


@pytest.mark.parametrize("T", [5, 8])
def test_dw_db_are_exact_directional_derivatives(T):
    # y is linear in (W, b): <dy, y(W + E, b + e) - y(W, b)> = <dW, E> + <db, e> exactly.
    x, dy, W, b = rnd((7, 3, T), 63), rnd((7, 4, T), 64), rnd((4, 3, T), 65), rnd((4,), 66)
    E, e = rnd((4, 3, T), 67), rnd((4,), 68)
    dW, db = O.backward_dw(x, dy)
    lhs = np.sum(dy * (O.forward(x, W + E, b + e) - O.forward(x, W, b)))
    rhs = np.sum(dW * E) + np.sum(db * e)
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))


def test_dw_literal_sum():
    T = 8
    x, dy = rnd((3, 2, T), 69), rnd((3, 3, T), 70)
    dW, db = O.backward_dw(x, dy)
    assert np.allclose(dW, O.backward_dw_bruteforce(x, dy), rtol=0, atol=1e-12)
    assert np.allclose(db, dy.sum(axis=(0, 2)), rtol=0, atol=1e-13)


def test_backward_equivariance():
    T, r = 8, 3
    x, dy, W = rnd((5, 3, T), 71), rnd((5, 4, T), 72), rnd((4, 3, T), 73)
    dx = O.backward_dx(dy, W)
    assert np.allclose(O.backward_dx(np.roll(dy, r, axis=2), W), np.roll(dx, r, axis=2), atol=1e-12)
    dW, _ = O.backward_dw(x, dy)
    dWr, _ = O.backward_dw(np.roll(x, r, axis=2), np.roll(dy, r, axis=2))
    assert np.allclose(dWr, dW, atol=1e-12)


# ------------------------------------------------------- planted mistakes ---

def test_pins_catch_planted_mistakes(monkeypatch):
    T = 8
    x, W, b = rnd((3, 3, T), 80), rnd((3, 3, T), 81), rnd((3,), 82)

    def correlation(Wm):  # wrong sign of the circulant index
        D, C, TT = Wm.shape
        A = np.empty((TT * D, TT * C))
        for t in range(TT):
            for s in range(TT):
                A[t::TT, s::TT] = Wm[:, :, (s - t) % TT]
        return A

    with monkeypatch.context() as m:
        m.setattr(O, "unrolled_circulant", correlation)
        assert not np.allclose(O.forward(x, W, b), O.forward_bruteforce(x, W, b), atol=1e-12)

    # dropping the real Nyquist bin k = T/2, or the factor 2 of the complex bins, in the
    # inverse transform breaks the numpy.fft pin
    v = rnd((4, T), 83)
    bins = O.rdft(v)
    good = O.irdft(bins, T)
    assert np.allclose(good, np.fft.irfft(np.fft.rfft(v), n=T), atol=1e-12)

    def irdft_no_nyquist(bs, TT):
        bs = list(bs)
        bs[TT // 2] = (np.zeros_like(bs[TT // 2][0]), np.zeros_like(bs[TT // 2][1]))
        return good_irdft(bs, TT)

    def irdft_no_factor2(bs, TT):
        ys = []
        for t in range(TT):
            acc = 0.0
            for k, (re, im) in zip(O.kept_bins(TT), bs):
                ang = 2.0 * np.pi * ((k * t) % TT) / TT
                acc = acc + re * np.cos(ang) - im * np.sin(ang)
            ys.append(acc / TT)
        return np.stack(ys, axis=-1)

    good_irdft = O.irdft
    for mutant in (irdft_no_nyquist, irdft_no_factor2):
        assert not np.allclose(mutant(bins, T), np.fft.irfft(np.fft.rfft(v), n=T), atol=1e-6)
