"""Pins of the float64 oracle of the p4-equivariant MLP block (fc1 -> GELU -> fc2).

Each test ties the oracle to something other than itself: printed values of
the standard normal CDF, the standard library's erf, literal loops, the
rotation equivariance of the block, and the linear regime of GELU in which
the block collapses to a single EQ-Linear layer with a group-convolved
weight.  The last test plants mistakes and checks that a pin catches them.
"""

import math

import numpy as np
import pytest

from oracle import feql_mlp_oracle as M
from oracle import feql_oracle as P4


def rnd(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


# Standard normal CDF values (any statistics table): Phi(z)
PHI = {0.5: 0.6914624612740131, 1.0: 0.8413447460685429, 2.0: 0.9772498680518208,
       -1.0: 0.15865525393145707, -3.0: 0.0013498980316301035}


def test_gelu_is_z_times_the_normal_cdf():
    for z, phi in PHI.items():
        assert M.gelu(z) == pytest.approx(z * phi, rel=1e-13, abs=1e-16)
    zs = np.linspace(-7.0, 7.0, 57)
    lib = np.array([0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0))) for z in zs])
    assert np.allclose(M.gelu(zs), lib, rtol=1e-14, atol=1e-300)
    assert M.gelu(0.0) == 0.0


def test_gelu_odd_part_and_limits():
    z = np.linspace(-9.0, 9.0, 101)
    assert np.allclose(M.gelu(z) - M.gelu(-z), z, atol=1e-14)  # z*Phi(z) - (-z)*Phi(-z) = z
    assert M.gelu(40.0) == 40.0 and abs(M.gelu(-40.0)) < 1e-300


def test_block_is_the_literal_composition():
    N, C, H, Co = 3, 2, 5, 3
    x, W1, b1 = rnd((N, C, 4), 1), rnd((H, C, 4), 2, 0.5), rnd(H, 3)
    W2, b2 = rnd((Co, H, 4), 4, 0.5), rnd(Co, 5)
    assert np.allclose(M.forward(x, W1, b1, W2, b2), M.forward_bruteforce(x, W1, b1, W2, b2),
                       atol=1e-12)
    assert np.allclose(M.forward(x, W1, None, W2, None),
                       M.forward_bruteforce(x, W1, None, W2, None), atol=1e-12)


@pytest.mark.parametrize("r", [1, 2, 3])
def test_block_is_rotation_equivariant(r):
    N, C, H, Co = 7, 3, 8, 4
    x, W1, b1 = rnd((N, C, 4), 6), rnd((H, C, 4), 7, 0.4), rnd(H, 8)
    W2, b2 = rnd((Co, H, 4), 9, 0.3), rnd(Co, 10)
    y = M.forward(x, W1, b1, W2, b2)
    yr = M.forward(np.roll(x, r, axis=2), W1, b1, W2, b2)
    assert np.allclose(yr, np.roll(y, r, axis=2), atol=1e-12)


def test_identity_second_layer_gives_the_hidden_activations():
    N, C, H = 4, 3, 6
    x, W1, b1 = rnd((N, C, 4), 11), rnd((H, C, 4), 12, 0.5), rnd(H, 13)
    I = np.zeros((H, H, 4))
    I[:, :, 0] = np.eye(H)  # W2[o,j,u] = [o = j][u = 0]: y = g
    h = P4.forward_bruteforce(x, W1, b1)
    assert np.allclose(M.forward(x, W1, b1, I, None), 0.5 * h * (1 + np.vectorize(math.erf)(
        h / math.sqrt(2.0))), atol=1e-13)


def test_linear_regime_is_one_layer_with_the_group_convolved_weight():
    # with every pre-activation far above zero, GELU(z) = z in float64 and the block
    # is fc2(fc1(x)): one EQ-Linear layer with weight W2 (*) W1 and bias b2 + fc2(b1)
    N, C, H, Co = 5, 3, 4, 2
    x, W1 = rnd((N, C, 4), 14, 0.5), rnd((H, C, 4), 15, 0.3)
    b1 = 60.0 + rnd(H, 16)
    W2, b2 = rnd((Co, H, 4), 17), rnd(Co, 18)
    b_eff = b2 + W2.sum(axis=2) @ b1
    W = M.composed_weight(W2, W1)
    assert np.allclose(M.forward(x, W1, b1, W2, b2), P4.forward_bruteforce(x, W, b_eff),
                       atol=1e-10)
    # the composed weight, literally: sum over the hidden channel and the shift
    o, c, u = 1, 2, 3
    lit = sum(W2[o, j, v] * W1[j, c, (u - v) % 4] for j in range(H) for v in range(4))
    assert W[o, c, u] == pytest.approx(lit, abs=1e-13)


def test_mac_counts():
    f, d = M.macs(100, 24, 96, 24)
    assert (f, d) == (6 * 100 * 96 * 48, 16 * 100 * 96 * 48) and d / f == pytest.approx(16 / 6)


def gelu_tanh(z):
    """The tanh approximation of GELU (Hendrycks and Gimpel), used by the fused kernel."""
    k = math.sqrt(2.0 / math.pi)
    return 0.5 * z * (1.0 + np.tanh(k * (z + 0.044715 * z ** 3)))


def test_tanh_form_stays_within_its_bound_of_the_exact_gelu():
    # the fused kernel evaluates the tanh form; its distance to the exact GELU is
    # below 5e-4 everywhere, an order of magnitude inside the 5e-3 parity bound
    z = np.linspace(-12.0, 12.0, 200001)
    dev = np.max(np.abs(gelu_tanh(z) - M.gelu(z)))
    assert 1e-5 < dev < 5e-4


def test_pins_catch_planted_mistakes(monkeypatch):
    # a tanh-form GELU in the oracle misses the printed CDF values
    assert any(abs(gelu_tanh(z) - z * phi) > 1e-6 for z, phi in PHI.items())
    # GELU dropped: the identity-second-layer pin fails
    N, C, H = 4, 3, 6
    x, W1, b1 = rnd((N, C, 4), 11), rnd((H, C, 4), 12, 0.5), rnd(H, 13)
    I = np.zeros((H, H, 4))
    I[:, :, 0] = np.eye(H)
    h = P4.forward_bruteforce(x, W1, b1)
    with monkeypatch.context() as m:
        m.setattr(M, "gelu", lambda z: np.asarray(z, dtype=np.float64))
        assert not np.allclose(M.forward(x, W1, b1, I, None),
                               0.5 * h * (1 + np.vectorize(math.erf)(h / math.sqrt(2.0))),
                               atol=1e-6)
    # GELU on the Fourier bins instead of the group values: equivariance survives, but
    # the literal composition does not
    def gelu_on_bins(x_, W1_, b1_):
        hh = P4.forward(x_, W1_, b1_)
        bins = np.fft.fft(hh, axis=2)
        return np.real(np.fft.ifft(M.gelu(np.real(bins)) + 1j * np.imag(bins), axis=2))
    W2 = rnd((3, H, 4), 19, 0.5)
    with monkeypatch.context() as m:
        m.setattr(M, "hidden", gelu_on_bins)
        assert not np.allclose(M.forward(x, W1, b1, W2, None),
                               M.forward_bruteforce(x, W1, b1, W2, None), atol=1e-6)
