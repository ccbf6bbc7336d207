"""Pins of the float64 oracle of the p4m (point group D4) equivariant linear layer.

The pins tie the oracle to the mathematics: the group axioms and the defining
relations of D4, the irreps (homomorphism, orthogonality of characters,
Plancherel), literal loops, explicit translations by a rotation and by the
reflection, the p4 layer as the rotation-only special case, equivariance under
every group element, the convolution theorem with its MAC count (12 of 64),
the adjoint identity and exact derivatives, and planted mistakes.
"""

import numpy as np
import pytest

from oracle import feql_oracle as P4
from oracle import feql_p4m_oracle as O

G = range(O.ORDER)
R1 = O.index(1, 0)   # rotation by 90 degrees
M1 = O.index(0, 1)   # the reflection


def rnd(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def power(g, k):
    out = 0
    for _ in range(k):
        out = O.mul(out, g)
    return out


# ------------------------------------------------------------------ group ---

def test_group_axioms_and_dihedral_relations():
    for a in G:
        assert O.mul(0, a) == a == O.mul(a, 0)
        assert O.mul(a, O.inv(a)) == 0 == O.mul(O.inv(a), a)
        for b in G:
            assert O.mul(a, b) in G
            for c in G:
                assert O.mul(O.mul(a, b), c) == O.mul(a, O.mul(b, c))
    assert power(R1, 4) == 0 and power(R1, 2) != 0 and O.mul(M1, M1) == 0
    assert O.mul(O.mul(M1, R1), M1) == O.inv(R1)         # m r m = r^-1
    assert O.mul(R1, M1) != O.mul(M1, R1)                # not abelian
    assert sorted({O.mul(power(R1, k), power(M1, j)) for k in range(4) for j in range(2)}) == list(G)


# ----------------------------------------------------------------- irreps ---

def test_irreps_are_orthogonal_homomorphisms():
    for name in O.IRREPS:
        for a in G:
            Ra = O.rho(name, a)
            assert np.allclose(Ra @ Ra.T, np.eye(O.DIM[name]), atol=1e-14)
            for b in G:
                assert np.allclose(O.rho(name, O.mul(a, b)), Ra @ O.rho(name, b), atol=1e-14)
    assert sum(O.DIM[n] ** 2 for n in O.IRREPS) == O.ORDER


def test_characters_are_orthonormal():
    chi = {n: np.array([np.trace(O.rho(n, g)) for g in G]) for n in O.IRREPS}
    for a in O.IRREPS:
        for b in O.IRREPS:
            assert np.dot(chi[a], chi[b]) / O.ORDER == pytest.approx(1.0 if a == b else 0.0, abs=1e-14)


def test_fourier_inverts_and_preserves_energy():
    v = rnd((5, O.ORDER), 1)
    F = O.fourier(v)
    assert np.allclose(O.inverse(F), v, atol=1e-13)
    energy = sum(O.DIM[n] * np.sum(F[n] ** 2, axis=(-2, -1)) for n in O.IRREPS) / O.ORDER
    assert np.allclose(energy, np.sum(v ** 2, axis=-1), atol=1e-12)


# ------------------------------------------------------------------ layer ---

def test_forward_equals_literal_sum():
    x, W, b = rnd((3, 2, 8), 2), rnd((3, 2, 8), 3), rnd(3, 4)
    assert np.allclose(O.forward(x, W, b), O.forward_bruteforce(x, W, b), atol=1e-12)
    assert np.allclose(O.forward(x, W, None), O.forward_bruteforce(x, W, None), atol=1e-12)


def _delta_weight(C, k):
    W = np.zeros((C, C, 8))
    W[:, :, k] = np.eye(C)
    return W


def test_translation_by_the_reflection_swaps_the_halves():
    # W = identity at k = m: y(g) = x(g m^-1) = x(r, 1 - m)
    x = rnd((4, 3, 8), 5)
    y = O.forward(x, _delta_weight(3, M1), None)
    assert np.array_equal(y[..., :4], x[..., 4:]) and np.array_equal(y[..., 4:], x[..., :4])


def test_translation_by_a_rotation_turns_the_halves_opposite_ways():
    # W = identity at k = r: y(t, 0) = x(t - 1, 0) and y(t, 1) = x(t + 1, 1)
    x = rnd((4, 3, 8), 6)
    y = O.forward(x, _delta_weight(3, R1), None)
    assert np.array_equal(y[..., :4], np.roll(x[..., :4], 1, axis=-1))
    assert np.array_equal(y[..., 4:], np.roll(x[..., 4:], -1, axis=-1))


def test_rotation_only_case_is_the_p4_layer():
    x, W, b = rnd((6, 3, 8), 7), rnd((4, 3, 8), 8), rnd(4, 9)
    x[..., 4:] = 0.0
    W[..., 4:] = 0.0
    y = O.forward(x, W, b)
    assert np.allclose(y[..., :4], P4.forward(x[..., :4], W[..., :4], b), atol=1e-12)
    assert np.allclose(y[..., 4:], np.broadcast_to(b[None, :, None], y[..., 4:].shape), atol=1e-12)


@pytest.mark.parametrize("u", list(G))
def test_equivariance_under_every_group_element(u):
    x, W, b = rnd((5, 3, 8), 10), rnd((2, 3, 8), 11), rnd(2, 12)
    act = lambda v: v[..., [O.mul(O.inv(u), h) for h in G]]  # (L_u v)(h) = v(u^-1 h)
    assert np.allclose(O.forward(act(x), W, b), act(O.forward(x, W, b)), atol=1e-12)


def test_fourier_route_equals_dense_and_costs_12_of_64():
    N, C, D = 7, 3, 5
    x, W, b = rnd((N, C, 8), 13), rnd((D, C, 8), 14), rnd(D, 15)
    y, macs = O.fourier_forward_counted(x, W, b)
    assert np.allclose(y, O.forward(x, W, b), atol=1e-12)
    assert macs == 12 * N * C * D and macs / O.dense_macs(N, C, D) == pytest.approx(3 / 16)


def test_backward_fourier_forms():
    # the kernels' formulas: dx^ = dy^ W^T, dW^ = x^T dy^ (summed over tokens)
    N, C, D = 6, 3, 4
    x, W, dy = rnd((N, C, 8), 16), rnd((D, C, 8), 17), rnd((N, D, 8), 18)
    X, Wh, dY = O.fourier(x), O.fourier(W), O.fourier(dy)
    dX = {n: np.einsum("ndij,dckj->ncik", dY[n], Wh[n]) for n in O.IRREPS}
    assert np.allclose(O.inverse(dX), O.backward_dx(dy, W), atol=1e-12)
    dWh = {n: np.einsum("ncji,ndjk->dcik", X[n], dY[n]) for n in O.IRREPS}
    dW, _ = O.backward_dw(x, dy)
    assert np.allclose(O.inverse(dWh), dW, atol=1e-12)


def test_adjoint_and_exact_derivatives():
    N, C, D = 5, 3, 4
    x, W, b, dy = rnd((N, C, 8), 19), rnd((D, C, 8), 20), rnd(D, 21), rnd((N, D, 8), 22)
    assert np.sum(dy * O.forward(x, W, None)) == pytest.approx(np.sum(O.backward_dx(dy, W) * x),
                                                               rel=1e-12)
    dW, db = O.backward_dw(x, dy)
    base = np.sum(dy * O.forward(x, W, b))
    for d, c, k in [(0, 0, 0), (3, 2, 5), (1, 1, 7)]:
        E = np.zeros_like(W)
        E[d, c, k] = 1.0  # the loss is linear in W: the difference is exact
        assert np.sum(dy * O.forward(x, W + E, b)) - base == pytest.approx(dW[d, c, k], rel=1e-9)
    e = np.zeros(D)
    e[2] = 1.0
    assert np.sum(dy * O.forward(x, W, b + e)) - base == pytest.approx(db[2], rel=1e-9)
    # literal sum: dW[d,c,k] = sum_{n,g} dy[n,d,g] x[n,c,g k^-1]
    d, c, k = 2, 1, O.index(3, 1)
    lit = sum(dy[n, d, g] * x[n, c, O.mul(g, O.inv(k))] for n in range(N) for g in G)
    assert dW[d, c, k] == pytest.approx(lit, rel=1e-12)


# -------------------------------------------------------- planted mistakes ---

def test_pins_catch_planted_mistakes(monkeypatch):
    x = rnd((4, 3, 8), 23)
    # convolution on the other side (W[g h^-1]): the rotation-translation pin fails
    with monkeypatch.context() as m:
        def unrolled_right(W):
            D, C, _ = W.shape
            A = np.empty((8 * D, 8 * C))
            for g in G:
                for h in G:
                    A[g::8, h::8] = W[:, :, O.mul(g, O.inv(h))]
            return A
        m.setattr(O, "unrolled", unrolled_right)
        y = O.forward(x, _delta_weight(3, R1), None)
        assert not np.array_equal(y[..., 4:], np.roll(x[..., 4:], -1, axis=-1))
    # E with the reflection on the left is not a homomorphism
    with monkeypatch.context() as m:
        orig = O.rho

        def rho_left(name, g):
            if name != "E":
                return orig(name, g)
            r, mm = O.element(g)
            th = r * np.pi / 2
            R = np.array([[np.cos(th), -np.sin(th)], [np.sin(th), np.cos(th)]])
            return np.diag([1.0, -1.0]) @ R if mm else R
        m.setattr(O, "rho", rho_left)
        assert not all(np.allclose(O.rho("E", O.mul(a, b)), O.rho("E", a) @ O.rho("E", b))
                       for a in G for b in G)
    # the product in the wrong order (W^ x^) disagrees with the dense layer
    W = rnd((2, 3, 8), 24)
    X, Wh = O.fourier(x), O.fourier(W)
    Y = {n: np.einsum("dcij,ncjk->ndik", Wh[n], X[n]) for n in O.IRREPS}
    assert not np.allclose(O.inverse(Y), O.forward(x, W, None), atol=1e-6)
