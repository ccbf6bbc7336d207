"""Float64 CPU oracle for the equivariant linear layer of p4m (point group D4).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
and the CPU-baseline leg of the benchmark may import this module.  It shares
no code, table or constant with the CUDA library, and the library never calls
it.

What it computes
----------------
Sources: "Flash EQ-Linear" technical summary, "Limitazioni e Lavoro Futuro"
(generalising the method to reflection groups is named as future work) and
"Intuizione Centrale" (the EQ-Linear layer is a convolution along the group
axis composed with a channel map).  The plain reading for p4m: its point group
D4 = {rotations by 90 degrees} x {reflection}, order 8, acting on itself (the
regular representation on input and output), and the layer is the group
convolution

    y[n,d,g] = b[d] + sum_c sum_h W[d,c,h^-1 g] x[n,c,h]

which for the rotation subgroup is the p4 layer W[d,c,(t-s) mod 4].

Group elements g = (r, m): rotation by r * 90 degrees (r = 0..3) after the
reflection m (m = 0, 1); stored at index 4 m + r.  Product
(r1, m1)(r2, m2) = (r1 + (-1)^m1 r2 mod 4, m1 xor m2); (r, m)^-1 =
(-(-1)^m r mod 4, m).

Fourier transform over D4 (real orthogonal irreps): four of dimension one,
A1 = 1, A2 = (-1)^m, B1 = (-1)^r, B2 = (-1)^(r+m), and E of dimension two,
E(r, m) = R(r * 90 deg) F^m with R the rotation matrix and F = diag(1, -1).
f^(rho) = sum_g f(g) rho(g); f(g) = 1/8 sum_rho d_rho tr(rho(g)^T f^(rho)).
Convolution theorem for the layer: y^(rho) = x^(rho) W^(rho) (a matrix
product for E), so per token the layer is 4 scalar channel contractions and one
2 x 2 block contraction: 4 + 8 = 12 real products of N x C x D instead of 64.
Backward: dx^(rho) = dy^(rho) W^(rho)^T,  dW^(rho) = x^(rho)^T dy^(rho)
(summed over tokens), db[d] = sum_{n,g} dy[n,d,g].

``forward`` materialises the unrolled matrix A[8 d + g, 8 c + h] =
W[d, c, h^-1 g] and applies it with a library matmul; the backward is its
adjoint.  ``fourier_forward_counted`` follows the Fourier route with explicit
irreps and counts real multiply-accumulates.

Pins live in tests/test_p4m_oracle.py.
"""

from __future__ import annotations

import numpy as np

ORDER = 8


def element(g: int) -> tuple[int, int]:
    """(r, m) of index g = 4 m + r."""
    return g % 4, g // 4


def index(r: int, m: int) -> int:
    return 4 * m + (r % 4)


def mul(g1: int, g2: int) -> int:
    r1, m1 = element(g1)
    r2, m2 = element(g2)
    return index(r1 + (-1) ** m1 * r2, m1 ^ m2)


def inv(g: int) -> int:
    r, m = element(g)
    return index(-((-1) ** m) * r, m)


def unrolled(W: np.ndarray) -> np.ndarray:
    """A[8 d + g, 8 c + h] = W[d, c, h^-1 g]  (shape [8 D, 8 C])."""
    D, C, T = W.shape
    assert T == ORDER
    A = np.empty((ORDER * D, ORDER * C))
    for g in range(ORDER):
        for h in range(ORDER):
            A[g::ORDER, h::ORDER] = W[:, :, mul(inv(h), g)]
    return A


def forward(x: np.ndarray, W: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    N, C, _ = x.shape
    D = W.shape[0]
    y = x.reshape(N, ORDER * C).astype(np.float64) @ unrolled(W.astype(np.float64)).T
    y = y.reshape(N, D, ORDER)
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None]
    return y


def backward_dx(dy: np.ndarray, W: np.ndarray) -> np.ndarray:
    N, D, _ = dy.shape
    C = W.shape[1]
    dx = dy.reshape(N, ORDER * D).astype(np.float64) @ unrolled(W.astype(np.float64))
    return dx.reshape(N, C, ORDER)


def backward_dw(x: np.ndarray, dy: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """dW[d,c,k] = sum over (g, h) with h^-1 g = k of dA[8d+g, 8c+h]; db = sum dy."""
    N, C, _ = x.shape
    D = dy.shape[1]
    dA = dy.reshape(N, ORDER * D).astype(np.float64).T @ x.reshape(N, ORDER * C).astype(np.float64)
    dW = np.zeros((D, C, ORDER))
    for g in range(ORDER):
        for h in range(ORDER):
            dW[:, :, mul(inv(h), g)] += dA[g::ORDER, h::ORDER]
    db = dy.astype(np.float64).sum(axis=(0, 2))
    return dW, db


def forward_bruteforce(x, W, b):
    """Literal loops over the definition (tiny sizes only)."""
    x = np.asarray(x, dtype=np.float64)
    N, C, _ = x.shape
    D = W.shape[0]
    y = np.zeros((N, D, ORDER))
    for n in range(N):
        for d in range(D):
            for g in range(ORDER):
                acc = 0.0 if b is None else float(b[d])
                for c in range(C):
                    for h in range(ORDER):
                        acc += float(W[d, c, mul(inv(h), g)]) * x[n, c, h]
                y[n, d, g] = acc
    return y


# ---------------------------------------------------------------------------
# Fourier route over the irreps of D4
# ---------------------------------------------------------------------------
IRREPS = ("A1", "A2", "B1", "B2", "E")
DIM = {"A1": 1, "A2": 1, "B1": 1, "B2": 1, "E": 2}


def rho(name: str, g: int) -> np.ndarray:
    """The irrep's (real orthogonal) matrix of group element g."""
    r, m = element(g)
    if name == "A1":
        return np.array([[1.0]])
    if name == "A2":
        return np.array([[(-1.0) ** m]])
    if name == "B1":
        return np.array([[(-1.0) ** r]])
    if name == "B2":
        return np.array([[(-1.0) ** (r + m)]])
    th = r * np.pi / 2
    R = np.array([[np.cos(th), -np.sin(th)], [np.sin(th), np.cos(th)]])
    return R @ np.diag([1.0, -1.0]) if m else R


def fourier(v: np.ndarray) -> dict:
    """f^(rho) = sum_g f(g) rho(g) along the last axis: {irrep: [..., d, d]}."""
    v = np.asarray(v, dtype=np.float64)
    return {name: sum(v[..., g, None, None] * rho(name, g) for g in range(ORDER))
            for name in IRREPS}


def inverse(F: dict) -> np.ndarray:
    """f(g) = 1/8 sum_rho d_rho tr(rho(g)^T f^(rho))."""
    out = []
    for g in range(ORDER):
        acc = 0.0
        for name in IRREPS:
            acc = acc + DIM[name] * np.einsum("ij,...ij->...", rho(name, g), F[name])
        out.append(acc / ORDER)
    return np.stack(out, axis=-1)


def fourier_forward_counted(x, W, b):
    """Forward by the convolution theorem; returns (y, real MACs of the products)."""
    x = np.asarray(x, dtype=np.float64)
    N, C, _ = x.shape
    D = W.shape[0]
    X, Wh = fourier(x), fourier(np.asarray(W, dtype=np.float64))
    Y = {}
    macs = 0
    for name in IRREPS:
        k = DIM[name]
        # Y[n,d] = sum_c X[n,c] W[d,c] as k x k blocks: k^3 real products per (n, c, d)
        Y[name] = np.einsum("ncij,dcjk->ndik", X[name], Wh[name])
        macs += k ** 3 * N * C * D
    y = inverse(Y)
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None]
    return y, macs


def dense_macs(N: int, C: int, D: int) -> int:
    return ORDER * ORDER * N * C * D


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    err = np.max(np.abs(got - ref)) if ref.size else 0.0
    return float(err / scale) if scale > 0 else float(err)
