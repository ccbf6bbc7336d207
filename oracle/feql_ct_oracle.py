"""Float64 CPU oracle for the equivariant linear layer of a general cyclic group C_T.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
and the CPU-baseline leg of the benchmark may import this module.  It shares
no code, table or constant with the CUDA library (nor with the p4 oracle in
feql_oracle.py), and the library never calls it.

What it computes
----------------
Sources: "Flash EQ-Linear: Accelerating Equivariant Linear Layers via
Group-wise Discrete Fourier Transform" — the arXiv abstract states the
method for a cyclic group of order T (cost 2(T-1)/T^2 of the dense layer) and
the technical summary ("Intuizione Centrale", "Approccio Algoritmico",
"Sfruttamento della Simmetria Coniugata", "Limitazioni e Lavoro Futuro")
describes the same circulant structure, the per-frequency products and the
conjugate symmetry of real signals; p4 (T = 4) is the case the paper builds.
For x[N,C,T], W[D,C,T], b[D]:

    y[n,d,t] = b[d] + sum_c sum_s W[d,c,(t-s) mod T] * x[n,c,s]

``forward`` materialises the unrolled group-circulant matrix

    A[T*d + t, T*c + s] = W[d, c, (t - s) mod T]          (shape [T*D, T*C])

and applies it with a library matmul (the dense method the paper replaces);
the backward is its adjoint:

    dx[n,c,s] = sum_{d,t} W[d,c,(t-s) mod T] dy[n,d,t]
    dW[d,c,u] = sum_{n,t} dy[n,d,t] x[n,c,(t-u) mod T]
    db[d]     = sum_{n,t} dy[n,d,t]

``fourier_forward_counted`` follows the paper's algorithm for any T: a real
DFT along the group axis (bins k = 0 .. floor(T/2); the others are complex
conjugates), one product per kept bin — real for k = 0 and k = T/2, complex
(four real products) otherwise — and the inverse DFT.  It counts real
multiply-accumulates: (2T-2)*N*C*D for even T, (2T-1)*N*C*D for odd T.

Pins live in tests/test_ct_oracle.py (literal sums, identity and shift
weights, equivariance, numpy.fft for the transforms, the adjoint identity,
exact directional derivatives, the MAC counts and the printed cost ratio).
"""

from __future__ import annotations

import math

import numpy as np


def group_order(a: np.ndarray) -> int:
    """T, the length of the last (group) axis."""
    return int(np.shape(a)[-1])


# ---------------------------------------------------------------------------
# Dense definition (the unrolled method, in float64)
# ---------------------------------------------------------------------------

def unrolled_circulant(W: np.ndarray) -> np.ndarray:
    """A[T*d+t, T*c+s] = W[d, c, (t-s) mod T], shape [T*D, T*C]."""
    W = np.asarray(W, dtype=np.float64)
    D, C, T = W.shape
    A = np.empty((T * D, T * C), dtype=np.float64)
    for t in range(T):
        for s in range(T):
            A[t::T, s::T] = W[:, :, (t - s) % T]
    return A


def forward(x: np.ndarray, W: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    """y = x_flat @ A^T (+ b), shape [N, D, T]."""
    x = np.asarray(x, dtype=np.float64)
    N, C, T = x.shape
    D = np.shape(W)[0]
    assert np.shape(W) == (D, C, T)
    y = (x.reshape(N, T * C) @ unrolled_circulant(W).T).reshape(N, D, T)
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None]
    return y


def backward_dx(dy: np.ndarray, W: np.ndarray) -> np.ndarray:
    """dx = dy_flat @ A, shape [N, C, T]."""
    dy = np.asarray(dy, dtype=np.float64)
    N, D, T = dy.shape
    C = np.shape(W)[1]
    return (dy.reshape(N, T * D) @ unrolled_circulant(W)).reshape(N, C, T)


def backward_dw(x: np.ndarray, dy: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(dW [D,C,T], db [D]) of the loss <dy, y>: dA = dy_flat^T x_flat folded
    along the circulant diagonals (each W entry appears once per t in A)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    N, C, T = x.shape
    D = dy.shape[1]
    dA = dy.reshape(N, T * D).T @ x.reshape(N, T * C)
    dW = np.zeros((D, C, T), dtype=np.float64)
    for t in range(T):
        for u in range(T):
            dW[:, :, u] += dA[t::T, ((t - u) % T)::T]
    return dW, dy.sum(axis=(0, 2))


def forward_bruteforce(x, W, b):
    """The layer's formula summed term by term (pure Python; tiny shapes)."""
    N, C, T = np.shape(x)
    D = np.shape(W)[0]
    y = np.zeros((N, D, T), dtype=np.float64)
    for n in range(N):
        for d in range(D):
            for t in range(T):
                acc = 0.0 if b is None else float(b[d])
                for c in range(C):
                    for s in range(T):
                        acc += float(W[d][c][(t - s) % T]) * float(x[n][c][s])
                y[n, d, t] = acc
    return y


def backward_dw_bruteforce(x, dy):
    """dW[d,c,u] = sum_{n,t} dy[n,d,t] x[n,c,(t-u) mod T] term by term."""
    N, C, T = np.shape(x)
    D = np.shape(dy)[1]
    dW = np.zeros((D, C, T), dtype=np.float64)
    for d in range(D):
        for c in range(C):
            for u in range(T):
                acc = 0.0
                for n in range(N):
                    for t in range(T):
                        acc += float(dy[n][d][t]) * float(x[n][c][(t - u) % T])
                dW[d, c, u] = acc
    return dW


# ---------------------------------------------------------------------------
# Real DFT along the group axis and the instrumented Fourier restatement
# ---------------------------------------------------------------------------

def kept_bins(T: int) -> list[int]:
    """Non-redundant bins of a real T-point signal: 0 .. floor(T/2)."""
    return list(range(T // 2 + 1))


def is_real_bin(k: int, T: int) -> bool:
    """Bin 0 and, for even T, bin T/2 are real for real input."""
    return k == 0 or 2 * k == T


def rdft(v: np.ndarray) -> list[tuple[np.ndarray, np.ndarray]]:
    """[(Re V_k, Im V_k) for k in kept_bins(T)], V_k = sum_s v_s e^{-2 pi i k s / T},
    written out as sums of cosines and sines over the last axis."""
    v = np.asarray(v, dtype=np.float64)
    T = v.shape[-1]
    out = []
    for k in kept_bins(T):
        re = np.zeros(v.shape[:-1])
        im = np.zeros(v.shape[:-1])
        for s in range(T):
            ang = 2.0 * math.pi * ((k * s) % T) / T
            re = re + v[..., s] * math.cos(ang)
            im = im - v[..., s] * math.sin(ang)
        out.append((re, im))
    return out


def irdft(bins: list[tuple[np.ndarray, np.ndarray]], T: int) -> np.ndarray:
    """Inverse of ``rdft`` for a real signal, stacked on a new last axis:
    y_t = (1/T) [ sum over real kept bins of Re Y_k cos(...) + 2 sum over the
    complex kept bins of Re(Y_k e^{2 pi i k t / T}) ] (bins T-k = conj(Y_k))."""
    ys = []
    for t in range(T):
        acc = 0.0
        for k, (re, im) in zip(kept_bins(T), bins):
            ang = 2.0 * math.pi * ((k * t) % T) / T
            term = re * math.cos(ang) - im * math.sin(ang)
            acc = acc + (term if is_real_bin(k, T) else 2.0 * term)
        ys.append(acc / T)
    return np.stack(ys, axis=-1)


class MacCounter:
    """Real multiply-accumulate counter for matrix products."""

    def __init__(self) -> None:
        self.macs = 0

    def mm(self, a: np.ndarray, b: np.ndarray) -> np.ndarray:
        assert a.ndim == 2 and b.ndim == 2 and a.shape[1] == b.shape[0]
        self.macs += a.shape[0] * a.shape[1] * b.shape[1]
        return a @ b


def fourier_forward_counted(x, W, b):
    """The paper's algorithm for C_T with its real MACs counted: (y, macs).

    Y_k[n,d] = sum_c W_k[d,c] X_k[n,c] per kept bin (convolution theorem along
    the group axis); a real bin is one real product, a complex bin four.
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    T = group_order(x)
    Xb, Wb = rdft(x), rdft(W)
    k = MacCounter()
    Yb = []
    for kk, (xr, xi), (wr, wi) in zip(kept_bins(T), Xb, Wb):
        if is_real_bin(kk, T):
            Yb.append((k.mm(xr, wr.T), np.zeros((x.shape[0], W.shape[0]))))
        else:
            yr = k.mm(xr, wr.T) - k.mm(xi, wi.T)
            yi = k.mm(xr, wi.T) + k.mm(xi, wr.T)
            Yb.append((yr, yi))
    y = irdft(Yb, T)
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None]
    return y, k.macs


def dense_macs(N: int, C: int, D: int, T: int) -> int:
    """MACs of the unrolled product: (T*C) * (T*D) per token."""
    return N * T * C * T * D


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max|got - ref| / max|ref| (0 when both are empty)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    den = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(got - ref)))
    return num if den == 0.0 else num / den
