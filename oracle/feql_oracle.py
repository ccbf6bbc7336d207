"""Float64 CPU oracle for the p4 equivariant linear layer (EQ-Linear).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
and the CPU-baseline leg of the benchmark may import this module.  It shares
no code, table or constant with the CUDA library, and the library never calls
it.

What it computes
----------------
Sources: "Flash EQ-Linear: Accelerating Equivariant Linear Layers via
Group-wise Discrete Fourier Transform" (technical summary, section
"Intuizione Centrale"; and the arXiv abstract of the same paper).  The
EQ-Linear layer is a circular convolution along the group axis composed with
a linear map along the channels; its dense form is the "group-circulant"
matrix obtained by cyclically shifting and replicating the learnable weights.
For the rotation group p4 (T = 4) with x[N,C,T], W[D,C,T], b[D]:

    y[n,d,t] = b[d] + sum_c sum_s W[d,c,(t-s) mod T] * x[n,c,s]

This oracle is the *naive* method the paper accelerates (the "replicate and
multiply densely" strategy of the technical summary, section "Problematica"):
it materialises the unrolled circulant matrix

    A[T*d + t, T*c + s] = W[d, c, (t - s) mod T]          (shape [T*D, T*C])

and applies it with a library matmul in float64.  The paper states that the
Fourier method is exact (technical summary, "Garanzie Teoriche"), so the
dense definition is the right reference.

Backward (adjoint of the same linear map; the pages print no formulas):

    dx = dy_flat @ A                       dx[n,c,s] = sum_{d,t} W[d,c,(t-s)%T] dy[n,d,t]
    dA = dy_flat^T @ x_flat                (shape [T*D, T*C])
    dW[d,c,u] = sum_t dA[T*d+t, T*c+((t-u) mod T)]
    db[d] = sum_{n,t} dy[n,d,t]

A second, instrumented restatement (``fourier_forward_counted``) follows the
paper's algorithm (technical summary, "Approccio Algoritmico" and
"Specializzazione per il Gruppo di Rotazione p4"): a real DFT along the group
axis, one product per non-redundant frequency bin, conjugate symmetry for the
rest, inverse DFT.  It counts the real multiply-accumulates it performs so the
6/16 cost claim can be checked.  It is test-only, like everything here.

Pins (tests that tie this file to the mathematics rather than to itself) live
in tests/test_oracle.py: literal triple-sum brute force, identity and shift
weights, the t=0-only and t-constant special cases, equivariance, numpy.fft
for the butterflies, the adjoint identity and exact directional derivatives
for the backward, and the MAC count.
"""

from __future__ import annotations

import numpy as np

T = 4  # order of the cyclic rotation group p4


# ---------------------------------------------------------------------------
# Dense definition (the naive unrolled method, in float64)
# ---------------------------------------------------------------------------

def unrolled_circulant(W: np.ndarray) -> np.ndarray:
    """Return the dense group-circulant matrix A of shape [T*D, T*C].

    A[T*d+t, T*c+s] = W[d, c, (t-s) mod T]  — the cyclically shifted copies
    of the learnable weights (technical summary, "Intuizione Centrale").
    """
    W = np.asarray(W, dtype=np.float64)
    D, C, TT = W.shape
    assert TT == T
    A = np.empty((T * D, T * C), dtype=np.float64)
    for t in range(T):
        for s in range(T):
            A[t::T, s::T] = W[:, :, (t - s) % T]
    return A


def forward(x: np.ndarray, W: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    """y = x_flat @ A^T + b, reshaped to [N, D, T]."""
    x = np.asarray(x, dtype=np.float64)
    N, C, TT = x.shape
    assert TT == T
    D = W.shape[0]
    A = unrolled_circulant(W)
    y = (x.reshape(N, T * C) @ A.T).reshape(N, D, T)
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None]
    return y


def backward_dx(dy: np.ndarray, W: np.ndarray) -> np.ndarray:
    """dx = dy_flat @ A, reshaped to [N, C, T]."""
    dy = np.asarray(dy, dtype=np.float64)
    N, D, TT = dy.shape
    assert TT == T
    C = W.shape[1]
    A = unrolled_circulant(W)
    return (dy.reshape(N, T * D) @ A).reshape(N, C, T)


def backward_dw(x: np.ndarray, dy: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(dW [D,C,T], db [D]) of the loss <dy, y>.

    dA = dy_flat^T @ x_flat is the gradient with respect to the unrolled
    matrix; every entry of W appears T times in A (once per t), so dW sums dA
    along the circulant diagonals.
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    N, C, _ = x.shape
    D = dy.shape[1]
    dA = dy.reshape(N, T * D).T @ x.reshape(N, T * C)  # [T*D, T*C]
    dW = np.zeros((D, C, T), dtype=np.float64)
    for t in range(T):
        for u in range(T):
            dW[:, :, u] += dA[t::T, ((t - u) % T)::T]
    db = dy.sum(axis=(0, 2))
    return dW, db


# ---------------------------------------------------------------------------
# Literal definitions for tiny shapes (pure-Python loops)
# ---------------------------------------------------------------------------

def forward_bruteforce(x, W, b):
    """The layer's formula summed term by term; tiny shapes only."""
    N, C, _ = np.shape(x)
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


# ---------------------------------------------------------------------------
# Instrumented Fourier restatement (counts real MACs)
# ---------------------------------------------------------------------------

class MacCounter:
    """Real multiply-accumulate counter for matrix products."""

    def __init__(self) -> None:
        self.macs = 0

    def mm(self, a: np.ndarray, b: np.ndarray) -> np.ndarray:
        """a[M,K] @ b[K,N], counting M*K*N real MACs."""
        assert a.ndim == 2 and b.ndim == 2 and a.shape[1] == b.shape[0]
        self.macs += a.shape[0] * a.shape[1] * b.shape[1]
        return a @ b


def dense_forward_counted(x, W, b):
    """The unrolled method with its MACs counted: (y, macs)."""
    x = np.asarray(x, dtype=np.float64)
    N, C, _ = x.shape
    D = W.shape[0]
    k = MacCounter()
    y = k.mm(x.reshape(N, T * C), unrolled_circulant(W).T).reshape(N, D, T)
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None]
    return y, k.macs


def rdft4(v: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """Non-redundant bins of the 4-point DFT along the last axis.

    V_k = sum_s v_s * (-i)^(s*k); for real v only bins 0, 1, 2 are needed,
    V_3 = conj(V_1) (technical summary, "Sfruttamento della Simmetria
    Coniugata").  The p4 transform has entries 0 and +-1 only
    ("Specializzazione per il Gruppo di Rotazione p4"), so the bins are sums
    and differences:

        V0 = v0+v1+v2+v3,  V2 = v0-v1+v2-v3,  V1 = (v0-v2) + i*(v3-v1)

    Returns (V0, V2, Re V1, Im V1).
    """
    v0, v1, v2, v3 = v[..., 0], v[..., 1], v[..., 2], v[..., 3]
    return v0 + v1 + v2 + v3, v0 - v1 + v2 - v3, v0 - v2, v3 - v1


def irdft4(Y0, Y2, Y1r, Y1i) -> np.ndarray:
    """Inverse of ``rdft4`` for a real signal, stacked on a new last axis.

    y_t = (1/4) sum_k Y_k i^(t*k) with Y_3 = conj(Y_1), i.e.
    y_t = (Y0 + (-1)^t Y2)/4 + Re(Y1 * i^t)/2; the coefficients are dyadic
    (1/4 and 1/2), so the inverse is adds and exact power-of-two scalings.
    """
    e = 0.25 * (Y0 + Y2)
    o = 0.25 * (Y0 - Y2)
    return np.stack([e + 0.5 * Y1r, o - 0.5 * Y1i, e - 0.5 * Y1r, o + 0.5 * Y1i], axis=-1)


def fourier_forward_counted(x, W, b):
    """The paper's algorithm for p4 with its real MACs counted: (y, macs).

    Convolution theorem along the group axis (technical summary,
    "Trasformazione nel Dominio delle Frequenze"): Y_k[n,d] =
    sum_c W_k[d,c] X_k[n,c] for each frequency bin k, computed for bins 0, 1,
    2 only.  Bins 0 and 2 are real products; bin 1 is one complex product,
    i.e. four real ones — six real matrix products in all ("sei
    moltiplicazioni di matrici a valori reali").
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    X0, X2, X1r, X1i = rdft4(x)          # each [N, C]
    W0, W2, W1r, W1i = rdft4(W)          # each [D, C]
    k = MacCounter()
    Y0 = k.mm(X0, W0.T)
    Y2 = k.mm(X2, W2.T)
    Y1r = k.mm(X1r, W1r.T) - k.mm(X1i, W1i.T)
    Y1i = k.mm(X1r, W1i.T) + k.mm(X1i, W1r.T)
    y = irdft4(Y0, Y2, Y1r, Y1i)         # [N, D, T]
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None]
    return y, k.macs


# ---------------------------------------------------------------------------
# Comparison metric
# ---------------------------------------------------------------------------

def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max|got - ref| / max|ref| (0 when both are empty)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    den = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(got - ref)))
    if den == 0.0:
        return num
    return num / den
