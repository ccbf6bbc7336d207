"""Float64 CPU oracle for the p4-equivariant MLP block (fc1 -> GELU -> fc2).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
and the CPU-baseline leg of the benchmark may import this module.  It shares
no code, table or constant with the CUDA library, and the library never calls
it.

What it computes
----------------
Sources: "Flash EQ-Linear" technical summary, section "Livello di Rete": the
layer is integrated into Flash EQ-ViT and Flash EQ-Swin, whose transformer
blocks end in an MLP of two EQ-Linear layers with a GELU between them; the
1.4-1.7x end-to-end inference speed-up is measured on these networks.  The
pages do not spell the block out; the plain reading taken here is the ViT/Swin
MLP with both linear layers replaced by p4 EQ-Linear layers:

    h[n,j,t] = b1[j] + sum_c sum_s W1[j,c,(t-s) mod 4] x[n,c,s]     (fc1, C -> H)
    g[n,j,t] = GELU(h[n,j,t])                                        (pointwise)
    y[n,o,t] = b2[o] + sum_j sum_s W2[o,j,(t-s) mod 4] g[n,j,s]      (fc2, H -> Co)

GELU is the exact form of the transformer MLPs, GELU(z) = z * Phi(z) =
z/2 * (1 + erf(z / sqrt 2)), with Phi the standard normal CDF.  A pointwise
function of the group-indexed features commutes with the cyclic shift of the
group axis, so the block is rotation-equivariant.

Each linear layer is the p4 oracle's dense definition (``feql_oracle.forward``,
the unrolled group-circulant matrix in float64); erf is scipy's.

Pins live in tests/test_mlp_oracle.py: printed values of the standard normal
CDF, the odd/even split of GELU, the literal per-element composition, the
rotation equivariance, a reduction to one EQ-Linear layer (identity second
layer), and the linear regime where GELU(z) = z, in which the block is one
EQ-Linear layer whose weight is the group convolution of W2 and W1.
"""

from __future__ import annotations

import numpy as np
from scipy.special import erf

from . import feql_oracle as P4


def gelu(z: np.ndarray) -> np.ndarray:
    """Exact GELU, z * Phi(z), in float64."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def hidden(x: np.ndarray, W1: np.ndarray, b1: np.ndarray | None) -> np.ndarray:
    """fc1 followed by GELU: g[N, H, 4]."""
    return gelu(P4.forward(x, W1, b1))


def forward(x: np.ndarray, W1: np.ndarray, b1: np.ndarray | None, W2: np.ndarray,
            b2: np.ndarray | None) -> np.ndarray:
    """y[N, Co, 4] of the block, float64."""
    return P4.forward(hidden(x, W1, b1), W2, b2)


def forward_bruteforce(x, W1, b1, W2, b2):
    """Literal per-element loops (tiny sizes only): the three formulas above."""
    x = np.asarray(x, dtype=np.float64)
    N, C, T = x.shape
    H, Co = W1.shape[0], W2.shape[0]
    g = np.zeros((N, H, T))
    for n in range(N):
        for j in range(H):
            for t in range(T):
                acc = 0.0 if b1 is None else float(b1[j])
                for c in range(C):
                    for s in range(T):
                        acc += float(W1[j, c, (t - s) % T]) * float(x[n, c, s])
                g[n, j, t] = float(gelu(np.float64(acc)))
    y = np.zeros((N, Co, T))
    for n in range(N):
        for o in range(Co):
            for t in range(T):
                acc = 0.0 if b2 is None else float(b2[o])
                for j in range(H):
                    for s in range(T):
                        acc += float(W2[o, j, (t - s) % T]) * g[n, j, s]
                y[n, o, t] = acc
    return y


def composed_weight(W2: np.ndarray, W1: np.ndarray) -> np.ndarray:
    """W[o,c,u] = sum_j sum_v W2[o,j,v] W1[j,c,(u-v) mod 4]: two EQ-Linear layers in a
    row with no nonlinearity are one, whose kernel is the group convolution of the two."""
    T = W1.shape[2]
    Co, C = W2.shape[0], W1.shape[1]
    W = np.zeros((Co, C, T))
    for u in range(T):
        for v in range(T):
            W[:, :, u] += W2[:, :, v].astype(np.float64) @ W1[:, :, (u - v) % T].astype(np.float64)
    return W


def macs(N: int, C: int, H: int, Co: int) -> tuple[int, int]:
    """Real multiply-accumulates of the block: (Fourier route, dense unrolled route)."""
    return 6 * N * H * (C + Co), 16 * N * H * (C + Co)


rel_err = P4.rel_err
