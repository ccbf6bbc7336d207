"""Workload shapes and seeded synthetic inputs for the EQ-Linear layer (p4 and C_8).

This module holds no arithmetic of the method: it only draws random numbers
and rounds them to the compute dtype.  Both the CUDA path (through the tests
and the benchmark) and the float64 oracle consume exactly the rounded arrays
produced here.

Recipe.  Layout x[N,C,T], W[D,C,T], b[D], dy[N,D,T] (group index innermost,
T = 4 for p4, 8 for the cyclic group C_8).  Values are drawn in float64 with
numpy's PCG64 generator and rounded (round-to-nearest-even) to the mode dtype:

* x, dy ~ N(0, 1)
* W ~ N(0, variance 1/(T C)), i.e. std 1/sqrt(T C): the fan-in of the
  unrolled TC-wide layer, so that Var(y) is about 1 (1/(2 sqrt C) for p4)
* b ~ N(0, std 0.02)

Seeds: 20260000 + 100 * workload_id + {x: 0, W: 1, b: 2, dy: 3}.

MLP block (fc1: C -> H, GELU, fc2: H -> Co; p4): x ~ N(0, 1); W1 std
1/(2 sqrt C), W2 std 1/(2 sqrt H) (the fan-ins 4C and 4H); b1, b2 std 0.02.
Seeds: 20260000 + 100 * workload_id + {x: 0, W1: 1, b1: 2, W2: 4, b2: 5}.

The shapes stand in for the token streams of the networks the paper
evaluates (Flash EQ-ViT and Flash EQ-Swin, technical summary "Livello di
Rete"): a ViT MLP fc1 at 64 x 197 tokens and a Swin stage-1 stream at
128 x 3136 tokens; no dataset is involved.  The C_8 workload keeps the Swin
stream's token count and unrolled widths (96 -> 384) with T = 8.  The MLP
workload is the Swin-T stage-1 block (96 -> 384 -> 96 unrolled) on the same
token stream (and the ViT-Ti block, 192 -> 768 -> 192, at the ViT batch), and the p4m workload the same stream for the point group D4
(8 group elements: rotations and reflections, element (r, m) at index 4 m + r).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    wid: int            # workload id (used in the seeds)
    name: str
    N: int              # tokens
    C: int              # input channels per group element
    D: int              # output channels per group element
    dtype: str          # "fp16" or "fp32"
    passes: tuple       # subset of ("fwd", "dx", "dw")
    note: str
    T: int = 4          # group order
    group: str = "cyclic"  # "cyclic" (C_T) or "p4m" (point group D4, T = 8)


WORKLOADS = {
    1: Workload(1, "p4_fwd_fp32_N256_C16_D16", 256, 16, 16, "fp32", ("fwd",),
                "small forward, fp32 (64->64 unrolled)"),
    2: Workload(2, "p4_fwd_fp16_vit_fc1_N12608_C48_D192", 12608, 48, 192, "fp16", ("fwd",),
                "ViT MLP fc1-like forward, 64x197 tokens (192->768 unrolled)"),
    3: Workload(3, "p4_fwd_fp16_square_N65536_C192_D192", 65536, 192, 192, "fp16", ("fwd",),
                "square forward (768->768 unrolled); also run in fp32 mode"),
    4: Workload(4, "p4_bwd_fp16_N32768_C256_D256", 32768, 256, 256, "fp16", ("dx", "dw"),
                "backward dX and dW (1024->1024 unrolled)"),
    5: Workload(5, "p4_fwdbwd_fp16_swin_N401408_C24_D96", 401408, 24, 96, "fp16",
                ("fwd", "dx", "dw"),
                "Swin stage-1-like forward+backward, 128x3136 tokens (96->384 unrolled)"),
    6: Workload(6, "c8_fwdbwd_fp16_swin_N401408_C12_D48", 401408, 12, 48, "fp16",
                ("fwd", "dx", "dw"),
                "cyclic group C_8, Swin stage-1-like stream (96->384 unrolled)", T=8),
    8: Workload(8, "p4m_fwdbwd_fp16_swin_N401408_C12_D48", 401408, 12, 48, "fp16",
                ("fwd", "dx", "dw"),
                "p4m (rotations and reflections, D4), Swin stage-1-like stream (96->384 unrolled)",
                T=8, group="p4m"),
    7: Workload(7, "p4_mlp_fp16_swin_N401408_C24_H96", 401408, 24, 96, "fp16", ("mlp",),
                "Swin stage-1-like MLP block fc1 -> GELU -> fc2 (96->384->96 unrolled); "
                "D is the hidden width, the output has C channels"),
    10: Workload(10, "c6_fwdbwd_fp16_swin_N401408_C16_D64", 401408, 16, 64, "fp16",
                 ("fwd", "dx", "dw"),
                 "cyclic group C_6 (non-dyadic twiddles, 12-byte fibres), Swin stage-1-like "
                 "stream (96->384 unrolled)", T=6),
    9: Workload(9, "p4_mlp_fp16_vit_ti_N12608_C48_H192", 12608, 48, 192, "fp16", ("mlp",),
                "ViT-Ti-like MLP block at 64x197 tokens (192->768->192 unrolled; weights "
                "streamed); D is the hidden width, the output has C channels"),
}


def np_dtype(dtype: str):
    return {"fp16": np.float16, "fp32": np.float32, "fp64": np.float64}[dtype]


def _normal(seed: int, shape, std: float, dtype: str) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    v = rng.standard_normal(size=shape, dtype=np.float64)
    if std != 1.0:
        v *= std
    return v.astype(np_dtype(dtype))


def make_inputs(wid: int, N: int, C: int, D: int, dtype: str,
                which=("x", "W", "b", "dy"), T: int = 4) -> dict:
    """Seeded, dtype-rounded inputs for a layer of the given shape.

    ``wid`` selects the seed block; any shape may be drawn with it (small
    parity cases reuse a workload's seeds at reduced sizes).
    """
    base = 20260000 + 100 * wid
    out = {}
    if "x" in which:
        out["x"] = _normal(base + 0, (N, C, T), 1.0, dtype)
    if "W" in which:
        out["W"] = _normal(base + 1, (D, C, T), 1.0 / np.sqrt(T * C), dtype)
    if "b" in which:
        out["b"] = _normal(base + 2, (D,), 0.02, dtype)
    if "dy" in which:
        out["dy"] = _normal(base + 3, (N, D, T), 1.0, dtype)
    return out


def workload_inputs(wid: int, dtype: str | None = None, N: int | None = None,
                    which=("x", "W", "b", "dy")) -> dict:
    w = WORKLOADS[wid]
    return make_inputs(wid, w.N if N is None else N, w.C, w.D, dtype or w.dtype, which, T=w.T)


def make_mlp_inputs(wid: int, N: int, C: int, H: int, Co: int, dtype: str) -> dict:
    """Seeded, dtype-rounded inputs of the MLP block (x, W1, b1, W2, b2)."""
    base = 20260000 + 100 * wid
    return {"x": _normal(base + 0, (N, C, 4), 1.0, dtype),
            "W1": _normal(base + 1, (H, C, 4), 1.0 / np.sqrt(4 * C), dtype),
            "b1": _normal(base + 2, (H,), 0.02, dtype),
            "W2": _normal(base + 4, (Co, H, 4), 1.0 / np.sqrt(4 * H), dtype),
            "b2": _normal(base + 5, (Co,), 0.02, dtype)}


def make_mlp_range_inputs(wid: int, N: int, C: int, H: int, Co: int, x, W1, W2,
                          b1_std: float = 0.02, b2_std: float = 0.02) -> dict:
    """fp16 inputs of the MLP block at the edges of the half-precision range.

    Each of x, W1, W2 is given either as a float s (normal values, N(0, s^2))
    or as a pair (lo, hi) (magnitudes uniform in [lo, hi] with random signs);
    b1 ~ N(0, b1_std^2), b2 ~ N(0, b2_std^2).
    Seeds: 20260000 + 100 * wid + {x: 0, W1: 1, b1: 2, W2: 4, b2: 5}.
    """
    base = 20260000 + 100 * wid

    def draw(seed, shape, spec):
        if isinstance(spec, tuple):
            return _magnitude(seed, shape, spec[0], spec[1], "fp16")
        return _normal(seed, shape, spec, "fp16")

    return {"x": draw(base + 0, (N, C, 4), x),
            "W1": draw(base + 1, (H, C, 4), W1),
            "b1": _normal(base + 2, (H,), b1_std, "fp16"),
            "W2": draw(base + 4, (Co, H, 4), W2),
            "b2": _normal(base + 5, (Co,), b2_std, "fp16")}


def _magnitude(seed: int, shape, lo: float, hi: float, dtype: str) -> np.ndarray:
    """Values with |v| uniform in [lo, hi] and a random sign (seeded)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    mag = rng.uniform(lo, hi, size=shape)
    sign = np.where(rng.integers(0, 2, size=shape) == 1, 1.0, -1.0)
    return (sign * mag).astype(np_dtype(dtype))


def make_range_inputs(wid: int, N: int, C: int, D: int, x_range, dy_range,
                      w_std: float, b_std: float = 0.02, T: int = 4) -> dict:
    """fp16 inputs at the edges of the half-precision range.

    x and dy have magnitudes uniform in x_range / dy_range (pairs (lo, hi)) with
    random signs; W ~ N(0, w_std^2), b ~ N(0, b_std^2).  Used to check that the
    fp16 path handles every finite fp16 input (large ones whose group-axis sums
    leave the fp16 range, and small ones near the subnormals) as long as the
    outputs themselves are representable: the caller picks w_std and the other
    operand's range so that y, dx and dW stay finite.
    Seeds: 20260000 + 100 * wid + {x: 0, W: 1, b: 2, dy: 3}.
    """
    base = 20260000 + 100 * wid
    return {"x": _magnitude(base + 0, (N, C, T), *x_range, "fp16"),
            "W": _normal(base + 1, (D, C, T), w_std, "fp16"),
            "b": _normal(base + 2, (D,), b_std, "fp16"),
            "dy": _magnitude(base + 3, (N, D, T), *dy_range, "fp16")}
