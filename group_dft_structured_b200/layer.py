"""Torch-facing convenience around the C ABI: allocates outputs, the Fourier
weight buffer and the dW workspace with torch (device memory only) and calls
the library.  No arithmetic happens here.
"""

from __future__ import annotations

import torch

from . import (FEQL_FP16, FEQL_FP16_SIMT, feql_backward, feql_backward_dw,
               feql_backward_dw_workspace_bytes, feql_backward_dx, feql_ct_backward_dw,
               feql_ct_backward_dw_workspace_bytes, feql_ct_backward_dx, feql_ct_forward,
               feql_ct_weight_fft, feql_ct_weight_fft_bytes, feql_forward, feql_mlp_forward,
               feql_mlp_weight_fft, feql_mlp_weight_fft_bytes, feql_p4m_backward_dw,
               feql_p4m_backward_dw_workspace_bytes, feql_p4m_backward_dx, feql_p4m_forward,
               feql_p4m_weight_fft, feql_p4m_weight_fft_bytes, feql_weight_fft,
               feql_weight_fft_bytes)


def torch_dtype(mode: int):
    return torch.float16 if mode in (FEQL_FP16, FEQL_FP16_SIMT) else torch.float32


def weight_fft(W: torch.Tensor, mode: int, stream=None) -> torch.Tensor:
    D, C, _ = W.shape
    nbytes = feql_weight_fft_bytes(C, D, mode)
    if nbytes == 0:
        raise ValueError("unsupported (C, D, mode)")
    What = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    feql_weight_fft(W, What, C, D, mode, stream)
    return What


def forward(x: torch.Tensor, What: torch.Tensor, b, D: int, mode: int, out=None,
            stream=None) -> torch.Tensor:
    N, C, _ = x.shape
    y = out if out is not None else torch.empty((N, D, 4), dtype=x.dtype, device=x.device)
    feql_forward(x, What, b, y, N, C, D, mode, stream)
    return y


def backward_dx(dy: torch.Tensor, What: torch.Tensor, C: int, mode: int, out=None,
                stream=None) -> torch.Tensor:
    N, D, _ = dy.shape
    dx = out if out is not None else torch.empty((N, C, 4), dtype=dy.dtype, device=dy.device)
    feql_backward_dx(dy, What, dx, N, C, D, mode, stream)
    return dx


def dw_workspace(N: int, C: int, D: int, mode: int, device) -> torch.Tensor:
    nbytes = feql_backward_dw_workspace_bytes(N, C, D, mode)
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def backward(x: torch.Tensor, dy: torch.Tensor, What: torch.Tensor, mode: int, ws=None,
             with_db: bool = True, stream=None):
    """dx, dW, db from one call (fused single pass over dy where supported)."""
    N, C, _ = x.shape
    D = dy.shape[1]
    if ws is None:
        ws = dw_workspace(N, C, D, mode, x.device)
    dx = torch.empty((N, C, 4), dtype=x.dtype, device=x.device)
    dW = torch.empty((D, C, 4), dtype=x.dtype, device=x.device)
    db = torch.empty((D,), dtype=x.dtype, device=x.device) if with_db else None
    feql_backward(x, dy, What, dx, dW, db, ws, ws.numel(), N, C, D, mode, stream)
    return dx, dW, db


def backward_dw(x: torch.Tensor, dy: torch.Tensor, mode: int, ws=None, out=None,
                with_db: bool = True, stream=None):
    N, C, _ = x.shape
    D = dy.shape[1]
    if ws is None:
        ws = dw_workspace(N, C, D, mode, x.device)
    if out is None:
        dW = torch.empty((D, C, 4), dtype=x.dtype, device=x.device)
        db = torch.empty((D,), dtype=x.dtype, device=x.device) if with_db else None
    else:
        dW, db = out
    feql_backward_dw(x, dy, dW, db, ws, ws.numel(), N, C, D, mode, stream)
    return dW, db


# --------------------------------------------------------- cyclic group C_T
# The group order T is the length of the last axis (T = 4 goes to the p4 path).

def ct_weight_fft(W: torch.Tensor, mode: int, stream=None) -> torch.Tensor:
    D, C, T = W.shape
    nbytes = feql_ct_weight_fft_bytes(T, C, D, mode)
    if nbytes == 0:
        raise ValueError("unsupported (T, C, D, mode)")
    What = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    feql_ct_weight_fft(T, W, What, C, D, mode, stream)
    return What


def ct_forward(x: torch.Tensor, What: torch.Tensor, b, D: int, mode: int, stream=None):
    N, C, T = x.shape
    y = torch.empty((N, D, T), dtype=x.dtype, device=x.device)
    feql_ct_forward(T, x, What, b, y, N, C, D, mode, stream)
    return y


def ct_backward_dx(dy: torch.Tensor, What: torch.Tensor, C: int, mode: int, stream=None):
    N, D, T = dy.shape
    dx = torch.empty((N, C, T), dtype=dy.dtype, device=dy.device)
    feql_ct_backward_dx(T, dy, What, dx, N, C, D, mode, stream)
    return dx


def ct_backward_dw(x: torch.Tensor, dy: torch.Tensor, mode: int, with_db: bool = True,
                   stream=None):
    N, C, T = x.shape
    D = dy.shape[1]
    nbytes = feql_ct_backward_dw_workspace_bytes(T, N, C, D, mode)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    dW = torch.empty((D, C, T), dtype=x.dtype, device=x.device)
    db = torch.empty((D,), dtype=x.dtype, device=x.device) if with_db else None
    feql_ct_backward_dw(T, x, dy, dW, db, ws, ws.numel(), N, C, D, mode, stream)
    return dW, db


# --------------------------------------------------------- p4m (D4, order 8)

def p4m_weight_fft(W: torch.Tensor, mode: int, stream=None) -> torch.Tensor:
    D, C, _ = W.shape
    nbytes = feql_p4m_weight_fft_bytes(C, D, mode)
    if nbytes == 0:
        raise ValueError("unsupported (C, D, mode) for p4m")
    What = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    feql_p4m_weight_fft(W, What, C, D, mode, stream)
    return What


def p4m_forward(x: torch.Tensor, What: torch.Tensor, b, D: int, mode: int, stream=None):
    N, C, _ = x.shape
    y = torch.empty((N, D, 8), dtype=x.dtype, device=x.device)
    feql_p4m_forward(x, What, b, y, N, C, D, mode, stream)
    return y


def p4m_backward_dx(dy: torch.Tensor, What: torch.Tensor, C: int, mode: int, stream=None):
    N, D, _ = dy.shape
    dx = torch.empty((N, C, 8), dtype=dy.dtype, device=dy.device)
    feql_p4m_backward_dx(dy, What, dx, N, C, D, mode, stream)
    return dx


def p4m_backward_dw(x: torch.Tensor, dy: torch.Tensor, mode: int, with_db: bool = True,
                    stream=None):
    N, C, _ = x.shape
    D = dy.shape[1]
    nbytes = feql_p4m_backward_dw_workspace_bytes(N, C, D, mode)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    dW = torch.empty((D, C, 8), dtype=x.dtype, device=x.device)
    db = torch.empty((D,), dtype=x.dtype, device=x.device) if with_db else None
    feql_p4m_backward_dw(x, dy, dW, db, ws, ws.numel(), N, C, D, mode, stream)
    return dW, db


# ------------------------------------------------------------ MLP block (p4)

def mlp_weight_fft(W1: torch.Tensor, W2: torch.Tensor, mode: int, stream=None) -> torch.Tensor:
    H, C, _ = W1.shape
    Co = W2.shape[0]
    nbytes = feql_mlp_weight_fft_bytes(C, H, Co, mode)
    if nbytes == 0:
        raise ValueError("unsupported (C, H, Co, mode) for the fused MLP block")
    What = torch.empty(nbytes, dtype=torch.uint8, device=W1.device)
    feql_mlp_weight_fft(W1, W2, What, C, H, Co, mode, stream)
    return What


def mlp_forward(x: torch.Tensor, What: torch.Tensor, b1, b2, H: int, Co: int, mode: int,
                stream=None) -> torch.Tensor:
    N, C, _ = x.shape
    y = torch.empty((N, Co, 4), dtype=x.dtype, device=x.device)
    feql_mlp_forward(x, What, b1, b2, y, N, C, H, Co, mode, stream)
    return y
