"""Python binding of libfeql.so — the B200 (sm_100a) p4 Flash EQ-Linear kernels.

Argument marshalling only: each function below forwards to the C entry point
of the same name declared in include/feql.h; every step of the computation
runs in the library's CUDA kernels.  Tensors (torch) or raw integer device
addresses are accepted; ``stream`` is a torch.cuda.Stream, a raw cudaStream_t
integer, or None for torch's current stream.  A non-OK status raises
FeqlError.  There is no fallback: if the library is missing, importing any
compute function raises.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfeql.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "feql.h")

FEQL_FP16 = 0
FEQL_FP32 = 1
FEQL_FP32_SIMT = 2
FEQL_FP32_3XTF32 = 3
FEQL_FP16_SIMT = 4

FEQL_OK = 0
FEQL_ERR_INVALID_ARG = 1
FEQL_ERR_UNSUPPORTED = 2
FEQL_ERR_CUDA = 3
FEQL_ERR_TIMEOUT = 4

DTYPES = {"fp16": FEQL_FP16, "fp32": FEQL_FP32, "fp32_simt": FEQL_FP32_SIMT,
          "fp32_3xtf32": FEQL_FP32_3XTF32, "fp16_simt": FEQL_FP16_SIMT}


class FeqlError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {feql_status_string(status)} (status {status})")


_lib = None

_VP = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "feql_weight_fft_bytes": (_SZ, [_I, _I, _I]),
    "feql_weight_fft": (_I, [_VP, _VP, _I, _I, _I, _VP]),
    "feql_forward": (_I, [_VP, _VP, _VP, _VP, _I64, _I, _I, _I, _VP]),
    "feql_backward_dx": (_I, [_VP, _VP, _VP, _I64, _I, _I, _I, _VP]),
    "feql_backward_dw_workspace_bytes": (_SZ, [_I64, _I, _I, _I]),
    "feql_backward_dw": (_I, [_VP, _VP, _VP, _VP, _VP, _SZ, _I64, _I, _I, _I, _VP]),
    "feql_backward": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _I64, _I, _I, _I, _VP]),
    "feql_backward_dw_noalloc": (_I, [_VP, _VP, _VP, _VP, _I64, _I, _I, _I, _VP]),
    "feql_ct_weight_fft_bytes": (_SZ, [_I, _I, _I, _I]),
    "feql_ct_weight_fft": (_I, [_I, _VP, _VP, _I, _I, _I, _VP]),
    "feql_ct_forward": (_I, [_I, _VP, _VP, _VP, _VP, _I64, _I, _I, _I, _VP]),
    "feql_ct_backward_dx": (_I, [_I, _VP, _VP, _VP, _I64, _I, _I, _I, _VP]),
    "feql_ct_backward_dw_workspace_bytes": (_SZ, [_I, _I64, _I, _I, _I]),
    "feql_ct_backward_dw": (_I, [_I, _VP, _VP, _VP, _VP, _VP, _SZ, _I64, _I, _I, _I, _VP]),
    "feql_p4m_weight_fft_bytes": (_SZ, [_I, _I, _I]),
    "feql_p4m_weight_fft": (_I, [_VP, _VP, _I, _I, _I, _VP]),
    "feql_p4m_forward": (_I, [_VP, _VP, _VP, _VP, _I64, _I, _I, _I, _VP]),
    "feql_p4m_backward_dx": (_I, [_VP, _VP, _VP, _I64, _I, _I, _I, _VP]),
    "feql_p4m_backward_dw_workspace_bytes": (_SZ, [_I64, _I, _I, _I]),
    "feql_p4m_backward_dw": (_I, [_VP, _VP, _VP, _VP, _VP, _SZ, _I64, _I, _I, _I, _VP]),
    "feql_mlp_weight_fft_bytes": (_SZ, [_I, _I, _I, _I]),
    "feql_mlp_weight_fft": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    "feql_mlp_forward": (_I, [_VP, _VP, _VP, _VP, _VP, _I64, _I, _I, _I, _I, _VP]),
    "feql_device_status": (_I, [_VP]),
    "feql_status_string": (ctypes.c_char_p, [_I]),
}


def load(path: str = LIB_PATH):
    """Loads libfeql.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libfeql.so not built ({path}); run "
                               "python -m group_dft_structured_b200.build")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str) -> None:
    if st != FEQL_OK:
        raise FeqlError(st, where)


def feql_status_string(status: int) -> str:
    return load().feql_status_string(status).decode()


def feql_weight_fft_bytes(C: int, D: int, dtype: int) -> int:
    return int(load().feql_weight_fft_bytes(C, D, dtype))


def feql_weight_fft(W, What, C: int, D: int, dtype: int, stream=None) -> None:
    _check(load().feql_weight_fft(_ptr(W), _ptr(What), C, D, dtype, _stream(stream)),
           "feql_weight_fft")


def feql_forward(x, What, b, y, N: int, C: int, D: int, dtype: int, stream=None) -> None:
    _check(load().feql_forward(_ptr(x), _ptr(What), _ptr(b), _ptr(y), N, C, D, dtype,
                               _stream(stream)), "feql_forward")


def feql_backward_dx(dy, What, dx, N: int, C: int, D: int, dtype: int, stream=None) -> None:
    _check(load().feql_backward_dx(_ptr(dy), _ptr(What), _ptr(dx), N, C, D, dtype,
                                   _stream(stream)), "feql_backward_dx")


def feql_backward_dw_workspace_bytes(N: int, C: int, D: int, dtype: int) -> int:
    return int(load().feql_backward_dw_workspace_bytes(N, C, D, dtype))


def feql_backward_dw(x, dy, dW, db, ws, ws_bytes: int, N: int, C: int, D: int, dtype: int,
                     stream=None) -> None:
    _check(load().feql_backward_dw(_ptr(x), _ptr(dy), _ptr(dW), _ptr(db), _ptr(ws), ws_bytes,
                                   N, C, D, dtype, _stream(stream)), "feql_backward_dw")


def feql_backward(x, dy, What, dx, dW, db, ws, ws_bytes: int, N: int, C: int, D: int,
                  dtype: int, stream=None) -> None:
    _check(load().feql_backward(_ptr(x), _ptr(dy), _ptr(What), _ptr(dx), _ptr(dW), _ptr(db),
                                _ptr(ws), ws_bytes, N, C, D, dtype, _stream(stream)),
           "feql_backward")


def feql_backward_dw_noalloc(x, dy, dW, db, N: int, C: int, D: int, dtype: int,
                             stream=None) -> None:
    """Weight gradient without a workspace argument, for callers that cannot
    allocate device memory; scratch comes from a fixed array in the library
    (see include/feql.h for the size limit and the no-overlap rule)."""
    _check(load().feql_backward_dw_noalloc(_ptr(x), _ptr(dy), _ptr(dW), _ptr(db), N, C, D,
                                           dtype, _stream(stream)), "feql_backward_dw_noalloc")


def feql_ct_weight_fft_bytes(T: int, C: int, D: int, dtype: int) -> int:
    return int(load().feql_ct_weight_fft_bytes(T, C, D, dtype))


def feql_ct_weight_fft(T: int, W, What, C: int, D: int, dtype: int, stream=None) -> None:
    _check(load().feql_ct_weight_fft(T, _ptr(W), _ptr(What), C, D, dtype, _stream(stream)),
           "feql_ct_weight_fft")


def feql_ct_forward(T: int, x, What, b, y, N: int, C: int, D: int, dtype: int,
                    stream=None) -> None:
    _check(load().feql_ct_forward(T, _ptr(x), _ptr(What), _ptr(b), _ptr(y), N, C, D, dtype,
                                  _stream(stream)), "feql_ct_forward")


def feql_ct_backward_dx(T: int, dy, What, dx, N: int, C: int, D: int, dtype: int,
                        stream=None) -> None:
    _check(load().feql_ct_backward_dx(T, _ptr(dy), _ptr(What), _ptr(dx), N, C, D, dtype,
                                      _stream(stream)), "feql_ct_backward_dx")


def feql_ct_backward_dw_workspace_bytes(T: int, N: int, C: int, D: int, dtype: int) -> int:
    return int(load().feql_ct_backward_dw_workspace_bytes(T, N, C, D, dtype))


def feql_ct_backward_dw(T: int, x, dy, dW, db, ws, ws_bytes: int, N: int, C: int, D: int,
                        dtype: int, stream=None) -> None:
    _check(load().feql_ct_backward_dw(T, _ptr(x), _ptr(dy), _ptr(dW), _ptr(db), _ptr(ws),
                                      ws_bytes, N, C, D, dtype, _stream(stream)),
           "feql_ct_backward_dw")


def feql_p4m_weight_fft_bytes(C: int, D: int, dtype: int) -> int:
    return int(load().feql_p4m_weight_fft_bytes(C, D, dtype))


def feql_p4m_weight_fft(W, What, C: int, D: int, dtype: int, stream=None) -> None:
    _check(load().feql_p4m_weight_fft(_ptr(W), _ptr(What), C, D, dtype, _stream(stream)),
           "feql_p4m_weight_fft")


def feql_p4m_forward(x, What, b, y, N: int, C: int, D: int, dtype: int, stream=None) -> None:
    _check(load().feql_p4m_forward(_ptr(x), _ptr(What), _ptr(b), _ptr(y), N, C, D, dtype,
                                   _stream(stream)), "feql_p4m_forward")


def feql_p4m_backward_dx(dy, What, dx, N: int, C: int, D: int, dtype: int, stream=None) -> None:
    _check(load().feql_p4m_backward_dx(_ptr(dy), _ptr(What), _ptr(dx), N, C, D, dtype,
                                       _stream(stream)), "feql_p4m_backward_dx")


def feql_p4m_backward_dw_workspace_bytes(N: int, C: int, D: int, dtype: int) -> int:
    return int(load().feql_p4m_backward_dw_workspace_bytes(N, C, D, dtype))


def feql_p4m_backward_dw(x, dy, dW, db, ws, ws_bytes: int, N: int, C: int, D: int, dtype: int,
                         stream=None) -> None:
    _check(load().feql_p4m_backward_dw(_ptr(x), _ptr(dy), _ptr(dW), _ptr(db), _ptr(ws), ws_bytes,
                                       N, C, D, dtype, _stream(stream)), "feql_p4m_backward_dw")


def feql_mlp_weight_fft_bytes(C: int, H: int, Co: int, dtype: int) -> int:
    return int(load().feql_mlp_weight_fft_bytes(C, H, Co, dtype))


def feql_mlp_weight_fft(W1, W2, What, C: int, H: int, Co: int, dtype: int, stream=None) -> None:
    _check(load().feql_mlp_weight_fft(_ptr(W1), _ptr(W2), _ptr(What), C, H, Co, dtype,
                                      _stream(stream)), "feql_mlp_weight_fft")


def feql_mlp_forward(x, What, b1, b2, y, N: int, C: int, H: int, Co: int, dtype: int,
                     stream=None) -> None:
    _check(load().feql_mlp_forward(_ptr(x), _ptr(What), _ptr(b1), _ptr(b2), _ptr(y), N, C, H, Co,
                                   dtype, _stream(stream)), "feql_mlp_forward")


def feql_device_status(stream=None) -> int:
    return int(load().feql_device_status(_stream(stream)))
