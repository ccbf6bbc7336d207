"""Drop-in PyTorch module for the equivariant linear layer of the cyclic group
C_T (T = 4: the rotation group p4; any T in 2..16, T = 6 and 8 on the tensor
cores) and of p4m (rotations and reflections, point group D4), with autograd.

Flash EQ-Linear (arXiv abstract) presents the method as a plug-and-play
replacement for the EQ-Linear layers of existing equivariant models: the layer
computes the same function as the naive form, an ``nn.Linear`` whose (T*D) x
(T*C) weight is the group-circulant unrolling of W[D][C][T],

    A[d*T + t, c*T + s] = W[d, c, (t - s) mod T],   bias[d*T + t] = b[d],

acting on features laid out as (channel, group element) with the group index
innermost.  For p4m (group="p4m", 8 elements (r, m) at index 4 m + r) the
unrolling is A[d*8 + g, c*8 + h] = W[d, c, h^-1 g].  ``EqLinear.from_unrolled``
takes such a dense layer apart into (W, b); ``EqLinear.forward`` runs the
library's kernels.

Argument marshalling only: every step of the forward and backward passes runs
in libfeql.so through the C ABI (``layer`` allocates outputs with torch).
Tensors must live on a CUDA device; there is no CPU path.
"""

from __future__ import annotations

import math

import torch

from . import FEQL_FP16, FEQL_FP32
from . import layer as _L


def mode_for(dtype: torch.dtype) -> int:
    if dtype == torch.float16:
        return FEQL_FP16
    if dtype == torch.float32:
        return FEQL_FP32
    raise TypeError(f"EqLinear computes in float16 or float32, not {dtype}")


def _p4m_index(r: int, m: int) -> int:
    return 4 * m + (r % 4)


def p4m_kernel_index(g: int, h: int) -> int:
    """Index of h^-1 g in p4m's point group D4, elements (r, m) at 4 m + r."""
    rg, mg = g % 4, g // 4
    rh, mh = h % 4, h // 4
    return _p4m_index((-1) ** mh * (rg - rh), mh ^ mg)


class EqLinearFunction(torch.autograd.Function):
    """y[n,d,t] = b[d] + sum_c sum_s W[d,c,(t-s) mod T] x[n,c,s] on (N, C, T) tensors
    (group "cyclic"), or the p4m group convolution W[d,c,h^-1 g] (group "p4m").

    ``What`` is the layer's Fourier weight buffer (``layer.ct_weight_fft`` of W),
    passed in so that callers can reuse it while W is unchanged.  Backward
    returns the gradients autograd asks for: dx from the dX pass, dW and db from
    the dW pass; for p4 with all of them needed, from the fused single pass.
    """

    @staticmethod
    def forward(ctx, x, W, b, What, mode: int, group: str = "cyclic"):
        D = W.shape[0]
        y = (_L.p4m_forward(x, What, b, D, mode) if group == "p4m"
             else _L.ct_forward(x, What, b, D, mode))
        ctx.save_for_backward(x, What)
        ctx.mode = mode
        ctx.group = group
        ctx.shape = (x.shape[1], D, x.shape[2])
        return y

    @staticmethod
    def backward(ctx, dy):
        x, What = ctx.saved_tensors
        C, D, T = ctx.shape
        need_x, need_W, need_b = ctx.needs_input_grad[:3]
        dy = dy.contiguous()
        dx = dW = db = None
        if ctx.group == "p4m":
            if need_x:
                dx = _L.p4m_backward_dx(dy, What, C, ctx.mode)
            if need_W or need_b:
                dW, db = _L.p4m_backward_dw(x, dy, ctx.mode, with_db=need_b)
        elif T == 4 and need_x and need_W:
            dx, dW, db = _L.backward(x, dy, What, ctx.mode, with_db=need_b)
        else:
            if need_x:
                dx = _L.ct_backward_dx(dy, What, C, ctx.mode)
            if need_W or need_b:
                dW, db = _L.ct_backward_dw(x, dy, ctx.mode, with_db=need_b)
        return dx, (dW if need_W else None), (db if need_b else None), None, None, None


class EqLinear(torch.nn.Module):
    """Equivariant linear layer of C_T (or p4m) on features (..., C*T), group index innermost.

    Parameters: ``weight`` [D][C][T] and ``bias`` [D] (or None), in float16
    (any T; the tensor cores serve T = 4, 8, p4m, and 6 with C and D multiples
    of 4) or float32.  ``group="p4m"`` selects the point
    group D4 (T = 8: rotations (r, 0) at 0..3, reflected (r, 1) at 4..7).  The
    Fourier weight buffer is rebuilt when the weight changes (tracked by its
    storage and version counter), so it is computed once per optimizer step, or
    once for inference.
    """

    def __init__(self, in_channels: int, out_channels: int, group_order: int = 4,
                 bias: bool = True, dtype: torch.dtype = torch.float16, device=None,
                 group: str = "cyclic"):
        super().__init__()
        if group not in ("cyclic", "p4m"):
            raise ValueError(f"group is 'cyclic' or 'p4m', not {group!r}")
        if group == "p4m" and group_order != 8:
            raise ValueError("p4m has 8 group elements")
        self.group = group
        self.in_channels, self.out_channels = in_channels, out_channels
        self.group_order = group_order
        mode_for(dtype)
        self.weight = torch.nn.Parameter(
            torch.empty((out_channels, in_channels, group_order), dtype=dtype, device=device))
        self.bias = (torch.nn.Parameter(torch.empty((out_channels,), dtype=dtype, device=device))
                     if bias else None)
        self._what = None
        self._what_key = None
        self.reset_parameters()

    def reset_parameters(self) -> None:
        # the bound nn.Linear uses for the unrolled layer: fan-in T*C
        bound = 1.0 / math.sqrt(self.group_order * self.in_channels)
        with torch.no_grad():
            self.weight.uniform_(-bound, bound)
            if self.bias is not None:
                self.bias.uniform_(-bound, bound)

    def fourier_weight(self) -> torch.Tensor:
        W = self.weight
        key = (W.device, W.dtype, W.data_ptr(), W._version, tuple(W.shape))
        if self._what is None or self._what_key != key:
            with torch.no_grad():
                Wc = W.detach().contiguous()
                self._what = (_L.p4m_weight_fft(Wc, mode_for(W.dtype)) if self.group == "p4m"
                              else _L.ct_weight_fft(Wc, mode_for(W.dtype)))
            self._what_key = key
        return self._what

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        C, D, T = self.in_channels, self.out_channels, self.group_order
        if x.shape[-1] != C * T:
            raise ValueError(f"expected features of size C*T = {C * T}, got {x.shape[-1]}")
        if not x.is_cuda:
            raise RuntimeError("EqLinear runs on CUDA tensors only (libfeql.so kernels)")
        lead = x.shape[:-1]
        x3 = x.reshape(-1, C, T).contiguous()
        if x3.dtype != self.weight.dtype:
            raise TypeError(f"input dtype {x3.dtype} differs from the weight's {self.weight.dtype}")
        y = EqLinearFunction.apply(x3, self.weight, self.bias, self.fourier_weight(),
                                   mode_for(self.weight.dtype), self.group)
        return y.reshape(*lead, D * T)

    def extra_repr(self) -> str:
        return (f"in_channels={self.in_channels}, out_channels={self.out_channels}, "
                f"group_order={self.group_order}, group={self.group}, "
                f"bias={self.bias is not None}")

    @classmethod
    def from_unrolled(cls, weight: torch.Tensor, bias: torch.Tensor | None, group_order: int,
                      atol: float = 0.0, group: str = "cyclic") -> "EqLinear":
        """The layer equal to the dense (T*D) x (T*C) map ``weight`` (+ ``bias``).

        ``weight`` must be group-circulant in the layout above (entries that
        should be equal may differ by ``atol``) and ``bias`` constant over the
        group index; otherwise ValueError.  Parameters keep weight's dtype and
        device.
        """
        T = group_order
        rows, cols = weight.shape
        if rows % T or cols % T:
            raise ValueError(f"dense shape {tuple(weight.shape)} is not a multiple of T = {T}")
        D, C = rows // T, cols // T
        A = weight.detach().reshape(D, T, C, T)  # [d][t][c][s]
        W = A[:, :, :, 0].permute(0, 2, 1).contiguous()  # W[d,c,u] = A[d, u, c, s=e]
        if group == "p4m":
            if T != 8:
                raise ValueError("p4m has 8 group elements")
            u = torch.tensor([[p4m_kernel_index(g, h) for h in range(8)] for g in range(8)],
                             device=weight.device)  # u[g][h] = h^-1 g
        else:
            t = torch.arange(T, device=weight.device)
            u = (t[:, None] - t[None, :]) % T  # u[t][s] = (t - s) mod T
        rebuilt = W[:, :, u].permute(0, 2, 1, 3)  # [d][t][c][s] = W[d, c, (t-s) mod T]
        if not torch.allclose(rebuilt, A, rtol=0.0, atol=atol):
            raise ValueError("weight is not group-circulant for this T")
        b = None
        if bias is not None:
            B = bias.detach().reshape(D, T)
            if not torch.allclose(B, B[:, :1].expand(D, T), rtol=0.0, atol=atol):
                raise ValueError("bias is not constant over the group index")
            b = B[:, 0].contiguous()
        m = cls(C, D, T, bias=b is not None, dtype=weight.dtype, device=weight.device,
                group=group)
        with torch.no_grad():
            m.weight.copy_(W)
            if b is not None:
                m.bias.copy_(b)
        return m
