"""The drop-in module EqLinear: host-side logic on the CPU, and parity of its
forward and autograd backward against the float64 C_T oracle on the GPU.

Plug-and-play replacement (Flash EQ-Linear, arXiv abstract): a naive EQ-Linear
layer is an nn.Linear whose weight is the group-circulant unrolling of W; the
module must compute the same function and the same gradients.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import group_dft_structured_b200 as F
from group_dft_structured_b200.module import EqLinear, mode_for
from group_dft_structured_b200.workloads import make_inputs
from oracle import feql_ct_oracle as O
from oracle import feql_p4m_oracle as P4M


def dense_layer(W, b):
    """The naive layer's parameters: the oracle's unrolled matrix, bias repeated over t."""
    T = W.shape[2]
    A = O.unrolled_circulant(W.astype(np.float64))
    bd = None if b is None else np.repeat(b.astype(np.float64), T)
    return A, bd


# ------------------------------------------------------------------ CPU ---

@pytest.mark.parametrize("T", [4, 8, 3])
def test_from_unrolled_recovers_the_weights(T):
    rng = np.random.default_rng(70 + T)
    C, D = 5, 7
    W = rng.standard_normal((D, C, T)).astype(np.float32)
    b = rng.standard_normal(D).astype(np.float32)
    A, bd = dense_layer(W, b)
    m = EqLinear.from_unrolled(torch.from_numpy(A.astype(np.float32)),
                               torch.from_numpy(bd.astype(np.float32)), T)
    assert (m.in_channels, m.out_channels, m.group_order) == (C, D, T)
    assert m.weight.dtype == torch.float32
    assert np.array_equal(m.weight.detach().numpy(), W)
    assert np.array_equal(m.bias.detach().numpy(), b)


def test_unrolled_layout_is_the_layers_function():
    # the naive dense layer on (C*T)-features, group index innermost, is the layer
    rng = np.random.default_rng(71)
    N, C, D, T = 6, 3, 4, 8
    x = rng.standard_normal((N, C, T))
    W = rng.standard_normal((D, C, T))
    b = rng.standard_normal(D)
    A, bd = dense_layer(W, b)
    y_dense = x.reshape(N, C * T) @ A.T + bd
    assert np.allclose(y_dense, O.forward_bruteforce(x, W, b).reshape(N, D * T), atol=1e-12)


def test_from_unrolled_rejects_non_equivariant_layers():
    rng = np.random.default_rng(72)
    W = rng.standard_normal((3, 2, 4)).astype(np.float32)
    b = rng.standard_normal(3).astype(np.float32)
    A, bd = dense_layer(W, b)
    At = torch.from_numpy(A.astype(np.float32))
    bt = torch.from_numpy(bd.astype(np.float32))
    bad = At.clone()
    bad[1, 2] += 0.5
    with pytest.raises(ValueError):
        EqLinear.from_unrolled(bad, bt, 4)
    m = EqLinear.from_unrolled(bad, bt, 4, atol=1.0)  # within the caller's tolerance
    assert m.weight.shape == (3, 2, 4)
    badb = bt.clone()
    badb[1] += 0.5
    with pytest.raises(ValueError):
        EqLinear.from_unrolled(At, badb, 4)
    with pytest.raises(ValueError):
        EqLinear.from_unrolled(At, bt, 8)  # 12 x 8 is not a multiple of 8 x 8
    with pytest.raises(ValueError):
        EqLinear.from_unrolled(At[:, :6], None, 2)  # the 2-group reading is not circulant


def test_from_unrolled_p4m_recovers_the_weights_and_rejects_the_cyclic_reading():
    rng = np.random.default_rng(73)
    C, D = 3, 5
    W = rng.standard_normal((D, C, 8)).astype(np.float32)
    b = rng.standard_normal(D).astype(np.float32)
    A = torch.from_numpy(P4M.unrolled(W.astype(np.float64)).astype(np.float32))
    bd = torch.from_numpy(np.repeat(b, 8))
    m = EqLinear.from_unrolled(A, bd, 8, group="p4m")
    assert m.group == "p4m" and np.array_equal(m.weight.detach().numpy(), W)
    with pytest.raises(ValueError):
        EqLinear.from_unrolled(A, bd, 8)  # a p4m layer is not C_8-circulant
    with pytest.raises(ValueError):
        EqLinear(3, 5, 4, group="p4m")


def test_module_has_no_cpu_path():
    m = EqLinear(4, 6, 4, dtype=torch.float16)
    assert m.weight.shape == (6, 4, 4) and m.bias.shape == (6,)
    bound = 1.0 / np.sqrt(16)
    assert float(m.weight.detach().abs().max()) <= bound
    with pytest.raises(RuntimeError):
        m(torch.zeros((3, 16), dtype=torch.float16))
    with pytest.raises(TypeError):
        mode_for(torch.bfloat16)


# ------------------------------------------------------------------ GPU ---

def _cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from group_dft_structured_b200 import build
    build.build()
    F.load()


def _module(W, b):
    D, C, T = W.shape
    m = EqLinear(C, D, T, bias=b is not None, dtype=torch.from_numpy(W).dtype, device="cuda")
    with torch.no_grad():
        m.weight.copy_(torch.from_numpy(W))
        if b is not None:
            m.bias.copy_(torch.from_numpy(b))
    return m


def _host(t):
    return t.detach().cpu().numpy().astype(np.float64)


CASES = [(4, "fp16", 300, 24, 96, 5e-3), (8, "fp16", 300, 12, 48, 5e-3),
         (6, "fp16", 300, 16, 64, 5e-3), (4, "fp32", 130, 16, 24, 1e-5)]


@pytest.mark.gpu
@pytest.mark.parametrize("T,dtype,N,C,D,tol", CASES)
def test_module_forward_and_autograd_match_oracle(T, dtype, N, C, D, tol):
    _cuda_ready()
    inp = make_inputs(31, N, C, D, dtype, T=T)
    m = _module(inp["W"], inp["b"])
    x = torch.from_numpy(inp["x"].reshape(N, C * T)).cuda().requires_grad_(True)
    g = torch.from_numpy(inp["dy"].reshape(N, D * T)).cuda()
    y = m(x)
    (y * g).sum().backward()
    assert F.feql_device_status() == F.FEQL_OK
    x64, W64, b64, dy64 = (inp[k].astype(np.float64) for k in ("x", "W", "b", "dy"))
    dW, db = O.backward_dw(x64, dy64)
    assert O.rel_err(_host(y).reshape(N, D, T), O.forward(x64, W64, b64)) <= tol
    assert O.rel_err(_host(x.grad).reshape(N, C, T), O.backward_dx(dy64, W64)) <= tol
    assert O.rel_err(_host(m.weight.grad), dW) <= tol
    assert O.rel_err(_host(m.bias.grad), db) <= tol


@pytest.mark.gpu
@pytest.mark.parametrize("T", [4, 6, 8])
def test_module_gradient_subsets(T):
    _cuda_ready()
    N, C, D = 200, 8, 16
    inp = make_inputs(32, N, C, D, "fp16", T=T)
    x64, W64, dy64 = (inp[k].astype(np.float64) for k in ("x", "W", "dy"))
    dW_ref, db_ref = O.backward_dw(x64, dy64)
    g = torch.from_numpy(inp["dy"].reshape(N, D * T)).cuda()
    # no input gradient: weight and bias only
    m = _module(inp["W"], inp["b"])
    x = torch.from_numpy(inp["x"].reshape(N, C * T)).cuda()
    (m(x) * g).sum().backward()
    assert O.rel_err(_host(m.weight.grad), dW_ref) <= 5e-3
    assert O.rel_err(_host(m.bias.grad), db_ref) <= 5e-3
    # frozen weights, no bias: input gradient only
    m = _module(inp["W"], None)
    m.weight.requires_grad_(False)
    x = torch.from_numpy(inp["x"].reshape(N, C * T)).cuda().requires_grad_(True)
    (m(x) * g).sum().backward()
    assert m.weight.grad is None
    assert O.rel_err(_host(x.grad).reshape(N, C, T), O.backward_dx(dy64, W64)) <= 5e-3


@pytest.mark.gpu
def test_module_tracks_weight_updates_and_batch_shapes():
    _cuda_ready()
    B, L, C, D, T = 4, 50, 12, 20, 4
    inp = make_inputs(33, B * L, C, D, "fp16", T=T)
    m = _module(inp["W"], inp["b"])
    x = torch.from_numpy(inp["x"].reshape(B, L, C * T)).cuda()
    y1 = m(x)
    assert y1.shape == (B, L, D * T)
    with torch.no_grad():
        m.weight.mul_(2.0)  # in place: the Fourier buffer must be rebuilt
    y2 = m(x)
    x64, W64, b64 = (inp[k].astype(np.float64) for k in ("x", "W", "b"))
    ref2 = O.forward(x64, 2.0 * W64, b64).reshape(B, L, D * T)
    assert O.rel_err(_host(y2), ref2) <= 5e-3
    assert O.rel_err(_host(y1), O.forward(x64, W64, b64).reshape(B, L, D * T)) <= 5e-3


@pytest.mark.gpu
def test_module_p4m_forward_and_autograd_match_oracle():
    _cuda_ready()
    N, C, D = 300, 12, 48
    inp = make_inputs(35, N, C, D, "fp16", T=8)
    m = EqLinear(C, D, 8, dtype=torch.float16, device="cuda", group="p4m")
    with torch.no_grad():
        m.weight.copy_(torch.from_numpy(inp["W"]))
        m.bias.copy_(torch.from_numpy(inp["b"]))
    x = torch.from_numpy(inp["x"].reshape(N, C * 8)).cuda().requires_grad_(True)
    g = torch.from_numpy(inp["dy"].reshape(N, D * 8)).cuda()
    y = m(x)
    (y * g).sum().backward()
    x64, W64, b64, dy64 = (inp[k].astype(np.float64) for k in ("x", "W", "b", "dy"))
    dW, db = P4M.backward_dw(x64, dy64)
    assert P4M.rel_err(_host(y).reshape(N, D, 8), P4M.forward(x64, W64, b64)) <= 5e-3
    assert P4M.rel_err(_host(x.grad).reshape(N, C, 8), P4M.backward_dx(dy64, W64)) <= 5e-3
    assert P4M.rel_err(_host(m.weight.grad), dW) <= 5e-3
    assert P4M.rel_err(_host(m.bias.grad), db) <= 5e-3


@pytest.mark.gpu
def test_from_unrolled_replaces_a_naive_layer():
    _cuda_ready()
    N, C, D, T = 257, 16, 32, 8
    inp = make_inputs(34, N, C, D, "fp16", T=T)
    A, bd = dense_layer(inp["W"], inp["b"])
    lin = torch.nn.Linear(C * T, D * T, dtype=torch.float16, device="cuda")
    with torch.no_grad():
        lin.weight.copy_(torch.from_numpy(A))  # exact: the entries are fp16 values
        lin.bias.copy_(torch.from_numpy(bd))
    m = EqLinear.from_unrolled(lin.weight, lin.bias, T)
    x = torch.from_numpy(inp["x"].reshape(N, C * T)).cuda()
    ref = inp["x"].astype(np.float64).reshape(N, C * T) @ A.T + bd  # the naive layer, float64
    assert O.rel_err(_host(m(x)), ref) <= 5e-3
