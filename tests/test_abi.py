"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/feql.h declares, validates its arguments before any
CUDA call, and sizes the Fourier-weight buffer as documented."""

import ctypes
import os
import re

import pytest

import group_dft_structured_b200 as F
from group_dft_structured_b200 import build as B


@pytest.fixture(scope="module")
def lib():
    B.build()
    return F.load()


def header_functions():
    src = open(F.HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(feql_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = header_functions()
    for n in ["feql_weight_fft", "feql_forward", "feql_backward_dx", "feql_backward_dw",
              "feql_weight_fft_bytes", "feql_backward_dw_workspace_bytes",
              "feql_device_status", "feql_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_status_strings(lib):
    assert F.feql_status_string(F.FEQL_OK) == "ok"
    assert "invalid" in F.feql_status_string(F.FEQL_ERR_INVALID_ARG)
    assert "timed out" in F.feql_status_string(F.FEQL_ERR_TIMEOUT)
    assert F.feql_status_string(99) == "unknown status"


def test_invalid_arguments_rejected_before_cuda(lib):
    st = lib.feql_forward(None, None, None, None, 10, 4, 4, F.FEQL_FP16, None)
    assert st == F.FEQL_ERR_INVALID_ARG
    p = 1 << 20  # aligned fake address; never dereferenced because N < 0
    assert lib.feql_forward(p, p, None, p, -1, 4, 4, F.FEQL_FP16, None) == F.FEQL_ERR_INVALID_ARG
    assert lib.feql_forward(p, p, None, p, 8, 0, 4, F.FEQL_FP16, None) == F.FEQL_ERR_INVALID_ARG
    assert lib.feql_forward(p, p, None, p, 8, 4, 4, 17, None) == F.FEQL_ERR_INVALID_ARG
    assert lib.feql_forward(p + 4, p, None, p, 8, 4, 4, F.FEQL_FP16, None) == F.FEQL_ERR_INVALID_ARG
    assert lib.feql_backward_dx(p, None, p, 8, 4, 4, F.FEQL_FP16, None) == F.FEQL_ERR_INVALID_ARG
    assert lib.feql_backward_dw(p, p, p, None, None, 0, 8, 4, 4, F.FEQL_FP16, None) == \
        F.FEQL_ERR_INVALID_ARG
    assert lib.feql_weight_fft(None, p, 4, 4, F.FEQL_FP16, None) == F.FEQL_ERR_INVALID_ARG
    # odd channel counts cannot be tiled by TMA in fp16 (row stride not a multiple of 16 B)
    assert lib.feql_forward(p, p, None, p, 8, 3, 4, F.FEQL_FP16, None) == F.FEQL_ERR_UNSUPPORTED
    assert lib.feql_weight_fft(p, p, 4, 5, F.FEQL_FP16, None) == F.FEQL_ERR_UNSUPPORTED


def _tc_plan(Ci, Do):
    nK = -(-Ci // 16)
    nD = -(-Do // (64 if nK <= 4 else 128))
    BD = -(-(-(-Do // nD)) // 16) * 16
    return nD, BD, nK, nD * nK * 5 * BD * 16 * 2


def _tf32_plan(Ci, Do):
    """Split-TF32 direction: chunks of 8 channels, the fp16 tiling of outputs
    (BD <= 64 when the contraction is at most 64 channels), hi and lo tiles."""
    nK = -(-Ci // 8)
    nD = -(-Do // (64 if Ci <= 64 else 128))
    BD = -(-(-(-Do // nD)) // 16) * 16
    return nD, BD, nK, nD * nK * 2 * 5 * BD * 32


@pytest.mark.parametrize("C,D", [(16, 16), (48, 192), (192, 192), (256, 256), (24, 96), (6, 40),
                                 (3, 5), (600, 16)])
def test_weight_buffer_sizes(lib, C, D):
    def al(v):
        return -(-v // 1024) * 1024
    tc = al(_tc_plan(C, D)[3]) + al(_tc_plan(D, C)[3])
    tf32 = al(_tf32_plan(C, D)[3]) + al(_tf32_plan(D, C)[3])
    simt = 2 * 4 * C * D * 4
    if ((C | D) & 1) == 0:
        assert F.feql_weight_fft_bytes(C, D, F.FEQL_FP16) == tc
    assert F.feql_weight_fft_bytes(C, D, F.FEQL_FP32_SIMT) == simt
    assert F.feql_weight_fft_bytes(C, D, F.FEQL_FP32_3XTF32) == tf32
    # FEQL_FP32 is split TF32 up to 512 channels on either side, CUDA cores beyond
    assert F.feql_weight_fft_bytes(C, D, F.FEQL_FP32) == (tf32 if max(C, D) <= 512 else simt)
    assert F.feql_weight_fft_bytes(C, D, F.FEQL_FP16_SIMT) == simt
    assert F.feql_weight_fft_bytes(0, D, F.FEQL_FP16) == 0


def test_tile_plans_cover_the_workloads():
    # output-channel tiles of at most 128 (complex-bin MMA N = 2*BD <= 256);
    # at most 64 (double-buffered TMEM) when the contraction is <= 64 channels
    assert _tc_plan(48, 192)[:2] == (3, 64)
    assert _tc_plan(192, 192)[:2] == (2, 96)
    assert _tc_plan(256, 256)[:2] == (2, 128)
    assert _tc_plan(24, 96)[:2] == (2, 48)
    assert _tc_plan(96, 24)[:2] == (1, 32)
    assert _tc_plan(16, 16)[:2] == (1, 16)


def test_product_path_has_no_oracle_dependency():
    pkg = os.path.dirname(F.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(root, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", src, flags=re.M), f
                assert "feql_oracle" not in src, f


def test_group_and_block_entry_points_reject_bad_arguments_before_cuda(lib):
    p = 1 << 20  # aligned fake address; never dereferenced
    FP16, FP32 = F.FEQL_FP16, F.FEQL_FP32
    INV, UNS = F.FEQL_ERR_INVALID_ARG, F.FEQL_ERR_UNSUPPORTED
    # cyclic C_T: orders outside 2..16, split-TF32 for T != 4, bad sizes and pointers
    assert lib.feql_ct_forward(17, p, p, None, p, 8, 4, 4, FP16, None) == UNS
    assert lib.feql_ct_forward(1, p, p, None, p, 8, 4, 4, FP32, None) == UNS
    assert lib.feql_ct_forward(8, p, p, None, p, 8, 4, 4, F.FEQL_FP32_3XTF32, None) == UNS
    assert lib.feql_ct_forward(6, p, p, None, p, -1, 4, 4, FP16, None) == INV
    assert lib.feql_ct_forward(6, p + 4, p, None, p, 8, 4, 4, FP32, None) == INV
    assert lib.feql_ct_backward_dw(12, p, p, None, None, p, 0, 8, 4, 4, FP32, None) == INV
    assert lib.feql_ct_weight_fft(5, None, p, 4, 4, FP32, None) == INV
    assert lib.feql_ct_forward(8, p, p, None, p, -1, 4, 4, FP16, None) == INV
    assert lib.feql_ct_forward(8, p + 4, p, None, p, 8, 4, 4, FP16, None) == INV
    assert lib.feql_ct_backward_dx(8, p, None, p, 8, 4, 4, FP16, None) == INV
    assert lib.feql_ct_backward_dw(8, p, p, None, None, p, 0, 8, 4, 4, FP16, None) == INV
    assert lib.feql_ct_weight_fft(8, None, p, 4, 4, FP16, None) == INV
    # p4m
    assert lib.feql_p4m_forward(p, p, None, p, 8, 4, 4, FP32, None) == UNS
    assert lib.feql_p4m_forward(p, p, None, p, 8, 0, 4, FP16, None) == INV
    assert lib.feql_p4m_backward_dx(p, None, p, 8, 4, 4, FP16, None) == INV
    assert lib.feql_p4m_backward_dw(p, p, None, None, p, 0, 8, 4, 4, FP16, None) == INV
    assert lib.feql_p4m_weight_fft(None, p, 4, 4, FP16, None) == INV
    assert lib.feql_p4m_weight_fft(p, p, 4, 4, 17, None) == INV
    # MLP block: odd C or Co (TMA rows), bad sizes and pointers
    assert lib.feql_mlp_forward(p, p, None, None, p, 8, 5, 16, 8, FP16, None) == UNS
    assert lib.feql_mlp_forward(p, p, None, None, p, 8, 4, 16, 7, FP16, None) == UNS
    assert lib.feql_mlp_forward(p, p, None, None, p, -1, 4, 16, 8, FP16, None) == INV
    assert lib.feql_mlp_forward(p, p, p + 2, None, p, 8, 4, 16, 8, FP16, None) == INV
    assert lib.feql_mlp_weight_fft(None, p, p, 4, 16, 8, FP16, None) == INV


def _g8_bytes(C, D, rows):
    def plan(Ci, Do):
        nK, nD = -(-Ci // 16), -(-Do // 64)
        BD = -(-(-(-Do // nD)) // 16) * 16
        return nD * nK * rows * BD * 16 * 2
    al = lambda v: -(-v // 1024) * 1024
    return al(plan(C, D)) + al(plan(D, C))


@pytest.mark.parametrize("C,D", [(12, 48), (8, 8), (40, 130), (64, 16), (6, 40)])
def test_order8_weight_buffer_sizes(lib, C, D):
    # C_8: 11 weight rows per output channel (W0, W4, (Re, Im, -Re) of bins 1..3); p4m: 8
    assert F.feql_ct_weight_fft_bytes(8, C, D, F.FEQL_FP16) == _g8_bytes(C, D, 11)
    assert F.feql_p4m_weight_fft_bytes(C, D, F.FEQL_FP16) == _g8_bytes(C, D, 8)
    assert F.feql_ct_weight_fft_bytes(4, C, D, F.FEQL_FP16) == F.feql_weight_fft_bytes(C, D, F.FEQL_FP16)
    for T in (2, 3, 6, 8, 12, 16):  # CUDA-core orders: fp32 planes of both directions
        assert F.feql_ct_weight_fft_bytes(T, C, D, F.FEQL_FP32) == 2 * T * C * D * 4
    assert F.feql_p4m_weight_fft_bytes(C, D, F.FEQL_FP32) == 0
    # C_6 in fp16: tensor cores (8 weight rows: W0, W3, (Re, Im, -Re) of bins 1, 2) when C
    # and D are multiples of 4, else the CUDA-core planes
    if C % 4 == 0 and D % 4 == 0:
        assert F.feql_ct_weight_fft_bytes(6, C, D, F.FEQL_FP16) == _g8_bytes(C, D, 8)
    else:
        assert F.feql_ct_weight_fft_bytes(6, C, D, F.FEQL_FP16) == 2 * 6 * C * D * 4


def test_mlp_weight_buffer_covers_both_layers(lib):
    # at least the tiled Fourier weights of fc1 and fc2 (5 planes per 16 channels of each)
    for C, H, Co in [(24, 96, 24), (48, 192, 48), (96, 384, 96), (6, 40, 10)]:
        n = F.feql_mlp_weight_fft_bytes(C, H, Co, F.FEQL_FP16)
        a16 = lambda v: -(-v // 16) * 16
        assert n >= 5 * 2 * (a16(C) * a16(H) + a16(H) * a16(Co)), (C, H, Co)
    assert F.feql_mlp_weight_fft_bytes(192, 768, 192, F.FEQL_FP16) == 0
