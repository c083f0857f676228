"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, sizes its buffers, and rejects bad arguments on the host before any
launch (fake pointers are never dereferenced on these paths)."""
import ctypes
import os
import re

import pytest

import ternary_weight_bit_w2a8_b200 as bn
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bitnet_b200.h")


@pytest.fixture(scope="module")
def lib():
    from ternary_weight_bit_w2a8_b200 import build
    build.build()
    return bn.lib()


def header_symbols():
    text = open(HEADER, encoding="utf-8").read()
    return re.findall(r"BITNET_API\s+[\w\s\*]+?\**\s*(bitnet_\w+)\s*\(", text)


def test_exports_every_declared_symbol(lib):
    names = header_symbols()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
    # and the binding wraps each of them under the same name
    for name in names:
        assert name in bn._SIGNATURES, name


def test_status_strings(lib):
    for code in range(7):
        s = bn.status_string(code)
        assert s.startswith("BITNET_")
    assert "unknown" in bn.status_string(99)


def test_layout_version(lib):
    assert bn.layout_version() == 1


def test_packed_bytes_matches_layout_spec(lib, oracle_mod):
    for N, K in [(1, 1), (3, 17), (2560, 2560), (55296, 5120), (7, 129), (1, 0), (0, 5)]:
        assert bn.bitnet_packed_bytes(N, K) == oracle_mod.device_packed_bytes(N, K)
    assert lib.bitnet_packed_bytes(-1, 4) == -1
    assert lib.bitnet_packed_bytes(4, (1 << 21) + 1) == -1


def test_workspace_bytes(lib):
    assert lib.bitnet_workspace_bytes(-1, 2, 2) == -1
    assert lib.bitnet_workspace_bytes(1, 2560, 2560) >= 8 * 1024  # absmean partials
    # split-K problems need room for partials
    assert lib.bitnet_workspace_bytes(1, 64, 65536) >= 64 * 4 * 2
    # depends only on the shape
    assert lib.bitnet_workspace_bytes(3, 100, 1000) == lib.bitnet_workspace_bytes(3, 100, 1000)


def test_workspace_bytes_cover_the_bitlinear_quantisation(lib):
    # 5..16 tokens: BitLinear quantises them into the workspace (q, then the
    # scales) before the one-pass GEMV
    for M in (5, 8, 12, 16):
        assert lib.bitnet_workspace_bytes(M, 300, 2560) >= M * 2560 + M * 4
    # prefill: K_pad-strided q and the scales ahead of the tensor-core GEMM
    assert lib.bitnet_workspace_bytes(128, 13824, 2560) >= 128 * 2560 + 128 * 4
    assert lib.bitnet_workspace_bytes(2048, 2560, 6912) >= 2048 * 6912 + 2048 * 4


# The tests below pass fake pointers; each call is built to fail a host-side
# check before any device work.  They are skipped where a GPU is present, so
# that a wrong expectation can never turn into a launch on fake pointers.
def _no_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake-pointer host checks run only where no GPU is present")


A = ctypes.c_void_p(0x10000)       # aligned fake device pointer
A2 = ctypes.c_void_p(0x20000)
MIS = ctypes.c_void_p(0x10001)     # misaligned
NULL = None
S = None                           # default stream


def test_gemm_argument_errors(lib):
    _no_gpu()
    g = lib.bitnet_w2a8_gemm
    assert g(A, A, A, -1, 4, 4, NULL, 0, S) == bn.BITNET_ERR_INVALID_ARG
    assert g(A, A, A, 1, 4, (1 << 21) + 1, NULL, 0, S) == bn.BITNET_ERR_INVALID_ARG
    assert g(NULL, A, A, 1, 4, 4, NULL, 0, S) == bn.BITNET_ERR_INVALID_ARG
    assert g(A, NULL, A, 1, 4, 4, NULL, 0, S) == bn.BITNET_ERR_INVALID_ARG
    assert g(A, A, NULL, 1, 4, 4, NULL, 0, S) == bn.BITNET_ERR_INVALID_ARG
    assert g(A, MIS, A, 1, 4, 4, NULL, 0, S) == bn.BITNET_ERR_ALIGNMENT
    assert g(A, A, MIS, 1, 4, 4, NULL, 0, S) == bn.BITNET_ERR_ALIGNMENT
    # empty problems are no-ops that touch nothing
    assert g(NULL, NULL, NULL, 0, 4, 4, NULL, 0, S) == bn.BITNET_OK
    assert g(NULL, NULL, NULL, 3, 0, 4, NULL, 0, S) == bn.BITNET_OK
    # a prefill batch (tensor-core path) with K not a multiple of 16: the
    # activations are always repacked into the workspace, so one is required
    need = lib.bitnet_workspace_bytes(200, 64, 1000)
    assert need >= 200 * 1024
    assert g(A, A, A, 200, 64, 1000, NULL, 0, S) == bn.BITNET_ERR_WORKSPACE
    assert g(A, A, A, 200, 64, 1000, A2, 64, S) == bn.BITNET_ERR_WORKSPACE
    assert g(A, A, A, 200, 64, 1000, MIS, need, S) == bn.BITNET_ERR_ALIGNMENT


def test_bitlinear_argument_errors(lib):
    # every call here fails its host-side checks: none may reach a launch.
    # a prefill batch: the quantised activations always go to the workspace
    _no_gpu()
    f = lib.bitnet_bitlinear
    ws_need = lib.bitnet_workspace_bytes(200, 64, 1000)
    assert f(A, A, NULL, A, 200, 64, 1000, A2, ws_need, S) == bn.BITNET_ERR_INVALID_ARG  # gamma
    assert f(MIS, A, A, A, 200, 64, 1000, A2, ws_need, S) == bn.BITNET_ERR_ALIGNMENT
    assert f(A, A, A, A, 200, 64, 1000, NULL, 0, S) == bn.BITNET_ERR_WORKSPACE
    assert f(A, A, A, A, 200, 64, 1000, A2, 16, S) == bn.BITNET_ERR_WORKSPACE
    assert f(A, A, A, A, 200, 64, 1000, MIS, ws_need, S) == bn.BITNET_ERR_ALIGNMENT
    assert f(NULL, NULL, NULL, NULL, 0, 8, 64, NULL, 0, S) == bn.BITNET_OK


def test_prep_argument_errors(lib):
    _no_gpu()
    assert lib.bitnet_absmean(A, 4, 4, NULL, A2, 8192, S) == bn.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_absmean(A, 4, 4, A, NULL, 0, S) == bn.BITNET_ERR_WORKSPACE
    assert lib.bitnet_absmean(A, 4, 4, A, A2, 4, S) == bn.BITNET_ERR_WORKSPACE
    assert lib.bitnet_absmean(MIS, 4, 4, A, A2, 8192, S) == bn.BITNET_ERR_ALIGNMENT
    assert lib.bitnet_ternarize(A, 4, 4, NULL, A, S) == bn.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_ternarize(A, -4, 4, A, A, S) == bn.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_pack_weights(NULL, 4, 4, A, NULL, S) == bn.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_pack_weights(A, 4, 4, MIS, NULL, S) == bn.BITNET_ERR_ALIGNMENT
    assert lib.bitnet_quant_act(A, 2, 4, A, NULL, NULL, S) == bn.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_quant_act(A, 2, 4, A, MIS, NULL, S) == bn.BITNET_ERR_ALIGNMENT
    assert lib.bitnet_quant_act(NULL, 0, 4, NULL, NULL, NULL, S) == bn.BITNET_OK


def test_valid_call_without_gpu_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; fake pointers must not reach a launch")
    assert lib.bitnet_w2a8_gemm(A, A, A, 1, 4, 4, NULL, 0, S) == bn.BITNET_ERR_CUDA
    assert lib.bitnet_launch_count() == 0
