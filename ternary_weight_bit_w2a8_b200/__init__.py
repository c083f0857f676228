"""Python binding of libbitnet_b200.so (BitNet b1.58 W2A8 BitLinear on B200).

Argument marshalling only: every function takes torch CUDA tensors, passes
their device pointers and the current CUDA stream to the C entry point of the
same name (declared in include/bitnet_b200.h) and raises BitnetError on a
non-zero status. All arithmetic runs in the library's CUDA kernels; there is
no CPU fallback. Importing the package does not load the library: the first
call does, and raises if it has not been built.
"""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libbitnet_b200.so")

BITNET_OK = 0
BITNET_ERR_INVALID_ARG = 1
BITNET_ERR_ALIGNMENT = 2
BITNET_ERR_WORKSPACE = 3
BITNET_ERR_CUDA = 4
BITNET_ERR_DEVICE_TIMEOUT = 5
BITNET_ERR_UNSUPPORTED = 6

_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p
_SIGNATURES = {
    "bitnet_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bitnet_layout_version": (ctypes.c_int, []),
    "bitnet_packed_bytes": (_i64, [_i64, _i64]),
    "bitnet_workspace_bytes": (_i64, [_i64, _i64, _i64]),
    "bitnet_absmean": (ctypes.c_int, [_p, _i64, _i64, _p, _p, _i64, _p]),
    "bitnet_ternarize": (ctypes.c_int, [_p, _i64, _i64, _p, _p, _p]),
    "bitnet_pack_weights": (ctypes.c_int, [_p, _i64, _i64, _p, _p, _p]),
    "bitnet_quant_act": (ctypes.c_int, [_p, _i64, _i64, _p, _p, _p, _p]),
    "bitnet_w2a8_gemm": (ctypes.c_int, [_p, _p, _p, _i64, _i64, _i64, _p, _i64, _p]),
    "bitnet_bitlinear": (ctypes.c_int, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _i64, _p]),
    "bitnet_w2a8_gemm_noalloc": (ctypes.c_int, [_p, _p, _p, _i64, _i64, _i64, _p]),
    "bitnet_get_device_error": (ctypes.c_int, [_p]),
    "bitnet_launch_count": (_i64, []),
}


class BitnetError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m ternary_weight_bit_w2a8_b200.build` "
                "(there is no fallback implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().bitnet_status_string(int(status)).decode()


def _check(rc: int, where: str):
    if rc != BITNET_OK:
        raise BitnetError(rc, where)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    import torch
    if stream is not None:
        return stream.cuda_stream
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)  # no Stream object per call
    if raw is not None:
        return raw(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _dev(t, name):
    if t is not None and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ------------------------------------------------------------------ sizes

def layout_version() -> int:
    return lib().bitnet_layout_version()


def bitnet_packed_bytes(N: int, K: int) -> int:
    n = lib().bitnet_packed_bytes(N, K)
    if n < 0:
        raise BitnetError(BITNET_ERR_INVALID_ARG, "bitnet_packed_bytes")
    return n


def bitnet_workspace_bytes(M: int, N: int, K: int) -> int:
    n = lib().bitnet_workspace_bytes(M, N, K)
    if n < 0:
        raise BitnetError(BITNET_ERR_INVALID_ARG, "bitnet_workspace_bytes")
    return n


def workspace(M: int, N: int, K: int, device="cuda"):
    """A workspace tensor of bitnet_workspace_bytes(M, N, K) bytes (at least 256)."""
    import torch
    return torch.empty(max(256, bitnet_workspace_bytes(M, N, K)), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ entry points

def bitnet_absmean(W, gamma=None, ws=None, stream=None):
    """gamma = mean |W| over the whole bf16 matrix W [N, K] -> float32 tensor [1]."""
    import torch
    _dev(W, "W")
    N, K = W.shape
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = workspace(0, N, K, W.device)
    _check(lib().bitnet_absmean(_ptr(W), N, K, _ptr(gamma), _ptr(ws), ws.numel(), _stream(stream)),
           "bitnet_absmean")
    return gamma


def bitnet_ternarize(W, gamma, W_t=None, stream=None):
    """W_t = clamp(rne(W / gamma), -1, 1) -> int8 [N, K]."""
    import torch
    _dev(W, "W")
    N, K = W.shape
    if W_t is None:
        W_t = torch.empty((N, K), dtype=torch.int8, device=W.device)
    _check(lib().bitnet_ternarize(_ptr(W), N, K, _ptr(gamma), _ptr(W_t), _stream(stream)), "bitnet_ternarize")
    return W_t


def bitnet_pack_weights(W_t, packed=None, invalid_count=None, stream=None):
    """Packs int8 ternary W_t [N, K] into layout v1 -> uint8 [bitnet_packed_bytes(N, K)]."""
    import torch
    _dev(W_t, "W_t")
    N, K = W_t.shape
    if packed is None:
        packed = torch.empty(bitnet_packed_bytes(N, K), dtype=torch.uint8, device=W_t.device)
    _check(lib().bitnet_pack_weights(_ptr(W_t), N, K, _ptr(packed), _ptr(invalid_count), _stream(stream)),
           "bitnet_pack_weights")
    return packed


def bitnet_quant_act(x, q=None, s=None, rowsum=None, stream=None):
    """Per-token absmax int8 quantisation of bf16 x [M, K] -> (q int8, s float32, rowsum int32)."""
    import torch
    _dev(x, "x")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if s is None:
        s = torch.empty(M, dtype=torch.float32, device=x.device)
    if rowsum is None:
        rowsum = torch.empty(M, dtype=torch.int32, device=x.device)
    _check(lib().bitnet_quant_act(_ptr(x), M, K, _ptr(q), _ptr(s), _ptr(rowsum), _stream(stream)),
           "bitnet_quant_act")
    return q, s, rowsum


def bitnet_w2a8_gemm(q, packed, N: int, y=None, ws=None, stream=None):
    """y = q @ W_t^T exactly in int32: q int8 [M, K], packed layout v1 of W_t [N, K] -> int32 [M, N]."""
    import torch
    _dev(q, "q")
    M, K = q.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(M, N, K, q.device)
    _check(lib().bitnet_w2a8_gemm(_ptr(q), _ptr(packed), _ptr(y), M, N, K, _ptr(ws), ws.numel(),
                                  _stream(stream)), "bitnet_w2a8_gemm")
    return y


def bitnet_bitlinear(x, packed, gamma, N: int, y=None, ws=None, stream=None):
    """BitLinear forward: bf16 x [M, K], packed W_t [N, K], gamma [1] -> bf16 y [M, N]."""
    import torch
    _dev(x, "x")
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = workspace(M, N, K, x.device)
    _check(lib().bitnet_bitlinear(_ptr(x), _ptr(packed), _ptr(gamma), _ptr(y), M, N, K, _ptr(ws), ws.numel(),
                                  _stream(stream)), "bitnet_bitlinear")
    return y


def bitnet_w2a8_gemm_noalloc(q, packed, N: int, y=None, stream=None):
    """bitnet_w2a8_gemm without a workspace: for callers that cannot allocate
    device memory.  Uses the library's one built-in scratch array (see the C
    header): calls that overlap on the GPU race on it."""
    import torch
    _dev(q, "q")
    M, K = q.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.int32, device=q.device)
    _check(lib().bitnet_w2a8_gemm_noalloc(_ptr(q), _ptr(packed), _ptr(y), M, N, K, _stream(stream)),
           "bitnet_w2a8_gemm_noalloc")
    return y


def bitnet_get_device_error(stream=None) -> int:
    return lib().bitnet_get_device_error(_stream(stream))


def bitnet_launch_count() -> int:
    return lib().bitnet_launch_count()
