"""CPU oracle for the BitNet b1.58 W2A8 BitLinear path.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library
never links, imports or calls it, and it never calls the CUDA library.

The arithmetic lives in ``oracle.c`` (plain loops, compiled with gcc into
``liboracle.so`` beside it); this module only marshals numpy arrays through
ctypes. Each wrapped function cites the passage it follows in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build_oracle import build as _build, library_path

_LIB = None

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def _lib():
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            _build()
        lib = ctypes.CDLL(path)
        sig = {
            "oracle_abi_version": (ctypes.c_int, []),
            "oracle_absmean": (ctypes.c_float, [_ptr, _i64, _i64]),
            "oracle_ternarize": (None, [_ptr, _i64, _i64, ctypes.c_float, _ptr]),
            "oracle_quant_act": (None, [_ptr, _i64, _i64, _ptr, _ptr, _ptr]),
            "oracle_gemm_i32": (ctypes.c_int, [_ptr, _ptr, _i64, _i64, _i64, _ptr]),
            "oracle_gemm_i32_sampled": (None, [_ptr, _ptr, _i64, _ptr, _ptr, _i64, _ptr]),
            "oracle_rescale": (None, [_ptr, _i64, _i64, ctypes.c_float, _ptr, _ptr]),
            "oracle_bitlinear": (ctypes.c_int, [_ptr, _ptr, ctypes.c_float, _i64, _i64, _i64,
                                                _ptr, _ptr, _ptr, _ptr]),
            "oracle_canonical_packed_bytes": (_i64, [_i64, _i64]),
            "oracle_pack_canonical": (None, [_ptr, _i64, _i64, _ptr]),
            "oracle_unpack_canonical": (None, [_ptr, _i64, _i64, _ptr]),
            "oracle_device_packed_bytes": (_i64, [_i64, _i64]),
            "oracle_pack_device": (_i64, [_ptr, _i64, _i64, _ptr]),
            "oracle_unpack_device": (_i64, [_ptr, _i64, _i64, _ptr]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def absmean(W_bf16: np.ndarray) -> np.float32:
    """Per-tensor absmean scale of bf16 weights [N, K] (bit patterns, uint16)."""
    W = _c(W_bf16, np.uint16)
    N, K = W.shape
    return np.float32(_lib().oracle_absmean(_p(W), N, K))


def ternarize(W_bf16: np.ndarray, gamma) -> np.ndarray:
    """W_t = clamp(rne(W / gamma), -1, 1) in fp32 -> int8 [N, K]."""
    W = _c(W_bf16, np.uint16)
    N, K = W.shape
    out = np.empty((N, K), dtype=np.int8)
    _lib().oracle_ternarize(_p(W), N, K, float(np.float32(gamma)), _p(out))
    return out


def quant_act(x_bf16: np.ndarray):
    """Per-token absmax int8 quantisation -> (q int8 [M, K], s fp32 [M], rowsum int32 [M])."""
    x = _c(x_bf16, np.uint16)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    rs = np.empty(M, dtype=np.int32)
    _lib().oracle_quant_act(_p(x), M, K, _p(q), _p(s), _p(rs))
    return q, s, rs


def gemm_i32(q: np.ndarray, Wt: np.ndarray) -> np.ndarray:
    """y[m, n] = sum_k q[m, k] * W_t[n, k] (exact) -> int32 [M, N]."""
    q = _c(q, np.int8)
    if q.ndim == 1:
        q = q.reshape(1, -1)
    Wt = _c(Wt, np.int8)
    M, K = q.shape
    N, K2 = Wt.shape
    assert K == K2
    y = np.empty((M, N), dtype=np.int32)
    of = _lib().oracle_gemm_i32(_p(q), _p(Wt), M, N, K, _p(y))
    if of:
        raise OverflowError("W2A8 accumulation left the int32 range")
    return y


def gemm_i32_sampled(q: np.ndarray, Wt: np.ndarray, ms, ns) -> np.ndarray:
    """The contraction at the listed output positions (m_i, n_i) only."""
    q = _c(q, np.int8)
    if q.ndim == 1:
        q = q.reshape(1, -1)
    Wt = _c(Wt, np.int8)
    K = q.shape[1]
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    out = np.empty(len(ms), dtype=np.int32)
    _lib().oracle_gemm_i32_sampled(_p(q), _p(Wt), K, _p(ms), _p(ns), len(ms), _p(out))
    return out


def rescale(acc: np.ndarray, gamma, s: np.ndarray) -> np.ndarray:
    """y = acc * gamma / s_m in fp64 -> float64 [M, N]."""
    acc = _c(acc, np.int32)
    M, N = acc.shape
    s = _c(s, np.float32)
    y = np.empty((M, N), dtype=np.float64)
    _lib().oracle_rescale(_p(acc), M, N, float(np.float32(gamma)), _p(s), _p(y))
    return y


def bitlinear(x_bf16: np.ndarray, Wt: np.ndarray, gamma):
    """Full BitLinear -> (y fp64 [M, N], acc int32 [M, N], q int8 [M, K], s fp32 [M])."""
    x = _c(x_bf16, np.uint16)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    Wt = _c(Wt, np.int8)
    M, K = x.shape
    N = Wt.shape[0]
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    acc = np.empty((M, N), dtype=np.int32)
    y = np.empty((M, N), dtype=np.float64)
    of = _lib().oracle_bitlinear(_p(x), _p(Wt), float(np.float32(gamma)), M, N, K,
                                 _p(q), _p(s), _p(acc), _p(y))
    if of:
        raise OverflowError("W2A8 accumulation left the int32 range")
    return y, acc, q, s


def pack_canonical(Wt: np.ndarray) -> np.ndarray:
    """Canonical 2-bit packing (code = w + 1, 4 per byte, low bits first)."""
    Wt = _c(Wt, np.int8)
    N, K = Wt.shape
    out = np.empty((N, (K + 3) // 4), dtype=np.uint8)
    _lib().oracle_pack_canonical(_p(Wt), N, K, _p(out))
    return out


def unpack_canonical(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    out = np.empty((N, K), dtype=np.int8)
    _lib().oracle_unpack_canonical(_p(packed), N, K, _p(out))
    return out


def device_packed_bytes(N: int, K: int) -> int:
    return int(_lib().oracle_device_packed_bytes(N, K))


def pack_device(Wt: np.ndarray):
    """Device layout v1 -> (packed uint8 [N, K_pad/4], invalid count)."""
    Wt = _c(Wt, np.int8)
    N, K = Wt.shape
    kpad = ((K + 127) // 128) * 128
    out = np.empty((N, kpad // 4), dtype=np.uint8)
    bad = _lib().oracle_pack_device(_p(Wt), N, K, _p(out))
    return out, int(bad)


def unpack_device(packed: np.ndarray, N: int, K: int):
    """Decode device layout v1 -> (W_t int8 [N, K], count of unused-code fields)."""
    packed = _c(packed, np.uint8)
    out = np.empty((N, K), dtype=np.int8)
    bad = _lib().oracle_unpack_device(_p(packed), N, K, _p(out))
    return out, int(bad)
