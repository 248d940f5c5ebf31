"""CPU oracle for the block-FP8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product (the CUDA library and its
binding) never does, and the two share no code. The arithmetic lives in
``fp8blk_oracle.cpp`` (plain C++, double-precision sums); this module only
marshals numpy arrays into it.

Layouts: BF16 tensors are passed as their uint16 bit patterns. A matrix is a
C-contiguous 2-D array ``[rows, ld]`` whose first ``K`` columns are the data
(``ld >= K``); scales are dense ``[ceil(rows/128), ceil(K/128)]`` for weights
and ``[M, ceil(K/128)]`` for activations.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_i64, _u64, _int, _p = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            from .build import build
            build()
        lib = ctypes.CDLL(_LIB_PATH)
        sig = {
            "orc_e4m3_table": (None, [_p]),
            "orc_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_e4m3_encode_fields": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_bf16_rne": (ctypes.c_uint16, [ctypes.c_float]),
            "orc_e4m3_encode_array": (None, [_p, _i64, _p]),
            "orc_bf16_rne_array": (None, [_p, _i64, _p]),
            "orc_crosscheck_encoders": (_i64, [_u64, _u64, _int]),
            "orc_crosscheck_encoders_planted": (_i64, [_u64, _u64, _u64, _int]),
            "orc_count_code_mismatches": (_i64, [_u64, _i64, _p, _int]),
            "orc_quantize_weight": (None, [_p, _i64, _i64, _i64, _p, _i64, _p, _int]),
            "orc_dequantize": (None, [_p, _i64, _p, _i64, _i64, _p, _i64, _int]),
            "orc_act_quant": (None, [_p, _i64, _i64, _i64, _p, _i64, _p, _int]),
            "orc_linear_w8a16": (None, [_p, _i64, _p, _i64, _p, _i64, _i64, _i64, _p, _i64, _p, _int]),
            "orc_linear_w8a8": (None, [_p, _i64, _p, _p, _i64, _p, _i64, _i64, _i64, _p, _i64, _p, _int]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype, f.argtypes = res, args
        _lib = lib
    return _lib


def threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


# ------------------------------------------------------------------ codecs
def e4m3_table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    _load().orc_e4m3_table(out.ctypes.data)
    return out


def e4m3_encode(v) -> np.ndarray:
    v, pv = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(pv, v.size, out.ctypes.data)
    return out


def e4m3_encode_fields(f: float) -> int:
    return int(_load().orc_e4m3_encode_fields(ctypes.c_float(f)))


def bf16_rne(v) -> np.ndarray:
    v, pv = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().orc_bf16_rne_array(pv, v.size, out.ctypes.data)
    return out


def crosscheck_encoders(lo: int, hi: int, nthreads: int | None = None) -> int:
    return int(_load().orc_crosscheck_encoders(lo, hi, nthreads or threads()))


def crosscheck_encoders_planted(lo: int, hi: int, planted: int, nthreads: int | None = None) -> int:
    """Test hook: the cross-check with the bit-field encoder's code at bit
    pattern `planted` deliberately wrong (lowest bit flipped)."""
    return int(_load().orc_crosscheck_encoders_planted(lo, hi, planted, nthreads or threads()))


def count_code_mismatches(lo: int, codes: np.ndarray, nthreads: int | None = None) -> int:
    codes, pc = _c(codes, np.uint8)
    return int(_load().orc_count_code_mismatches(lo, codes.size, pc, nthreads or threads()))


# ------------------------------------------------------------------ method
def quantize_weight(w_bits: np.ndarray, K: int | None = None, ldq: int | None = None):
    """BF16 weight bits [N, ldw] -> (q uint8 [N, ldq], scale_inv float32 [NB, KB])."""
    w, pw = _c(w_bits, np.uint16)
    N, ldw = w.shape
    K = ldw if K is None else K
    ldq = K if ldq is None else ldq
    q = np.zeros((N, ldq), dtype=np.uint8)
    s = np.empty((cdiv(N, 128), cdiv(K, 128)), dtype=np.float32)
    _load().orc_quantize_weight(pw, N, K, ldw, q.ctypes.data, ldq, s.ctypes.data, threads())
    return q, s


def dequantize(q: np.ndarray, scale_inv: np.ndarray, K: int | None = None) -> np.ndarray:
    """(q [N, ldq], scale_inv [NB, KB]) -> BF16 bits [N, K]."""
    q, pq = _c(q, np.uint8)
    s, ps = _c(scale_inv, np.float32)
    N, ldq = q.shape
    K = ldq if K is None else K
    assert s.shape == (cdiv(N, 128), cdiv(K, 128))
    w = np.empty((N, K), dtype=np.uint16)
    _load().orc_dequantize(pq, ldq, ps, N, K, w.ctypes.data, K, threads())
    return w


def act_quant(x_bits: np.ndarray, K: int | None = None):
    """BF16 activation bits [M, ldx] -> (qx uint8 [M, K], sx float32 [M, KB])."""
    x, px = _c(x_bits, np.uint16)
    M, ldx = x.shape
    K = ldx if K is None else K
    qx = np.zeros((M, K), dtype=np.uint8)
    sx = np.empty((M, cdiv(K, 128)), dtype=np.float32)
    _load().orc_act_quant(px, M, K, ldx, qx.ctypes.data, K, sx.ctypes.data, threads())
    return qx, sx


def _rows(rows, M):
    if rows is None:
        return None, 0, M
    r = np.ascontiguousarray(rows, dtype=np.int64)
    assert r.ndim == 1 and (r.size == 0 or (r.min() >= 0 and r.max() < M))
    return r, r.ctypes.data, r.size


def linear_w8a16(x_bits, q, scale_inv, N: int, K: int, rows=None) -> np.ndarray:
    """FP64 y[rows, N] for BF16 x [M, ldx] and block-FP8 (q, scale_inv)."""
    x, px = _c(x_bits, np.uint16)
    q, pq = _c(q, np.uint8)
    s, ps = _c(scale_inv, np.float32)
    M = x.shape[0]
    r, pr, nr = _rows(rows, M)
    ref = np.empty((nr, N), dtype=np.float64)
    _load().orc_linear_w8a16(px, x.shape[1], pq, q.shape[1], ps, M, N, K, pr, nr,
                             ref.ctypes.data, threads())
    return ref


def linear_w8a8(qx, sx, q, scale_inv, N: int, K: int, rows=None) -> np.ndarray:
    """FP64 y[rows, N] from quantized activations (qx, sx) and weights (q, scale_inv)."""
    qx, pqx = _c(qx, np.uint8)
    sx, psx = _c(sx, np.float32)
    q, pq = _c(q, np.uint8)
    s, ps = _c(scale_inv, np.float32)
    M = qx.shape[0]
    r, pr, nr = _rows(rows, M)
    ref = np.empty((nr, N), dtype=np.float64)
    _load().orc_linear_w8a8(pqx, qx.shape[1], psx, pq, q.shape[1], ps, M, N, K, pr, nr,
                            ref.ctypes.data, threads())
    return ref
