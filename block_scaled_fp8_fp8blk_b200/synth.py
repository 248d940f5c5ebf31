"""Seeded synthetic inputs for the block-FP8 linear layer.

Draws only random numbers: the values come from ``synth.c`` (counter-based
splitmix64 + Box-Muller) as float32 and are rounded to BF16 by torch's own
conversion. Nothing here performs any step of the layer (no FP8 coding, no
scales, no products), so the CUDA path and the CPU oracle can both consume
these tensors without sharing any of the method's arithmetic.

Recipe (the pages' workload is a 32B-class Qwen3-VL text encoder whose
checkpoint is not available, so these tensors stand in for its linears):

* weights ``W[N, K] ~ N(0, 0.02^2)``, optionally times a per-output-row gain
  ``g_n = exp(sigma * z_n)`` with ``z_n ~ N(0, 1)`` (LogNormal(0, sigma));
* activations ``x[M, K] ~ N(0, 1)``, with ``floor(frac * K)`` channels drawn
  without replacement and multiplied by 20 before rounding (outliers);
* streams per seed: x = 1, W = 2, row gains = 3, outlier channels = 4,
  checked-row subset = 5.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfp8blk_synth.so")

STREAM_X, STREAM_W, STREAM_GAIN, STREAM_OUTLIER, STREAM_ROWS = 1, 2, 3, 4, 5

_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: run __graft_entry__.build() or "
                "python -m block_scaled_fp8_fp8blk_b200.build")
        lib = ctypes.CDLL(_LIB_PATH)
        lib.synth_key.restype = ctypes.c_uint64
        lib.synth_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_uniform.restype = None
        lib.synth_uniform.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_normal_vec.restype = None
        lib.synth_normal_vec.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_matrix.restype = None
        lib.synth_matrix.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_int]
        _lib = lib
    return _lib


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def key(seed: int, stream: int) -> int:
    return int(_load().synth_key(seed, stream))


def uniform(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_uniform(key(seed, stream), n, out.ctypes.data)
    return out


def normal(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_normal_vec(key(seed, stream), n, out.ctypes.data)
    return out


def draw_without_replacement(seed: int, stream: int, population: int, count: int) -> np.ndarray:
    """``count`` distinct indices of ``range(population)``: the ones with the
    smallest uniform keys (a random permutation's prefix), returned sorted."""
    count = max(0, min(count, population))
    u = uniform(seed, stream, population)
    return np.sort(np.argsort(u, kind="stable")[:count]).astype(np.int64)


def outlier_channels(seed: int, K: int, frac: float) -> np.ndarray:
    return draw_without_replacement(seed, STREAM_OUTLIER, K, int(np.floor(frac * K + 1e-9)))


def sample_rows(seed: int, M: int, count: int) -> np.ndarray:
    return draw_without_replacement(seed, STREAM_ROWS, M, count)


def _matrix(k: int, rows: int, cols: int, stddev: float, row_gain=None, col_gain=None) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.float32)
    rg = None if row_gain is None else np.ascontiguousarray(row_gain, dtype=np.float64)
    cg = None if col_gain is None else np.ascontiguousarray(col_gain, dtype=np.float64)
    _load().synth_matrix(k, rows, cols, stddev,
                         None if rg is None else rg.ctypes.data,
                         None if cg is None else cg.ctypes.data,
                         out.ctypes.data, _threads())
    return out


def weight_f32(seed: int, N: int, K: int, row_gain_sigma: float = 0.0,
               stddev: float = 0.02) -> np.ndarray:
    gain = None
    if row_gain_sigma:
        gain = np.exp(row_gain_sigma * normal(seed, STREAM_GAIN, N))
    return _matrix(key(seed, STREAM_W), N, K, stddev, row_gain=gain)


def activation_f32(seed: int, M: int, K: int, outlier_frac: float = 0.0,
                   outlier_mult: float = 20.0) -> np.ndarray:
    col = None
    ch = outlier_channels(seed, K, outlier_frac) if outlier_frac else np.empty(0, np.int64)
    if ch.size:
        col = np.ones(K, dtype=np.float64)
        col[ch] = outlier_mult
    return _matrix(key(seed, STREAM_X), M, K, 1.0, col_gain=col)


def to_bf16(a: np.ndarray):
    """float32 array -> torch.bfloat16 CPU tensor (torch's round-to-nearest-even)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t) -> np.ndarray:
    """torch.bfloat16 tensor -> its uint16 bit patterns as a numpy array."""
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
