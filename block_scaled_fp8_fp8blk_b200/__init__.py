"""Python binding of the fp8blk C ABI (``include/fp8blk.h``).

Argument marshalling only: every step runs in ``libfp8blk.so`` (hand-written
sm_100a kernels). PyTorch supplies device memory and the current stream.
There is no fallback: if the library is missing or the device is not
compute capability 10.x, the calls raise.

Tensors are 2-D, row-major with unit column stride; the row stride is the
leading dimension, so padded buffers are passed as column slices of a wider
tensor (e.g. ``q = buf[:, :K]`` with ``buf`` of shape ``[N, ldq]``).
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "Fp8BlkError", "lib", "quantize_weight", "dequantize", "quantize_act", "linear_w8a16",
    "linear_w8a8", "linear_w8a8_quantized", "workspace_size", "encode_e4m3", "read_device_error",
    "version", "LinearJob", "stream_slot_bytes", "streamed_linears", "selftest_wait_timeout",
    "LinearArgs", "linear_sequence",
    "LIB_PATH", "EXPORTS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8blk.so")

STATUS = {
    0: "FP8BLK_OK", 1: "FP8BLK_ERR_INVALID_ARG", 2: "FP8BLK_ERR_ALIGNMENT",
    3: "FP8BLK_ERR_UNSUPPORTED_DEVICE", 4: "FP8BLK_ERR_WORKSPACE", 5: "FP8BLK_ERR_CUDA",
    6: "FP8BLK_ERR_TIMEOUT",
}

_i64, _p, _sz, _int = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_st = ctypes.c_int


class LinearJob(ctypes.Structure):
    """fp8blk_linear_job: one linear of a streamed sequence (host weights)."""
    _fields_ = [("mode", ctypes.c_int32), ("q_host", _p), ("scale_host", _p), ("ldq", _i64),
                ("x", _p), ("ldx", _i64), ("y", _p), ("ldy", _i64),
                ("M", _i64), ("N", _i64), ("K", _i64)]


class LinearArgs(ctypes.Structure):
    """fp8blk_linear_args: one linear of a sequence (device weights)."""
    _fields_ = [("mode", ctypes.c_int32), ("x", _p), ("ldx", _i64), ("q", _p), ("ldq", _i64),
                ("scale_inv", _p), ("y", _p), ("ldy", _i64), ("M", _i64), ("N", _i64), ("K", _i64)]


# name -> (restype, argtypes), mirroring include/fp8blk.h
EXPORTS = {
    "fp8blk_quantize_weight": (_st, [_p, _i64, _i64, _i64, _p, _i64, _p, _p]),
    "fp8blk_dequantize": (_st, [_p, _i64, _p, _i64, _i64, _p, _i64, _p]),
    "fp8blk_quantize_act": (_st, [_p, _i64, _i64, _i64, _p, _i64, _p, _i64, _p]),
    "fp8blk_linear_w8a16": (_st, [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "fp8blk_linear_w8a8": (_st, [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "fp8blk_linear_w8a8_noalloc": (_st, [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p]),
    "fp8blk_linear_w8a8_quantized": (_st, [_p, _i64, _p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p]),
    "fp8blk_workspace_size": (_sz, [_int, _i64, _i64, _i64]),
    "fp8blk_stream_slot_bytes": (_sz, [_i64, _i64, _i64]),
    "fp8blk_linear_sequence": (_st, [ctypes.POINTER(LinearArgs), _i64, _p, _sz, _p]),
    "fp8blk_streamed_linears": (_st, [ctypes.POINTER(LinearJob), _i64, _p, _sz, ctypes.c_int32,
                                      _p, _sz, _p, _p, ctypes.POINTER(_p)]),
    "fp8blk_encode_e4m3": (_st, [_p, _i64, _p, _p]),
    "fp8blk_read_device_error": (_st, [ctypes.POINTER(ctypes.c_uint32)]),
    "fp8blk_selftest_wait_timeout": (_st, [_i64, _p]),
    "fp8blk_status_string": (ctypes.c_char_p, [_int]),
    "fp8blk_version": (_int, []),
}

_lib = None


class Fp8BlkError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call} failed: {STATUS.get(status, status)}")


def lib() -> ctypes.CDLL:
    """The loaded libfp8blk.so (loaded once; raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "python -m block_scaled_fp8_fp8blk_b200.build")
        import torch  # noqa: F401  (loads the CUDA runtime the library shares)
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            f = getattr(handle, name)
            f.restype, f.argtypes = res, args
        _lib = handle
    return _lib


def _check(status: int, call: str) -> None:
    if status != 0:
        raise Fp8BlkError(status, call)


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def _round_up(a: int, b: int) -> int:
    return _cdiv(a, b) * b


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _ld(t) -> int:
    if t.dim() != 2:
        raise ValueError("expected a 2-D tensor")
    if t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError("expected unit column stride")
    return max(t.stride(0), t.shape[1]) if t.shape[0] > 1 else max(t.shape[1], t.stride(0), 1)


def _padded(rows: int, cols: int, ld: int, dtype, device):
    import torch
    return torch.empty((rows, ld), dtype=dtype, device=device)[:, :cols]


def version() -> int:
    return int(lib().fp8blk_version())


def workspace_size(mode: int, M: int, N: int, K: int) -> int:
    return int(lib().fp8blk_workspace_size(mode, M, N, K))


def quantize_weight(w, q=None, scale_inv=None, ldq: int | None = None):
    """BF16 w [N, K] -> (q uint8 [N, K] with row stride ldq, scale_inv float32 [NB, KB])."""
    import torch
    N, K = w.shape
    if q is None:
        q = _padded(N, K, ldq or _round_up(max(K, 1), 16), torch.uint8, w.device)
    if scale_inv is None:
        scale_inv = torch.empty((_cdiv(N, 128), _cdiv(K, 128)), dtype=torch.float32, device=w.device)
    _check(lib().fp8blk_quantize_weight(w.data_ptr(), N, K, _ld(w), q.data_ptr(), _ld(q),
                                        scale_inv.data_ptr(), _stream()), "fp8blk_quantize_weight")
    return q, scale_inv


def dequantize(q, scale_inv, out=None):
    import torch
    N, K = q.shape
    if out is None:
        out = _padded(N, K, _round_up(max(K, 1), 8), torch.bfloat16, q.device)
    _check(lib().fp8blk_dequantize(q.data_ptr(), _ld(q), scale_inv.data_ptr(), N, K,
                                   out.data_ptr(), _ld(out), _stream()), "fp8blk_dequantize")
    return out


def quantize_act(x, qx=None, sx=None):
    """BF16 x [M, K] -> (qx uint8 [M, K], sx float32 [KB, ldsx] with ldsx = round_up(M, 4))."""
    import torch
    M, K = x.shape
    if qx is None:
        qx = _padded(M, K, _round_up(max(K, 1), 16), torch.uint8, x.device)
    if sx is None:
        sx = torch.empty((_cdiv(K, 128), _round_up(max(M, 1), 4)), dtype=torch.float32, device=x.device)
    _check(lib().fp8blk_quantize_act(x.data_ptr(), M, K, _ld(x), qx.data_ptr(), _ld(qx),
                                     sx.data_ptr(), sx.stride(0), _stream()), "fp8blk_quantize_act")
    return qx, sx


def _linear(mode: int, name: str, x, q, scale_inv, out, workspace):
    import torch
    M, K = x.shape
    N = q.shape[0]
    if q.shape[1] != K:
        raise ValueError("x and q disagree on K")
    if out is None:
        out = _padded(M, N, _round_up(max(N, 1), 8), torch.bfloat16, x.device)
    need = workspace_size(mode, M, N, K)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(getattr(lib(), name)(x.data_ptr(), _ld(x), q.data_ptr(), _ld(q), scale_inv.data_ptr(),
                                out.data_ptr(), _ld(out), M, N, K, ws_ptr, ws_len, _stream()), name)
    return out


def linear_w8a16(x, q, scale_inv, out=None, workspace=None):
    """y = x . dequant(q, scale_inv)^T with BF16 activations; y BF16 [M, N]."""
    return _linear(0, "fp8blk_linear_w8a16", x, q, scale_inv, out, workspace)


def linear_w8a8(x, q, scale_inv, out=None, workspace=None):
    """y = x . dequant(q, scale_inv)^T with x quantized per 1x128 K-group to E4M3."""
    return _linear(1, "fp8blk_linear_w8a8", x, q, scale_inv, out, workspace)


def linear_w8a8_quantized(qx, sx, q, scale_inv, M=None, out=None):
    """W8A8 linear on (qx, sx) from quantize_act; M defaults to qx.shape[0]."""
    import torch
    M = qx.shape[0] if M is None else M
    K = qx.shape[1]
    N = q.shape[0]
    if out is None:
        out = _padded(M, N, _round_up(max(N, 1), 8), torch.bfloat16, qx.device)
    _check(lib().fp8blk_linear_w8a8_quantized(qx.data_ptr(), _ld(qx), sx.data_ptr(), sx.stride(0),
                                              q.data_ptr(), _ld(q), scale_inv.data_ptr(),
                                              out.data_ptr(), _ld(out), M, N, K, _stream()),
           "fp8blk_linear_w8a8_quantized")
    return out


def linear_sequence(jobs, workspace=None):
    """Runs linears back to back with their weight streams overlapping the
    kernels before them (fp8blk_linear_sequence). jobs: list of
    (mode, x, q, scale_inv, y) with mode 0 = W8A16, 1 = W8A8, all CUDA
    tensors as for linear_w8a16 / linear_w8a8. The workspace (allocated here
    if None) must cover the largest workspace_size over the jobs."""
    import torch
    arr = (LinearArgs * max(1, len(jobs)))()
    need = 0
    for i, (mode, x, q, s, y) in enumerate(jobs):
        M, K = x.shape
        N = q.shape[0]
        if q.shape[1] != K or y.shape != (M, N):
            raise ValueError("job shapes disagree")
        arr[i] = LinearArgs(mode, x.data_ptr(), _ld(x), q.data_ptr(), _ld(q), s.data_ptr(),
                            y.data_ptr(), _ld(y), M, N, K)
        need = max(need, workspace_size(mode, M, N, K))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=jobs[0][1].device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().fp8blk_linear_sequence(arr, len(jobs), ws_ptr, ws_len, _stream()),
           "fp8blk_linear_sequence")


def stream_slot_bytes(N: int, K: int, ldq: int) -> int:
    return lib().fp8blk_stream_slot_bytes(N, K, ldq)


def streamed_linears(jobs, slots, slot_bytes: int, nslots: int, workspace, compute, copy, events):
    """Run linears whose weights are in (pinned) host memory through nslots
    device weight slots (fp8blk_streamed_linears).

    jobs: list of (mode, q_host, s_host, x, y) with mode 0 = W8A16, 1 = W8A8,
    q_host uint8 [N, K] / s_host float32 (CPU tensors, pinned for overlap;
    q_host's row stride is ldq), x BF16 [M, K] and y BF16 [M, N] on the GPU.
    slots: uint8 CUDA tensor of nslots * slot_bytes; compute / copy:
    torch.cuda.Stream; events: 2 * nslots torch.cuda.Event (created here by
    a first record on `compute` if they have no handle yet).
    """
    arr = (LinearJob * max(1, len(jobs)))()
    for i, (mode, qh, sh, x, y) in enumerate(jobs):
        M, K = x.shape
        N = qh.shape[0]
        if qh.shape[1] != K or y.shape != (M, N):
            raise ValueError("job shapes disagree")
        arr[i] = LinearJob(mode, qh.data_ptr(), sh.data_ptr(), _ld(qh), x.data_ptr(), _ld(x),
                           y.data_ptr(), _ld(y), M, N, K)
    for e in events:
        if not e.cuda_event:
            e.record(compute)
    ev = (_p * max(1, len(events)))(*[e.cuda_event for e in events])
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().fp8blk_streamed_linears(arr, len(jobs), slots.data_ptr(), slot_bytes, nslots,
                                         ws_ptr, ws_len, compute.cuda_stream, copy.cuda_stream, ev),
           "fp8blk_streamed_linears")


def encode_e4m3(v):
    import torch
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _check(lib().fp8blk_encode_e4m3(v.data_ptr(), v.numel(), out.data_ptr(), _stream()),
           "fp8blk_encode_e4m3")
    return out


def selftest_wait_timeout(limit_cycles: int = 2_000_000) -> None:
    """Launches the failure-detection self-test (a bounded wait that runs out)."""
    _check(lib().fp8blk_selftest_wait_timeout(limit_cycles, _stream()),
           "fp8blk_selftest_wait_timeout")


def read_device_error() -> int:
    """Reads and clears the device error word (synchronizes the device)."""
    word = ctypes.c_uint32(0)
    st = lib().fp8blk_read_device_error(ctypes.byref(word))
    if st not in (0, 6):
        raise Fp8BlkError(st, "fp8blk_read_device_error")
    return int(word.value)
