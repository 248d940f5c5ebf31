"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/fp8blk.h declares, and rejects bad arguments before it
makes any CUDA call."""
import ctypes
import os
import re

import pytest

import block_scaled_fp8_fp8blk_b200 as fb
from block_scaled_fp8_fp8blk_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8blk.h")


@pytest.fixture(scope="module")
def lib():
    fbuild.build_cuda()
    return fb.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FP8BLK_EXPORT\s+[\w\s\*]+?\b(fp8blk_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_symbols()
    for n in ("fp8blk_quantize_weight", "fp8blk_dequantize", "fp8blk_linear_w8a16",
              "fp8blk_linear_w8a8"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(fb.EXPORTS)


def test_version_and_status_strings(lib):
    assert lib.fp8blk_version() == 100
    for code in range(7):
        assert lib.fp8blk_status_string(code)
    assert lib.fp8blk_status_string(99) == b"unknown status"


def test_workspace_size(lib):
    M, N, K = 77, 1000, 1000
    ldqx, ldsx, KB = 1008, 128, 8
    sx_off = -(-M * ldqx // 256) * 256
    assert lib.fp8blk_workspace_size(1, M, N, K) == sx_off + KB * ldsx * 4
    assert lib.fp8blk_workspace_size(0, 0, N, K) == 0
    # W8A16: stream-K partials for M <= 128 (160 CTAs x 2 slots x BT x 128 floats)
    for m, bt in ((1, 16), (16, 16), (17, 32), (64, 64), (77, 128), (128, 128)):
        assert lib.fp8blk_workspace_size(0, m, N, K) == 160 * 2 * bt * 128 * 4
    # M > 128 (optional, for the stream-K last wave): two [256][128] float
    # slots per CTA, for min(160, tiles x KB) CTAs
    assert lib.fp8blk_workspace_size(0, 129, N, K) == 2 * min(160, 1 * 8 * 8) * 256 * 128 * 4
    assert lib.fp8blk_workspace_size(0, 512, 25600, 5120) == 2 * 160 * 256 * 128 * 4
    assert lib.fp8blk_workspace_size(1, M, N, 0) == 0
    assert lib.fp8blk_workspace_size(2, M, N, K) == 0
    assert lib.fp8blk_workspace_size(1, -1, N, K) == 0


# Arguments below are rejected before any CUDA call, so they run without a GPU.
P = 1 << 20          # a 16-byte-aligned fake address (never dereferenced)
PM = P + 2           # misaligned


def test_quantize_weight_validation(lib):
    f = lib.fp8blk_quantize_weight
    assert f(P, -1, 128, 128, P, 128, P, None) == 1
    assert f(P, 0, 128, 128, P, 128, P, None) == 0          # empty: nothing to do
    assert f(P, 128, 0, 128, P, 128, P, None) == 0
    assert f(None, 128, 128, 128, P, 128, P, None) == 1
    assert f(P, 128, 128, 64, P, 128, P, None) == 1         # ldw < K
    assert f(P, 128, 128, 128, P, 100, P, None) == 1        # ldq < K
    assert f(P, 128, 128, 132, P, 128, P, None) == 2        # ldw % 8
    assert f(P, 128, 128, 128, P, 136, P, None) == 2        # ldq % 16
    assert f(PM, 128, 128, 128, P, 128, P, None) == 2
    assert f(P, 128, 128, 128, P, 128, P + 1, None) == 2    # scale pointer 4-byte


def test_dequantize_validation(lib):
    f = lib.fp8blk_dequantize
    assert f(P, 128, P, -5, 128, P, 128, None) == 1
    assert f(P, 128, P, 0, 128, P, 128, None) == 0
    assert f(P, 120, P, 128, 128, P, 128, None) == 1
    assert f(P, 144, P, 128, 128, P, 132, None) == 2
    assert f(PM, 128, P, 128, 128, P, 128, None) == 2


def test_quantize_act_validation(lib):
    f = lib.fp8blk_quantize_act
    assert f(P, 64, 256, 256, P, 256, P, 32, None) == 1     # ldsx < M
    assert f(P, 64, 256, 256, P, 256, P, 66, None) == 2     # ldsx % 4
    assert f(P, 64, 256, 256, P, 256, PM, 64, None) == 2
    assert f(P, 0, 256, 256, P, 256, P, 64, None) == 0


@pytest.mark.parametrize("name", ["fp8blk_linear_w8a16", "fp8blk_linear_w8a8"])
def test_linear_validation(lib, name):
    f = getattr(lib, name)
    M, N, K = 64, 384, 256
    ws = lib.fp8blk_workspace_size(1 if name.endswith("a8") else 0, M, N, K)
    ok = (P, K, P, K, P, P, N, M, N, K, P if ws else None, ws, None)

    def call(**kw):
        a = list(ok)
        idx = dict(x=0, ldx=1, q=2, ldq=3, s=4, y=5, ldy=6, M=7, N=8, K=9, ws=10, wsb=11)
        for k, v in kw.items():
            a[idx[k]] = v
        return f(*a)

    assert call(M=-1) == 1
    assert call(M=0) == 0 and call(N=0) == 0
    assert call(x=None) == 1 and call(q=None) == 1 and call(s=None) == 1 and call(y=None) == 1
    assert call(ldx=K - 8) == 1 and call(ldq=K - 16) == 1 and call(ldy=N - 8) == 1
    assert call(ldx=K + 4) == 2 and call(ldq=K + 8) == 2 and call(ldy=N + 4) == 2
    assert call(x=PM) == 2 and call(q=PM) == 2 and call(y=PM) == 2 and call(s=P + 2) == 2
    if ws:
        assert call(ws=None) == 4
        assert call(wsb=ws - 1) == 4
        assert call(ws=P + 16) == 4   # workspace must be 256-byte aligned


def test_linear_w8a8_quantized_validation(lib):
    f = lib.fp8blk_linear_w8a8_quantized
    M, N, K = 64, 384, 256
    ok = [P, K, P, M, P, K, P, P, N, M, N, K, None]

    def call(**kw):
        a = list(ok)
        idx = dict(qx=0, ldqx=1, sx=2, ldsx=3, q=4, ldq=5, s=6, y=7, ldy=8, M=9, N=10, K=11)
        for k, v in kw.items():
            a[idx[k]] = v
        return f(*a)

    assert call(M=-1) == 1 and call(K=-1) == 1
    assert call(M=0) == 0 and call(N=0) == 0
    assert call(qx=None) == 1 and call(sx=None) == 1 and call(q=None) == 1 and call(y=None) == 1
    assert call(ldqx=K - 16) == 1 and call(ldsx=M - 1) == 1 and call(ldq=K - 16) == 1
    assert call(ldqx=K + 8) == 2 and call(qx=PM) == 2 and call(sx=P + 2) == 2 and call(y=PM) == 2


def test_encode_validation(lib):
    f = lib.fp8blk_encode_e4m3
    assert f(P, -1, P, None) == 1
    assert f(P, 0, P, None) == 0
    assert f(PM, 16, P, None) == 2
    assert f(None, 16, P, None) == 1


def test_read_error_rejects_null(lib):
    assert lib.fp8blk_read_device_error(None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fb, "_lib", None)
    monkeypatch.setattr(fb, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        fb.lib()


def test_stream_slot_bytes(lib):
    # codes 1000 x 1008 = 1008000 -> 1008128 (256-aligned), + 8 x 8 scales x 4 B
    assert lib.fp8blk_stream_slot_bytes(1000, 1000, 1008) == 1008128 + 256
    assert lib.fp8blk_stream_slot_bytes(25600, 5120, 5120) == 25600 * 5120 + 200 * 40 * 4
    assert lib.fp8blk_stream_slot_bytes(0, 0, 0) == 0
    assert lib.fp8blk_stream_slot_bytes(16, 64, 32) == 0      # ldq < K
    assert lib.fp8blk_stream_slot_bytes(-1, 64, 64) == 0


def test_streamed_linears_validation(lib):
    """Every job is checked before any CUDA call, so these run without a GPU."""
    M, N, K = 64, 384, 256
    slot = lib.fp8blk_stream_slot_bytes(N, K, K)
    slot = -(-slot // 256) * 256
    ws = lib.fp8blk_workspace_size(1, M, N, K)
    events = (ctypes.c_void_p * 4)(P, P + 16, P + 32, P + 48)

    def job(**kw):
        d = dict(mode=1, q_host=P, scale_host=P, ldq=K, x=P, ldx=K, y=P, ldy=N, M=M, N=N, K=K)
        d.update(kw)
        return fb.LinearJob(**d)

    def call(jobs, njobs=None, slots=P, slot_bytes=slot, nslots=2, wsp=P, wsb=ws, ev=events):
        arr = (fb.LinearJob * max(1, len(jobs)))(*jobs)
        return lib.fp8blk_streamed_linears(arr, len(jobs) if njobs is None else njobs, slots,
                                           slot_bytes, nslots, wsp, wsb, None, None, ev)

    assert call([], njobs=0) == 0
    assert call([job()], njobs=-1) == 1
    assert call([job()], nslots=0) == 1
    assert call([job()], slots=None) == 1
    assert call([job()], ev=None) == 1
    assert call([job()], slot_bytes=slot + 16) == 2               # slot size % 256
    assert call([job()], slots=P + 16) == 2                       # slots 256-byte aligned
    assert call([job()], ev=(ctypes.c_void_p * 4)(P, None, P, P)) == 1
    assert call([job(mode=2)]) == 1
    assert call([job(), job(N=N * 4, ldy=N * 4)]) == 1           # second job's weights exceed a slot
    assert call([job(ldq=K - 16)]) == 1
    assert call([job(q_host=None)]) == 1
    assert call([job(x=PM)]) == 2
    assert call([job(ldx=K + 4)]) == 2
    assert call([job()], wsp=None) == 4                           # W8A8 needs its workspace
    assert call([job()], wsb=ws - 1) == 4


def test_selftest_wait_timeout_validation(lib):
    assert lib.fp8blk_selftest_wait_timeout(999, None) == 1
    assert lib.fp8blk_selftest_wait_timeout(4_000_000_001, None) == 1


def test_linear_sequence_validation(lib):
    M, N, K = 64, 384, 256
    ws = lib.fp8blk_workspace_size(1, M, N, K)

    def job(**kw):
        d = dict(mode=1, x=P, ldx=K, q=P, ldq=K, scale_inv=P, y=P, ldy=N, M=M, N=N, K=K)
        d.update(kw)
        return fb.LinearArgs(**d)

    def call(jobs, njobs=None, wsp=P, wsb=ws):
        arr = (fb.LinearArgs * max(1, len(jobs)))(*jobs)
        return lib.fp8blk_linear_sequence(arr, len(jobs) if njobs is None else njobs, wsp, wsb, None)

    assert call([], njobs=0) == 0
    assert call([job()], njobs=-1) == 1
    assert lib.fp8blk_linear_sequence(None, 1, P, ws, None) == 1
    assert call([job(mode=3)]) == 1
    assert call([job(), job(x=PM)]) == 2            # every job checked before any launch
    assert call([job(), job(ldq=K + 8)]) == 2
    assert call([job(), job(y=None)]) == 1
    assert call([job()], wsp=None) == 4
    assert call([job(mode=0, M=16)], wsp=None) == 4  # W8A16 stream-K needs the workspace too
