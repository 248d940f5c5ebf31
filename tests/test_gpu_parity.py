"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: the E4M3 codec (every float32 bit pattern), the converter, the
dequantizer and the activation quantizer. Within tolerance (relative Frobenius
2e-3, per element 2^-7 |ref| + 1e-2 rms(ref)): both linears, on every
workload shape, full outputs for the small ones and seeded row samples at
full size. Plus edge cases: empty sizes, K = 0, ragged tiles, padded leading
dimensions with canaries, one-hot rows."""
import numpy as np
import pytest
import torch

import block_scaled_fp8_fp8blk_b200 as fb
import oracle
from block_scaled_fp8_fp8blk_b200 import synth, workloads as W
from helpers import bf16_bits, bf16_to_f64, check_linear, tie_heavy_weight

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    major, _ = torch.cuda.get_device_capability(0)
    assert major == 10, "the library targets compute capability 10.x"
    torch.cuda.set_device(0)
    fb.lib()
    yield
    assert fb.read_device_error() == 0, "a kernel reported a timed-out wait"


def to_dev_bf16(bits: np.ndarray, ld: int | None = None):
    R, C = bits.shape
    ld = ld or -(-C // 8) * 8
    buf = torch.zeros((R, ld), dtype=torch.int16)
    buf[:, :C] = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return buf.view(torch.bfloat16).to(DEV)[:, :C]


def to_dev_u8(a: np.ndarray, ld: int | None = None):
    R, C = a.shape
    ld = ld or -(-C // 16) * 16
    buf = torch.zeros((R, ld), dtype=torch.uint8)
    buf[:, :C] = torch.from_numpy(np.ascontiguousarray(a))
    return buf.to(DEV)[:, :C]


def u8(t) -> np.ndarray:
    return t.detach().cpu().numpy()


_W_CACHE = {}


def weight_case(wl):
    """(W bits, oracle q, oracle s) for a workload's weight, cached."""
    key = (wl.N, wl.K, wl.row_gain_sigma, wl.seed)
    if key not in _W_CACHE:
        _W_CACHE.clear()
        wb = synth.bf16_bits(wl.weight_bf16())
        q, s = oracle.quantize_weight(wb)
        _W_CACHE[key] = (wb, q, s)
    return _W_CACHE[key]


# ------------------------------------------------------------------ codec
def test_encode_every_float32():
    n = 1 << 28
    for lo in range(0, 1 << 32, n):
        v = torch.arange(n, dtype=torch.int64, device=DEV) + lo
        v = torch.where(v >= (1 << 31), v - (1 << 32), v).to(torch.int32).view(torch.float32)
        codes = u8(fb.encode_e4m3(v))
        del v
        assert oracle.count_code_mismatches(lo, codes) == 0, hex(lo)


# -------------------------------------------------------------- converter
CONVERTER_CASES = [W.TINY, W.RAGGED, W.Workload("one", 1, 1, 1), W.Workload("odd", 3, 200, 129),
                   W.Workload("full128", 1, 256, 256, row_gain_sigma=1.0), W.QKV, W.LINEAR_512]


@pytest.mark.parametrize("wl", CONVERTER_CASES, ids=lambda w: w.name)
def test_quantize_weight_bit_exact(wl):
    wb, q_ref, s_ref = weight_case(wl)
    ldw = -(-wl.K // 8) * 8 + (8 if wl is W.RAGGED else 0)
    ldq = -(-wl.K // 16) * 16 + (16 if wl in (W.RAGGED, W.TINY) else 0)
    w_d = to_dev_bf16(wb, ldw)
    qbuf = torch.full((wl.N, ldq), 0xA5, dtype=torch.uint8, device=DEV)
    s_d = torch.full((-(-wl.N // 128), -(-wl.K // 128)), -1.0, device=DEV)
    fb.quantize_weight(w_d, q=qbuf[:, :wl.K], scale_inv=s_d)
    qh = u8(qbuf)
    assert np.array_equal(qh[:, :wl.K], q_ref)
    assert np.all(qh[:, wl.K:] == 0xA5), "wrote past K"
    assert np.array_equal(s_d.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quantize_zero_blocks_and_signs():
    N, K = 260, 300
    w = np.zeros((N, K), np.float32)
    w[0, 0] = -0.0
    w[:128, 128:256] = -0.0
    w[200, 299] = 3.0
    w[200, 298] = -1e-30
    w[5, 200] = 2.0 ** -130          # a BF16 subnormal block amax
    w[6, 201] = -2.0 ** -133
    wb = synth.bf16_bits(synth.to_bf16(w))
    q_ref, s_ref = oracle.quantize_weight(wb)
    q_d, s_d = fb.quantize_weight(to_dev_bf16(wb))
    assert np.array_equal(u8(q_d), q_ref)
    assert np.array_equal(s_d.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quantize_tie_heavy_blocks():
    """Blocks whose quotients v / s sit exactly on E4M3 decision points (the
    product bracket straddles there and the exact quotient decides, ties to
    even): per warp of 16 rows none, a few, 31 / 33 / 40 / 63 / 64 / 65 of
    them, and whole blocks of them, with ragged edges."""
    wb = tie_heavy_weight()
    q_ref, s_ref = oracle.quantize_weight(wb)
    q_d, s_d = fb.quantize_weight(to_dev_bf16(wb))
    assert np.array_equal(s_d.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(u8(q_d), q_ref)


@pytest.mark.parametrize("amax_exp", [0, 120, -90])
def test_quantize_every_mantissa_pair(amax_exp):
    """One block per BF16 block-maximum mantissa (amax = 1.m x 2^amax_exp,
    128 blocks) holding every BF16 mantissa at every exponent from the
    maximum's down past the E4M3 zero threshold, both signs. E4M3(v / s)
    depends on the two mantissas and the exponent gap only, so this covers
    every case the converter's per-block multiplier (or, where none passes,
    its product bracket) can meet at these magnitudes."""
    blocks = []
    for ma in range(128):
        amax = (1.0 + ma / 128.0) * 2.0 ** amax_exp
        vals = [amax]
        for e in range(0, -26, -1):
            v = (1.0 + np.arange(128) / 128.0) * 2.0 ** (amax_exp + e)
            v = v[v <= amax]
            vals.extend(np.stack([v, -v], axis=1).ravel().tolist())
        blk = np.zeros(128 * 128, np.float64)
        blk[:len(vals)] = vals
        blocks.append(blk.reshape(128, 128))
    w = np.concatenate(blocks, axis=1).astype(np.float32)
    wb = synth.bf16_bits(synth.to_bf16(w))
    assert np.array_equal((wb.astype(np.uint32) << 16).view(np.float32), w)  # exact in BF16
    q_ref, s_ref = oracle.quantize_weight(wb)
    q_d, s_d = fb.quantize_weight(to_dev_bf16(wb))
    assert np.array_equal(s_d.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(u8(q_d), q_ref)


def test_quantize_every_bf16_value():
    allb = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = (allb.astype(np.uint32) << 16).view(np.float32)
    v = allb[np.isfinite(vals)]
    n = -(-v.size // 128) * 128
    wb = np.zeros(n, np.uint16)
    wb[:v.size] = v
    wb = wb.reshape(-1, 128)
    q_ref, s_ref = oracle.quantize_weight(wb)
    q_d, s_d = fb.quantize_weight(to_dev_bf16(wb))
    assert np.array_equal(u8(q_d), q_ref)
    assert np.array_equal(s_d.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# ------------------------------------------------------------ dequantizer
@pytest.mark.parametrize("wl", [W.TINY, W.RAGGED, W.Workload("odd", 3, 200, 129), W.LINEAR_512,
                                W.QKV, W.O_PROJ, W.GATE_UP, W.DOWN], ids=lambda w: w.name)
def test_dequantize_bit_exact(wl):
    wb, q, s = weight_case(wl)
    ref = oracle.dequantize(q, s)
    ldw = -(-wl.K // 8) * 8 + 8
    out = torch.full((wl.N, ldw), 0x7FC1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    fb.dequantize(to_dev_u8(q), torch.from_numpy(s).to(DEV), out=out[:, :wl.K])
    got = bf16_bits(out)
    assert np.array_equal(got[:, :wl.K], ref)
    assert np.all(got[:, wl.K:] == 0x7FC1)


def test_dequantize_all_codes_many_scales():
    rng = np.random.default_rng(7)
    codes = np.tile(np.arange(256, dtype=np.uint8), (256, 2))   # [256, 512]
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0x00
    s = (rng.random((2, 4)) * 10.0 ** rng.integers(-30, 3, (2, 4))).astype(np.float32)
    s[0, 0] = 0.0
    s[1, 3] = 1.0
    ref = oracle.dequantize(codes, s)
    got = bf16_bits(fb.dequantize(to_dev_u8(codes), torch.from_numpy(s).to(DEV)))
    assert np.array_equal(got, ref)


# --------------------------------------------------- activation quantizer
@pytest.mark.parametrize("wl", [W.TINY, W.RAGGED, W.Workload("k130", 5, 130, 8), W.LINEAR_512,
                                W.O_PROJ, W.DOWN, W.LARGE_4096, W.LARGE_16384],
                         ids=lambda w: w.name)
def test_quantize_act_bit_exact(wl):
    xb = synth.bf16_bits(wl.x_bf16())
    qx_ref, sx_ref = oracle.act_quant(xb)
    qx_d, sx_d = fb.quantize_act(to_dev_bf16(xb, -(-wl.K // 8) * 8 + 8))
    assert np.array_equal(u8(qx_d), qx_ref)
    sx = sx_d.cpu().numpy()[:, :wl.M].T       # group-major -> [M][KB]
    assert np.array_equal(sx.view(np.uint32), sx_ref.view(np.uint32))


# ---------------------------------------------------------------- linears
LINEAR_FULL = [W.TINY, W.RAGGED, W.Workload("k130_n300", 50, 130, 300),
               W.Workload("m200_k384_n640", 200, 384, 640, row_gain_sigma=0.5),
               W.Workload("m130_k256_n13", 130, 256, 13),
               W.Workload("m40_k128_n5", 40, 128, 5)]
LINEAR_SAMPLED = [W.QKV, W.O_PROJ, W.GATE_UP, W.DOWN, W.LINEAR_512, W.LARGE_4096, W.LARGE_16384]
SMALL_M = [w.with_m(m) for w in W.DECODER_SHAPES for m in W.SMALL_M]


def run_linear(wl, mode, rows=None, ldx_pad=0, ldy_pad=0):
    wb, q_ref, s_ref = weight_case(wl)
    xb = synth.bf16_bits(wl.x_bf16())
    q_d, s_d = fb.quantize_weight(to_dev_bf16(wb))
    assert np.array_equal(u8(q_d), q_ref)
    x_d = to_dev_bf16(xb, -(-wl.K // 8) * 8 + ldx_pad)
    ldy = -(-wl.N // 8) * 8 + ldy_pad
    ybuf = torch.full((wl.M, ldy), 0x7FC1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    f = fb.linear_w8a16 if mode == "w8a16" else fb.linear_w8a8
    f(x_d, q_d, s_d, out=ybuf[:, :wl.N])
    torch.cuda.synchronize()
    ybits = bf16_bits(ybuf)
    assert np.all(ybits[:, wl.N:] == 0x7FC1), "wrote past N"
    if mode == "w8a16":
        ref = oracle.linear_w8a16(xb, q_ref, s_ref, wl.N, wl.K, rows=rows)
    else:
        qx, sx = oracle.act_quant(xb)
        ref = oracle.linear_w8a8(qx, sx, q_ref, s_ref, wl.N, wl.K, rows=rows)
    y = bf16_to_f64(ybuf[:, :wl.N])
    if rows is not None:
        y = y[rows]
    return check_linear(y, ref, f"{wl.name}/{mode}")


@pytest.mark.parametrize("mode", ["w8a16", "w8a8"])
@pytest.mark.parametrize("wl", LINEAR_FULL, ids=lambda w: w.name)
def test_linear_full_output(wl, mode):
    run_linear(wl, mode, ldx_pad=8, ldy_pad=8)


@pytest.mark.parametrize("mode", ["w8a16", "w8a8"])
@pytest.mark.parametrize("wl", SMALL_M, ids=lambda w: w.name)
def test_linear_small_m(wl, mode):
    run_linear(wl, mode, rows=wl.checked_rows(64))


@pytest.mark.parametrize("mode", ["w8a16", "w8a8"])
@pytest.mark.parametrize("wl", LINEAR_SAMPLED, ids=lambda w: w.name)
def test_linear_full_size_sampled_rows(wl, mode):
    count = 256 if wl.M > 512 else 64
    run_linear(wl, mode, rows=wl.checked_rows(count))


@pytest.mark.parametrize("mode", ["w8a16", "w8a8"])
def test_linear_empty_and_k0(mode):
    f = fb.linear_w8a16 if mode == "w8a16" else fb.linear_w8a8
    q = torch.zeros((16, 0), dtype=torch.uint8, device=DEV)
    s = torch.zeros((1, 1), dtype=torch.float32, device=DEV)
    x = torch.zeros((8, 0), dtype=torch.bfloat16, device=DEV)
    y = torch.full((8, 16), 1.0, dtype=torch.bfloat16, device=DEV)
    f(x, q, s, out=y)
    assert torch.all(y == 0)
    x2 = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    q2 = torch.zeros((16, 64), dtype=torch.uint8, device=DEV)
    y2 = f(x2, q2, s)
    assert y2.shape == (0, 16)


def test_w8a16_one_hot_rows_reproduce_dequantized_weight():
    # x = e_k gives P = the exact BF16 image of the code, acc = fl(code * s),
    # y = BF16(acc) -- the dequantizer's value, bit for bit.
    wl = W.RAGGED
    wb, q, s = weight_case(wl)
    ks = np.array([0, 1, 127, 128, 500, 999])
    x = np.zeros((ks.size, wl.K), np.float32)
    x[np.arange(ks.size), ks] = 1.0
    y = fb.linear_w8a16(to_dev_bf16(synth.bf16_bits(synth.to_bf16(x))), to_dev_u8(q),
                        torch.from_numpy(s).to(DEV))
    deq = oracle.dequantize(q, s)
    got = bf16_bits(y)
    for i, k in enumerate(ks):
        assert np.array_equal(got[i], deq[:, k])


@pytest.mark.parametrize("M", [16, 128, 300])
def test_w8a16_every_code_through_the_gemm(M):
    """Every E4M3 code (NaNs excepted) as a weight, identity activations: each
    output is one code times its block scale, rounded once, so y must equal
    the dequantized weight bit for bit (zeros as +0) -- this pins the
    kernel's FP8 -> BF16 expansion on all 254 finite codes, subnormals
    included, on the small-token (M <= 128) and the two-sub-tile (M > 128)
    paths."""
    N, K = 256, 128
    q = (np.arange(N * K, dtype=np.int64).reshape(N, K) % 256).astype(np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x00
    s = np.array([[1.0], [2.0 ** -100]], dtype=np.float32)
    x = np.zeros((M, K), np.float32)
    x[np.arange(M), np.arange(M) % K] = 1.0
    y = fb.linear_w8a16(to_dev_bf16(synth.bf16_bits(synth.to_bf16(x))), to_dev_u8(q),
                        torch.from_numpy(s).to(DEV))
    got = bf16_bits(y)
    want = oracle.dequantize(q, s)[:, np.arange(M) % K].T.copy()   # [M, N]
    # a zero code's product is summed with the other columns' zero products,
    # so it comes out +0 whatever its sign (IEEE: -0 + +0 = +0)
    want[want == 0x8000] = 0
    assert np.array_equal(got, want)


def test_repeat_calls_are_deterministic():
    wl = W.Workload("m300_k640_n512", 300, 640, 512)
    wb, q, s = weight_case(wl)
    x_d = to_dev_bf16(synth.bf16_bits(wl.x_bf16()))
    q_d, s_d = to_dev_u8(q), torch.from_numpy(s).to(DEV)
    for f in (fb.linear_w8a16, fb.linear_w8a8):
        a = bf16_bits(f(x_d, q_d, s_d))
        b = bf16_bits(f(x_d, q_d, s_d))
        assert np.array_equal(a, b)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["w8a16", "w8a8"])
def test_large_repeat_calls_are_deterministic(mode):
    """Many tiles per CTA, so every ring in the persistent GEMMs wraps many
    times: six calls must give bit-identical outputs (a ring-reuse race shows
    up as a sub-tile or a band of weight rows differing between calls)."""
    M, K, N = 4096, 5120, 25600
    g = torch.Generator(device="cpu").manual_seed(7)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    q_d, s_d = fb.quantize_weight(w)
    f = fb.linear_w8a16 if mode == "w8a16" else fb.linear_w8a8
    first = f(x, q_d, s_d)
    out = torch.empty_like(first)
    for _ in range(5):
        f(x, q_d, s_d, out=out)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), first.view(torch.int16))
    assert fb.read_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("M", [300, 512])
def test_w8a16_stream_k_last_wave(M):
    """Above 128 tokens the last wave of 256-token tiles runs stream-K when
    the workspace allows (partials summed by the fix-up in slab order): the
    output is within tolerance of the oracle on sampled rows, bit-identical
    over repeated calls, and equal to the all-whole-tiles run (no
    workspace) within the linear tolerance."""
    wl = W.Workload(f"m{M}_k5120_n25600", M, 5120, 25600)
    wb, q, s = weight_case(wl)
    xb = synth.bf16_bits(wl.x_bf16())
    x_d = to_dev_bf16(xb)
    q_d, s_d = to_dev_u8(q), torch.from_numpy(s).to(DEV)
    ws = torch.empty(fb.workspace_size(0, M, wl.N, wl.K), dtype=torch.uint8, device=DEV)
    first = fb.linear_w8a16(x_d, q_d, s_d, workspace=ws)
    out = torch.empty_like(first)
    for _ in range(4):
        fb.linear_w8a16(x_d, q_d, s_d, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), first.view(torch.int16))
    rows = wl.checked_rows(64)
    ref = oracle.linear_w8a16(xb, q, s, wl.N, wl.K, rows=rows)
    check_linear(bf16_to_f64(first)[rows], ref, f"{wl.name}/stream-K last wave")
    whole = bf16_to_f64(_w8a16_no_workspace(x_d, q_d, s_d))
    check_linear(whole[rows], ref, f"{wl.name}/whole tiles")
    assert fb.read_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("mode,N", [("w8a16", 384), ("w8a16", 1000), ("w8a8", 1000)])
def test_large_token_raster_groups(mode, N):
    """9000 tokens with K = 3000 put more activation bytes in flight than one
    raster group holds, so the GEMMs walk their tiles in two unequal groups
    (W8A16 with 256-token tiles: 18 + 18 of 36; W8A8 with 128-token tiles:
    36 + 35 of 71). N = 384 leaves the W8A16 tiles in one short wave that
    runs stream-K; N = 1000 is ragged. Sampled rows (spread over both groups)
    match the oracle, and repeated calls are bit-identical."""
    wl = W.Workload(f"m9000_k3000_n{N}", 9000, 3000, N)
    wb, q, s = weight_case(wl)
    xb = synth.bf16_bits(wl.x_bf16())
    x_d = to_dev_bf16(xb)
    q_d, s_d = to_dev_u8(q), torch.from_numpy(s).to(DEV)
    f = fb.linear_w8a16 if mode == "w8a16" else fb.linear_w8a8
    first = f(x_d, q_d, s_d)
    again = f(x_d, q_d, s_d)
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), first.view(torch.int16))
    rows = np.unique(np.r_[wl.checked_rows(96), [0, 4607, 4608, 8999]])
    if mode == "w8a16":
        ref = oracle.linear_w8a16(xb, q, s, wl.N, wl.K, rows=rows)
    else:
        qx, sx = oracle.act_quant(xb)
        ref = oracle.linear_w8a8(qx, sx, q, s, wl.N, wl.K, rows=rows)
    check_linear(bf16_to_f64(first)[rows], ref, f"{mode}/{wl.name}")
    assert fb.read_device_error() == 0


def _w8a16_no_workspace(x, q, s):
    """W8A16 through the C ABI with no workspace (every tile whole)."""
    M, K = x.shape
    N = q.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    st = fb.lib().fp8blk_linear_w8a16(x.data_ptr(), x.stride(0), q.data_ptr(), q.stride(0),
                                      s.data_ptr(), y.data_ptr(), y.stride(0), M, N, K, None, 0,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    return y


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 16, 64, 128])
def test_small_m_repeat_calls_are_deterministic(M):
    """Stream-K at small token counts (both linears): split tiles are summed
    by the fix-up in a fixed order, so repeated calls must be bit-identical
    (a race in any ring shows up as differing rows)."""
    K, N = 5120, 51200
    g = torch.Generator(device="cpu").manual_seed(11)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    q_d, s_d = fb.quantize_weight(w)
    for f in (fb.linear_w8a16, fb.linear_w8a8):
        first = f(x, q_d, s_d)
        out = torch.empty_like(first)
        for _ in range(5):
            f(x, q_d, s_d, out=out)
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int16), first.view(torch.int16))
    assert fb.read_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [W.RAGGED, W.Workload("m300_k640_n512", 300, 640, 512), W.QKV],
                         ids=lambda w: w.name)
def test_linear_w8a8_quantized(wl):
    """Activations quantized once (fp8blk_quantize_act), then the GEMM on
    them: within the linear tolerance of the oracle's W8A8 result, and bit for
    bit what fp8blk_linear_w8a8 gives (the same kernels on the same codes)."""
    wb, q, s = weight_case(wl)
    xb = synth.bf16_bits(wl.x_bf16())
    x_d = to_dev_bf16(xb, -(-wl.K // 8) * 8)
    q_d, s_d = to_dev_u8(q), torch.from_numpy(s).to(DEV)
    qx, sx = fb.quantize_act(x_d)
    y = fb.linear_w8a8_quantized(qx, sx, q_d, s_d)
    torch.cuda.synchronize()
    rows = wl.checked_rows(64)
    qx_ref, sx_ref = oracle.act_quant(xb)
    ref = oracle.linear_w8a8(qx_ref, sx_ref, q, s, wl.N, wl.K, rows=rows)
    check_linear(bf16_to_f64(y)[rows], ref, f"{wl.name}/w8a8_quantized")
    assert np.array_equal(bf16_bits(y), bf16_bits(fb.linear_w8a8(x_d, q_d, s_d)))


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [W.RAGGED, W.LINEAR_512, W.GATE_UP.with_m(64)], ids=lambda w: w.name)
def test_library_bf16_route_within_tolerance(wl):
    """The pages' Hopper route as the benchmark runs it -- our dequantizer,
    then a library BF16 matmul (FP32 accumulation, no reduced-precision
    reduction) on the expanded weight. Its own definition is y = x . Wd^T with
    Wd the BF16 dequantized weight (rounded before the matmul, unlike the
    fused call); the output is within the linear tolerance of that, computed
    from the oracle's dequantized weight in FP64."""
    wb, q, s = weight_case(wl)
    xb = synth.bf16_bits(wl.x_bf16())
    x_d = to_dev_bf16(xb, -(-wl.K // 8) * 8)
    wd = fb.dequantize(to_dev_u8(q), torch.from_numpy(s).to(DEV))
    prev = torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction
    torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = False
    try:
        y = torch.matmul(x_d, wd.t())
        torch.cuda.synchronize()
    finally:
        torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = prev
    rows = wl.checked_rows(64)
    wd_ref = oracle.dequantize(q, s)
    assert np.array_equal(bf16_bits(wd), wd_ref)
    f64 = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = f64(xb[rows]) @ f64(wd_ref).T
    check_linear(bf16_to_f64(y)[rows], ref, f"{wl.name}/dequantize+matmul")


# ------------------------------------------------------- weight streaming
STREAM_JOBS = [(0, 64, 1024, 1536), (1, 300, 640, 512), (0, 1, 5120, 2048), (1, 77, 1000, 1000),
               (0, 200, 384, 640), (0, 16, 256, 384), (1, 8, 2048, 1024)]


_STREAM_REFS = {}


def stream_oracle_refs(jobs_w, jobs_x):
    """Oracle codes, scales and FP64 outputs of the streamed jobs (cached:
    the inputs are the same seeded tensors for every slot count)."""
    key = tuple(int(w.shape[0]) for w in jobs_w)
    if key not in _STREAM_REFS:
        refs = []
        for (mode, M, K, N), w, x in zip(STREAM_JOBS, jobs_w, jobs_x):
            wb, xb = bf16_bits(w), bf16_bits(x)
            q, s = oracle.quantize_weight(wb)
            if mode == 0:
                r = oracle.linear_w8a16(xb, q, s, N, K)
            else:
                qx, sx = oracle.act_quant(xb)
                r = oracle.linear_w8a8(qx, sx, q, s, N, K)
            refs.append((q, s, r))
        _STREAM_REFS[key] = refs
    return _STREAM_REFS[key]


@pytest.mark.gpu
@pytest.mark.parametrize("nslots", [1, 2, 3])
def test_streamed_linears(nslots):
    """Weights streamed from pinned host memory through nslots device slots:
    every output within the linear tolerance of the oracle of its mode, and
    bit for bit what the same linears give on resident weights."""
    g = torch.Generator(device="cpu").manual_seed(21)
    jobs, ref, outs, slot = [], [], [], 0
    ws_need = 0
    ws_cpu, xs_cpu, codes = [], [], []
    for mode, M, K, N in STREAM_JOBS:
        w_cpu = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
        w = w_cpu.to(DEV)
        ldx = -(-K // 8) * 8
        x = torch.randn(M, ldx, generator=g).to(torch.bfloat16).to(DEV)[:, :K]
        ws_cpu.append(w_cpu)
        xs_cpu.append(x.cpu())
        q, s = fb.quantize_weight(w)
        codes.append((q, s))
        ldq = q.stride(0)
        qh = torch.empty((N, ldq), dtype=torch.uint8, pin_memory=True)
        qh[:, :K] = q.cpu()
        sh = s.cpu().pin_memory()
        f = fb.linear_w8a16 if mode == 0 else fb.linear_w8a8
        ref.append(f(x, q, s))
        y = torch.full_like(ref[-1], 7.0)
        outs.append(y)
        jobs.append((mode, qh[:, :K], sh, x, y))
        slot = max(slot, fb.stream_slot_bytes(N, K, ldq))
        ws_need = max(ws_need, fb.workspace_size(mode, M, N, K))
    slot = -(-slot // 256) * 256
    slots = torch.empty(nslots * slot, dtype=torch.uint8, device=DEV)
    ws = torch.empty(max(1, ws_need), dtype=torch.uint8, device=DEV)
    compute, copy = torch.cuda.Stream(), torch.cuda.Stream()
    events = [torch.cuda.Event() for _ in range(2 * nslots)]
    compute.wait_stream(torch.cuda.current_stream())
    fb.streamed_linears(jobs, slots, slot, nslots, ws, compute, copy, events)
    torch.cuda.current_stream().wait_stream(compute)
    torch.cuda.synchronize()
    orefs = stream_oracle_refs(ws_cpu, xs_cpu)
    for (mode, M, K, N), r, y, (q, s), (q_o, s_o, y_o) in zip(STREAM_JOBS, ref, outs, codes, orefs):
        assert np.array_equal(u8(q), q_o), (mode, M, K, N)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))
        check_linear(bf16_to_f64(y), y_o, f"streamed/{mode}/{M}x{K}x{N}")
        assert torch.equal(y.view(torch.int16), r.view(torch.int16)), (mode, M, K, N)
    assert fb.read_device_error() == 0


# ----------------------------------------------------------- checkpoints
@pytest.mark.gpu
def test_checkpoint_conversion_matches_oracle(tmp_path):
    """BF16 checkpoint -> block-FP8 checkpoint on the GPU: every converted
    weight's codes and scales equal the oracle's, other tensors pass through,
    and a linear on the loaded weights equals one on the in-memory weights."""
    from block_scaled_fp8_fp8blk_b200 import checkpoint as ck
    g = torch.Generator(device="cpu").manual_seed(31)
    src = {
        "model.layers.0.self_attn.q_proj.weight": (torch.randn(384, 256, generator=g) * 0.02).to(torch.bfloat16),
        "model.layers.0.mlp.down_proj.weight": (torch.randn(300, 1000, generator=g) * 0.02).to(torch.bfloat16),
        "model.layers.0.input_layernorm.weight": torch.randn(256, generator=g).to(torch.bfloat16),
        "model.embed_tokens.weight": torch.randn(40, 256, generator=g).to(torch.bfloat16),
    }
    src_dir, dst_dir = str(tmp_path / "bf16"), str(tmp_path / "fp8")
    ck.save_checkpoint(src_dir, src, config={"model_type": "synthetic"})
    ck.convert_checkpoint(src_dir, dst_dir, max_shard_bytes=300_000)
    got, cfg = ck.load_checkpoint(dst_dir)
    assert cfg["quantization_config"]["weight_block_size"] == [128, 128]
    for name, w in src.items():
        if not ck.default_is_linear(name, w):
            assert torch.equal(got[name].view(torch.int16), w.view(torch.int16))
            assert name + "_scale_inv" not in got
            continue
        q_ref, s_ref = oracle.quantize_weight(w.view(torch.int16).numpy().view(np.uint16))
        assert np.array_equal(got[name].view(torch.uint8).numpy(), q_ref)
        assert np.array_equal(got[name + "_scale_inv"].numpy().view(np.uint32), s_ref.view(np.uint32))
    name = "model.layers.0.mlp.down_proj.weight"
    q, s = ck.linear_weights(got, name)
    x = torch.randn(64, 1008, generator=g).to(torch.bfloat16).to(DEV)[:, :1000]
    q_direct, s_direct = fb.quantize_weight(
        torch.nn.functional.pad(src[name], (0, 8)).to(DEV)[:, :1000])
    for f in (fb.linear_w8a16, fb.linear_w8a8):
        assert torch.equal(f(x, q, s).view(torch.int16), f(x, q_direct, s_direct).view(torch.int16))


# ------------------------------------------------------ failure detection
@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_stays_usable():
    """A wait that nothing completes gives up after its limit, reports through
    the device error word, and the context keeps working afterwards."""
    assert fb.read_device_error() == 0
    fb.selftest_wait_timeout(2_000_000)          # about a millisecond
    torch.cuda.synchronize()
    assert fb.read_device_error() == 16
    assert fb.read_device_error() == 0           # read-and-clear
    wl = W.RAGGED
    run_linear(wl, "w8a16")                       # still correct after the time-out
    assert fb.read_device_error() == 0


# ------------------------------------------------------- linear sequences
@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 64, 300])
def test_linear_sequence_matches_separate_calls(M):
    """A chain of linears (each x the previous y, modes mixed) launched as one
    sequence, weights streamed ahead of the previous kernel's end, gives
    exactly what separate calls give."""
    g = torch.Generator(device="cpu").manual_seed(41 + M)
    dims = [1024, 2048, 640, 1000, 1536]
    modes = [0, 1, 0, 0, 1, 0][:len(dims) - 1]
    weights = []
    for (K, N) in zip(dims[:-1], dims[1:]):
        ldw = -(-K // 8) * 8
        w = (torch.randn(N, ldw, generator=g) * 0.02).to(torch.bfloat16).to(DEV)[:, :K]
        weights.append(fb.quantize_weight(w))
    x0 = torch.randn(M, dims[0], generator=g).to(torch.bfloat16).to(DEV)
    # separate calls
    ref, h = [], x0
    for mode, (q, s) in zip(modes, weights):
        h = (fb.linear_w8a16 if mode == 0 else fb.linear_w8a8)(h, q, s)
        ref.append(h)
    # one sequence over fresh outputs
    outs, jobs, h = [], [], x0
    for mode, (q, s), r in zip(modes, weights, ref):
        y = torch.full_like(r, 3.0)
        jobs.append((mode, h, q, s, y))
        outs.append(y)
        h = y
    for _ in range(2):                                  # repeated: rings and workspace reused
        fb.linear_sequence(jobs)
        torch.cuda.synchronize()
        for r, y in zip(ref, outs):
            assert torch.equal(y.view(torch.int16), r.view(torch.int16))
    # each job against the oracle of its mode, on the x it read (the previous
    # job's BF16 output) and the weights it used
    h = x0
    for mode, (q, s), y, (K, N) in zip(modes, weights, outs, zip(dims[:-1], dims[1:])):
        xb = bf16_bits(h)
        q_h, s_h = u8(q), s.cpu().numpy()
        if mode == 0:
            want = oracle.linear_w8a16(xb, q_h, s_h, N, K)
        else:
            qx, sx = oracle.act_quant(xb)
            want = oracle.linear_w8a8(qx, sx, q_h, s_h, N, K)
        check_linear(bf16_to_f64(y), want, f"sequence/M{M}/{mode}/{K}x{N}")
        h = y
    assert fb.read_device_error() == 0


@pytest.mark.gpu
def test_sequence_and_streaming_edge_jobs():
    """Jobs with K = 0 (y = 0) and N = 0 (nothing) inside a sequence and a
    streamed run, between ordinary jobs."""
    g = torch.Generator(device="cpu").manual_seed(51)
    w = (torch.randn(384, 256, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    q, s = fb.quantize_weight(w)
    x = torch.randn(64, 256, generator=g).to(torch.bfloat16).to(DEV)
    ref = fb.linear_w8a16(x, q, s)
    x0 = torch.zeros((64, 0), dtype=torch.bfloat16, device=DEV)
    q0 = torch.zeros((384, 0), dtype=torch.uint8, device=DEV)
    s0 = torch.zeros((3, 1), dtype=torch.float32, device=DEV)
    qn = torch.zeros((0, 256), dtype=torch.uint8, device=DEV)
    sn = torch.zeros((1, 2), dtype=torch.float32, device=DEV)
    # sequence
    y1, y2 = torch.full_like(ref, 5.0), torch.full_like(ref, 5.0)
    yk0 = torch.full_like(ref, 5.0)
    yn0 = torch.empty((64, 0), dtype=torch.bfloat16, device=DEV)
    fb.linear_sequence([(0, x, q, s, y1), (1, x0, q0, s0, yk0), (0, x, qn, sn, yn0), (0, x, q, s, y2)])
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(y2.view(torch.int16), ref.view(torch.int16))
    assert torch.all(yk0 == 0)
    # streaming (host weights; the K = 0 job copies nothing)
    qh = torch.empty(q.shape, dtype=torch.uint8, pin_memory=True)
    qh.copy_(q)
    sh = s.cpu().pin_memory()
    q0h = torch.empty((384, 0), dtype=torch.uint8, pin_memory=True)
    s0h = torch.zeros((3, 1), dtype=torch.float32).pin_memory()
    y3, y4 = torch.full_like(ref, 5.0), torch.full_like(ref, 5.0)
    yk1 = torch.full_like(ref, 5.0)
    slot = -(-fb.stream_slot_bytes(384, 256, 256) // 256) * 256
    slots = torch.empty(2 * slot, dtype=torch.uint8, device=DEV)
    ws = torch.empty(fb.workspace_size(0, 64, 384, 256), dtype=torch.uint8, device=DEV)
    compute, copy = torch.cuda.Stream(), torch.cuda.Stream()
    events = [torch.cuda.Event() for _ in range(4)]
    compute.wait_stream(torch.cuda.current_stream())
    fb.streamed_linears([(0, qh, sh, x, y3), (0, q0h, s0h, x0, yk1), (0, qh, sh, x, y4)],
                        slots, slot, 2, ws, compute, copy, events)
    torch.cuda.current_stream().wait_stream(compute)
    torch.cuda.synchronize()
    assert torch.equal(y3.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(y4.view(torch.int16), ref.view(torch.int16))
    assert torch.all(yk1 == 0)
    assert fb.read_device_error() == 0
