"""Pins of the oracle's converter, dequantizer, activation quantizer and the two
FP64 linears against independent routes: a hand-worked example, torch's
float32 division / float8 cast / bfloat16 cast (the scale broadcast over each
block that FastVideo PR #1829, section "Changes", tests bullet, checks against), numpy float64 matmul on
small shapes, closed forms (one-hot rows, constant blocks, zero blocks) and
the format's invariants (the largest code of a block is 448)."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_fp8_fp8blk_b200 import synth
from block_scaled_fp8_fp8blk_b200.workloads import RAGGED, TINY, Workload
from conftest import read_golden
from helpers import e4m3_midpoints, tie_heavy_weight

TORCH_E4M3 = torch.float8_e4m3fn


def bf16_from_f32(a):
    return synth.bf16_bits(synth.to_bf16(a))


def f32_from_bf16(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def decode(q):
    return torch.from_numpy(np.ascontiguousarray(q)).view(TORCH_E4M3).to(torch.float64).numpy()


def broadcast(s, rows, cols, g_rows=128, g_cols=128):
    return np.repeat(np.repeat(s, g_rows, axis=0), g_cols, axis=1)[:rows, :cols]


def torch_codes(v_f32):
    return torch.from_numpy(np.ascontiguousarray(v_f32)).to(TORCH_E4M3).view(torch.uint8).numpy()


def block_amax(wf, N, K):
    NB, KB = -(-N // 128), -(-K // 128)
    a = np.zeros((NB, KB), np.float32)
    for i in range(NB):
        for j in range(KB):
            a[i, j] = np.abs(wf[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]).max()
    return a


@pytest.fixture(scope="module", params=[TINY, RAGGED], ids=lambda w: w.name)
def wl(request):
    return request.param


@pytest.fixture(scope="module")
def weights(wl):
    wb = bf16_from_f32(synth.weight_f32(wl.seed, wl.N, wl.K, wl.row_gain_sigma))
    q, s = oracle.quantize_weight(wb)
    return wb, q, s


def test_worked_example():
    rows = read_golden("quantize_worked_example.txt")
    data = [r for r in rows if r[0] != "scale_inv"]
    s_bits = int([r for r in rows if r[0] == "scale_inv"][0][1], 16)
    w = np.array([[float(r[0]) for r in data]], dtype=np.float32)
    q, s = oracle.quantize_weight(bf16_from_f32(w))
    assert s.shape == (1, 1) and s.view(np.uint32)[0, 0] == s_bits
    assert [int(c) for c in q[0]] == [int(r[1], 16) for r in data]
    d = f32_from_bf16(oracle.dequantize(q, s))
    assert list(d[0]) == [float(r[2]) for r in data]


def test_scale_is_amax_over_448(wl, weights):
    wb, q, s = weights
    amax = block_amax(f32_from_bf16(wb), wl.N, wl.K)
    assert s.shape == (-(-wl.N // 128), -(-wl.K // 128))
    assert np.array_equal(s, amax / np.float32(448.0))
    if wl.row_gain_sigma:
        assert s.max() / s.min() > 2  # row gains make blocks differ (catches index swaps)


def test_codes_match_torch_division_and_cast(wl, weights):
    wb, q, s = weights
    wf = f32_from_bf16(wb)
    sb = broadcast(s, wl.N, wl.K)
    ratio = (torch.from_numpy(wf) / torch.from_numpy(np.ascontiguousarray(sb))).numpy()
    assert np.abs(ratio).max() < 464
    assert np.array_equal(q, torch_codes(ratio))


def test_tie_heavy_blocks_round_to_even():
    """Quotients exactly on E4M3 decision points, whole blocks of them and a
    few per warp's rows, with ragged edges: the codes equal torch's float32
    division and float8 cast, and every tie took the even code."""
    wb = tie_heavy_weight()
    q, s = oracle.quantize_weight(wb)
    N, K = wb.shape
    wf = f32_from_bf16(wb)
    assert np.array_equal(s, block_amax(wf, N, K) / np.float32(448.0))
    sb = broadcast(s, N, K)
    ratio = (torch.from_numpy(wf) / torch.from_numpy(np.ascontiguousarray(sb))).numpy()
    assert np.array_equal(q, torch_codes(ratio))
    mids = set(e4m3_midpoints(464.0).tolist())
    tie = np.vectorize(lambda r: abs(float(r)) in mids)(ratio)
    assert tie.sum() > 20000                      # the blocks really are tie-heavy
    assert np.all((q[tie] & 1) == 0)              # ties to even: the code's last bit is 0


def test_block_max_code_is_448(wl, weights):
    wb, q, s = weights
    mag = np.abs(decode(q))
    for i in range(s.shape[0]):
        for j in range(s.shape[1]):
            assert mag[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128].max() == 448.0


def test_roundtrip_within_e4m3_precision(wl, weights):
    # FastVideo PR #1829, "Changes", tests bullet: the FP8 round trip is held
    # to the precision of E4M3: relative 2^-4 for normals, absolute 2^-10 * s for
    # subnormals, plus the final BF16 rounding (2^-9 relative).
    wb, q, s = weights
    wf = f32_from_bf16(wb).astype(np.float64)
    d = f32_from_bf16(oracle.dequantize(q, s)).astype(np.float64)
    sb = broadcast(s, wl.N, wl.K).astype(np.float64)
    bound = (2.0 ** -4 * np.abs(wf) + 2.0 ** -10 * sb) * (1 + 2.0 ** -8) + 2.0 ** -9 * np.abs(wf)
    assert np.all(np.abs(d - wf) <= bound)


def test_block_argmax_survives_roundtrip(wl, weights):
    wb, q, s = weights
    d = oracle.dequantize(q, s)
    wf = np.abs(f32_from_bf16(wb))
    for i in range(s.shape[0]):
        for j in range(s.shape[1]):
            blk = wf[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            r, c = np.unravel_index(np.argmax(blk), blk.shape)
            assert d[i * 128 + r, j * 128 + c] == wb[i * 128 + r, j * 128 + c]


def test_dequantize_is_reference_broadcast(wl, weights):
    wb, q, s = weights
    sb = torch.from_numpy(np.ascontiguousarray(broadcast(s, wl.N, wl.K)))
    codes = torch.from_numpy(q).view(TORCH_E4M3).to(torch.float32)
    ref = (codes * sb).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.dequantize(q, s), ref)


def test_dequantize_all_codes_many_scales():
    rng = np.random.default_rng(4)
    scales = np.concatenate([[0.0, 1.0, 2.0 ** -20, 3.0e-5], rng.random(60) * 10.0 ** rng.integers(-8, 3, 60)])
    scales = scales.astype(np.float32)
    codes = np.tile(np.arange(256, dtype=np.uint8), (128, 1))
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0
    for sv in scales:
        s = np.full((1, 2), sv, dtype=np.float32)
        got = oracle.dequantize(codes, s)
        ref = (torch.from_numpy(codes).view(TORCH_E4M3).to(torch.float32) * float(sv)).to(
            torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, ref)


def test_ragged_padding_is_ignored():
    N, K, ldw = 200, 300, 320
    wf = synth.weight_f32(5, N, K)
    wb = bf16_from_f32(wf)
    padded = np.full((N, ldw), bf16_from_f32(np.array([3.0e4], np.float32))[0], dtype=np.uint16)
    padded[:, :K] = wb
    q1, s1 = oracle.quantize_weight(wb)
    q2, s2 = oracle.quantize_weight(padded, K=K, ldq=336)
    assert np.array_equal(s1, s2) and s1.shape == (2, 3)
    assert np.array_equal(q1, q2[:, :K])
    assert np.array_equal(oracle.dequantize(q1, s1), oracle.dequantize(q2, s2, K=K))


def test_zero_block_and_signed_zero():
    w = np.zeros((130, 260), dtype=np.float32)
    w[0, 0] = -0.0
    w[129, 259] = 1.5
    w[129, 258] = -1e-30   # underflows to a negative zero code
    q, s = oracle.quantize_weight(bf16_from_f32(w))
    assert s[0, 0] == 0 and s[0, 1] == 0 and s[1, 2] == np.float32(1.5) / np.float32(448)
    assert q[0, 0] == 0x80 and q[0, 1] == 0x00 and q[129, 259] == 0x7E and q[129, 258] == 0x80
    d = oracle.dequantize(q, s)
    assert d[0, 0] == 0x8000 and d[0, 1] == 0


def test_every_bf16_value_as_a_code():
    # Blocks holding every finite BF16 value up to a block maximum A: codes
    # equal torch's cast of the float32 quotient w / (A / 448).
    allb = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = f32_from_bf16(allb)
    for A in (1.0, 0.02, 448.0, 3.3e-20):
        A = f32_from_bf16(bf16_from_f32(np.array([A], np.float32)))[0]  # a BF16 value
        v = vals[np.isfinite(vals) & (np.abs(vals) <= A)]
        n = -(-v.size // 128) * 128
        w = np.zeros(n, np.float32)
        w[:v.size] = v
        w[-1] = A  # ensure the block amax is exactly A in every block
        w = w.reshape(-1, 128)
        w[:, 0] = A
        wb = bf16_from_f32(w)
        q, s = oracle.quantize_weight(wb)
        sv = A / np.float32(448.0)
        assert np.all(s == sv)
        ref = torch_codes((torch.from_numpy(f32_from_bf16(wb)) / torch.tensor(sv)).numpy())
        assert np.array_equal(q, ref)


# ------------------------------------------------------------ activations
def test_act_quant_groups(wl):
    xb = bf16_from_f32(synth.activation_f32(wl.seed, wl.M, wl.K, 0.01))
    qx, sx = oracle.act_quant(xb)
    xf = f32_from_bf16(xb)
    KB = -(-wl.K // 128)
    amax = np.stack([np.abs(xf[:, j * 128:(j + 1) * 128]).max(axis=1) for j in range(KB)], axis=1)
    assert sx.shape == (wl.M, KB)
    assert np.array_equal(sx, amax / np.float32(448.0))
    ratio = (torch.from_numpy(xf) / torch.from_numpy(np.ascontiguousarray(broadcast(sx, wl.M, wl.K, 1, 128)))).numpy()
    assert np.array_equal(qx, torch_codes(ratio))


# ------------------------------------------------------------ linears
def dequant_f64(q, s, N, K):
    return decode(q[:, :K]) * broadcast(s, N, K).astype(np.float64)


def test_linear_w8a16_matches_numpy(wl, weights):
    wb, q, s = weights
    xb = bf16_from_f32(synth.activation_f32(wl.seed, wl.M, wl.K, wl.outlier_frac))
    ref = oracle.linear_w8a16(xb, q, s, wl.N, wl.K)
    want = f32_from_bf16(xb).astype(np.float64) @ dequant_f64(q, s, wl.N, wl.K).T
    assert ref.shape == (wl.M, wl.N)
    assert np.max(np.abs(ref - want)) <= 1e-12 * np.max(np.abs(want))
    rows = np.array([wl.M - 1, 0, 3], dtype=np.int64)
    assert np.array_equal(oracle.linear_w8a16(xb, q, s, wl.N, wl.K, rows=rows), ref[rows])


def test_linear_w8a8_matches_numpy(wl, weights):
    wb, q, s = weights
    xb = bf16_from_f32(synth.activation_f32(wl.seed, wl.M, wl.K, wl.outlier_frac))
    qx, sx = oracle.act_quant(xb)
    ref = oracle.linear_w8a8(qx, sx, q, s, wl.N, wl.K)
    a = decode(qx) * broadcast(sx, wl.M, wl.K, 1, 128).astype(np.float64)
    want = a @ dequant_f64(q, s, wl.N, wl.K).T
    assert np.max(np.abs(ref - want)) <= 1e-12 * np.max(np.abs(want))
    # and W8A8 stays close to W8A16 (activation quantization error only)
    r16 = oracle.linear_w8a16(xb, q, s, wl.N, wl.K)
    assert np.linalg.norm(ref - r16) / np.linalg.norm(r16) < 0.06


def test_linear_one_hot_rows_give_dequantized_weights(weights, wl):
    wb, q, s = weights
    ks = np.array([0, 1, 127, 128, wl.K - 1])
    x = np.zeros((ks.size, wl.K), np.float32)
    x[np.arange(ks.size), ks] = 1.0
    ref = oracle.linear_w8a16(bf16_from_f32(x), q, s, wl.N, wl.K)
    T = oracle.e4m3_table()
    for i, k in enumerate(ks):
        col = T[q[:, k]] * s[np.arange(wl.N) // 128, k // 128].astype(np.float64)
        assert np.array_equal(ref[i], col)


def test_linear_constant_block_closed_form():
    N, K, M = 256, 384, 3
    w = np.zeros((N, K), np.float32)
    c = np.float32(0.0625)
    w[128:256, 128:256] = c              # block (1, 1) constant -> codes 448, s = c/448
    w[0:128, 256:384] = -c                # block (0, 2) constant negative
    xb = bf16_from_f32(synth.activation_f32(9, M, K))
    xf = f32_from_bf16(xb).astype(np.float64)
    q, s = oracle.quantize_weight(bf16_from_f32(w))
    assert np.all(q[128:256, 128:256] == 0x7E) and np.all(q[0:128, 256:384] == 0xFE)
    ref = oracle.linear_w8a16(xb, q, s, N, K)
    sv = float(np.float32(c) / np.float32(448))
    want_hi = 448.0 * sv * xf[:, 128:256].sum(axis=1)
    want_lo = -448.0 * sv * xf[:, 256:384].sum(axis=1)
    assert np.allclose(ref[:, 128:256], want_hi[:, None], rtol=1e-13, atol=0)
    assert np.allclose(ref[:, 0:128], want_lo[:, None], rtol=1e-13, atol=0)


def test_all_zero_weight_gives_zero():
    N, K, M = 128, 256, 2
    q, s = oracle.quantize_weight(np.zeros((N, K), np.uint16))
    xb = bf16_from_f32(synth.activation_f32(1, M, K))
    assert np.all(oracle.linear_w8a16(xb, q, s, N, K) == 0)
    qx, sx = oracle.act_quant(xb)
    assert np.all(oracle.linear_w8a8(qx, sx, q, s, N, K) == 0)


def test_planted_mistake_is_caught():
    # A transposed scale grid (a plausible indexing slip) must break the
    # numpy cross-check on a non-square block grid.
    wl = Workload("t", 5, 256, 384, row_gain_sigma=0.5)
    wb = bf16_from_f32(synth.weight_f32(0, wl.N, wl.K, 0.5))
    q, s = oracle.quantize_weight(wb)
    xb = bf16_from_f32(synth.activation_f32(0, wl.M, wl.K))
    wrong = np.ascontiguousarray(np.resize(s.T.copy(), s.shape))
    good = oracle.linear_w8a16(xb, q, s, wl.N, wl.K)
    bad = oracle.linear_w8a16(xb, q, wrong, wl.N, wl.K)
    assert np.linalg.norm(bad - good) / np.linalg.norm(good) > 0.05
