"""Pins of the oracle's E4M3 and BF16 codecs against things other than itself:
the OCP OFP8 specification's values, torch's own float8/bfloat16 casts, an
independent bit-level encoder over every float bit pattern, and closed-form
tie/saturation/underflow cases."""
import math
import struct

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def f32(bits):
    return struct.unpack("<f", struct.pack("<I", bits))[0]


def bits32(x):
    return struct.unpack("<I", struct.pack("<f", x))[0]


def test_spec_values():
    T = oracle.e4m3_table()
    rows = read_golden("e4m3_ocp_values.txt")
    assert len(rows) == 10
    for code_s, val_s in rows:
        code, val = int(code_s, 16), float(val_s)
        if math.isnan(val):
            assert math.isnan(T[code])
        else:
            assert T[code] == val and math.copysign(1, T[code]) == math.copysign(1, val)


def test_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    T = oracle.e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(T))
    assert nan.sum() == 2
    assert np.array_equal(ref[~nan], T[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(T[~nan]))


def test_roundtrip_all_codes():
    T = oracle.e4m3_table()
    for c in range(256):
        if math.isnan(T[c]):
            continue
        assert oracle.e4m3_encode(np.float32(T[c]))[()] == c, hex(c)


def test_midpoints_round_to_even_code():
    T = oracle.e4m3_table()
    vals, want = [], []
    for c in range(0x7E):
        lo, hi = T[c], T[c + 1]
        mid = (lo + hi) / 2
        assert np.float32(mid) == mid  # midpoints need <= 5 significant bits
        even = c if c % 2 == 0 else c + 1
        up = np.nextafter(np.float32(mid), np.float32(np.inf))
        dn = np.nextafter(np.float32(mid), np.float32(-np.inf))
        vals += [mid, up, dn, -mid, -up, -dn]
        want += [even, c + 1, c, even | 0x80, (c + 1) | 0x80, c | 0x80]
    got = oracle.e4m3_encode(np.array(vals, dtype=np.float32))
    assert np.array_equal(got, np.array(want, dtype=np.uint8))


def test_saturation_and_underflow():
    big = [448.0, 448.0001, 463.9, 464.0, 480.0, 1e30, np.inf]
    got = oracle.e4m3_encode(np.array(big + [-v for v in big], dtype=np.float32))
    assert list(got) == [0x7E] * len(big) + [0xFE] * len(big)
    tiny = np.float32(2.0 ** -10)
    vals = np.array([tiny, -tiny, np.nextafter(tiny, np.float32(1)), 1e-30, -1e-30, 0.0, -0.0,
                     f32(1), f32(0x80000001)], dtype=np.float32)
    got = oracle.e4m3_encode(vals)
    assert list(got) == [0x00, 0x80, 0x01, 0x00, 0x80, 0x00, 0x80, 0x00, 0x80]
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_search_encoder_matches_torch_in_range():
    rng = np.random.default_rng(1)
    # every BF16 magnitude below 464 (a dense slice of the float grid) ...
    b = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    v = b.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) < 464)]
    # ... and random float32 values spread over all binades of the range
    r = (rng.standard_normal(2_000_000) * np.exp2(rng.integers(-14, 9, 2_000_000))).astype(np.float32)
    r = r[np.abs(r) < 464]
    v = np.concatenate([v, r])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


@pytest.mark.slow
def test_two_encoders_agree_on_every_float():
    # table search vs bit fields, all 2^32 float32 bit patterns (NaNs -> 0x7F)
    assert oracle.crosscheck_encoders(0, 1 << 32) == 0


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(2)
    u = rng.integers(0, 1 << 32, 4_000_000, dtype=np.uint64).astype(np.uint32)
    # add exact ties (low half == 0x8000) with both parities, and specials
    ties = (rng.integers(0, 1 << 16, 100_000, dtype=np.uint32) << 16) | 0x8000
    special = np.array([0, 0x80000000, 0x7F7FFFFF, 0x7F800000, 0xFF800000, 0x3F808000,
                        0x3F818000, 0x7F7F8000, 1], dtype=np.uint32)
    u = np.concatenate([u, ties, special])
    v = u.view(np.float32)
    v = v[~np.isnan(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_rne(v), ref)


def test_bf16_rne_is_nearest_ties_even():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(200_000) * np.exp2(rng.integers(-100, 100, 200_000))).astype(np.float32)
    out = oracle.bf16_rne(v).astype(np.uint32) << 16
    r = out.view(np.float32).astype(np.float64)
    lo = (v.view(np.uint32) & 0xFFFF0000).view(np.float32).astype(np.float64)  # truncation
    hi = ((v.view(np.uint32) & 0xFFFF0000) + 0x10000).view(np.float32).astype(np.float64)
    x = v.astype(np.float64)
    assert np.all((r == lo) | (r == hi))
    d_r, d_o = np.abs(r - x), np.minimum(np.abs(lo - x), np.abs(hi - x))
    assert np.all(d_r == d_o)
    tie = np.abs(lo - x) == np.abs(hi - x)
    assert np.all(((out[tie] >> 16) & 1) == 0)


# ------------------------------------------- the two whole-range checkers
# Both checkers return a count that the exhaustive tests require to be 0. A
# count that came out 0 for a wrong reason (a chunk skipped, a loop bound off
# by one, threads that never ran) would turn those tests into no-ops, so the
# counts themselves are pinned here: a planted error is counted exactly once
# wherever it sits (first or last pattern, either side of a chunk boundary,
# in a short last chunk) and with any number of threads.
CHUNK = 1 << 20


def _planted_positions(n):
    return sorted({0, 1, CHUNK - 1, CHUNK, CHUNK + 1, 2 * CHUNK - 1, 2 * CHUNK, n // 2, n - 2, n - 1})


def test_code_mismatch_count_against_torch_codes_and_planted_errors():
    lo = 0x3E000000 - 3                          # floats just below and above 0.125
    n = 2 * CHUNK + 123                           # three chunks, the last one short
    v = (np.arange(n, dtype=np.uint64) + lo).astype(np.uint32).view(np.float32)
    assert np.all(np.abs(v) < 448)                # torch's cast saturates nothing here
    codes = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    for nthreads in (1, 3, 16):
        assert oracle.count_code_mismatches(lo, codes, nthreads) == 0
    for pos in _planted_positions(n):
        bad = codes.copy()
        bad[pos] ^= 0x01
        for nthreads in (1, 3, 16):
            assert oracle.count_code_mismatches(lo, bad, nthreads) == 1, (pos, nthreads)
    bad = codes.copy()
    planted = _planted_positions(n)
    bad[planted] ^= 0x40
    assert oracle.count_code_mismatches(lo, bad) == len(planted)
    # a code array shifted by one pattern disagrees wherever neighbours differ
    shifted = np.roll(codes, 1)
    want = int(np.count_nonzero(shifted != codes))
    assert want > 0 and oracle.count_code_mismatches(lo, shifted) == want


def test_bit_field_encoder_matches_torch_on_a_range():
    # the encoder the device codec is counted against, checked against torch's
    # cast on every pattern of a range that crosses the E4M3 subnormal/normal
    # boundary (2^-6) and a few binades of normals
    lo, hi = 0x3C000000, 0x3C000000 + (1 << 24)  # 2^-7 up to 2^-5
    v = np.arange(lo, hi, 37, dtype=np.uint64).astype(np.uint32).view(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode_fields(float(f)) for f in v[::64]], dtype=np.uint8)
    assert np.array_equal(got, ref[::64])


def test_encoder_crosscheck_counts_a_planted_disagreement():
    lo = 0x43D00000 - 5                          # around 416 .. saturation
    hi = lo + 2 * CHUNK + 77
    assert oracle.crosscheck_encoders(lo, hi) == 0
    for off in _planted_positions(hi - lo):
        for nthreads in (1, 4, 16):
            assert oracle.crosscheck_encoders_planted(lo, hi, lo + off, nthreads) == 1, (off, nthreads)
    # a plant outside the range is not counted
    assert oracle.crosscheck_encoders_planted(lo, hi, lo - 1, 4) == 0
    assert oracle.crosscheck_encoders_planted(lo, hi, hi, 4) == 0
    # the top of the 32-bit range (the last chunk ends at 2^32 exactly)
    top = (1 << 32) - CHUNK - 9
    assert oracle.crosscheck_encoders_planted(top, 1 << 32, (1 << 32) - 1, 8) == 1
    assert oracle.crosscheck_encoders_planted(top, 1 << 32, top, 8) == 1


def test_encoder_crosscheck_equals_a_count_one_pattern_at_a_time():
    # brute force over a small range: the count equals the number of patterns
    # where the two single-value encoders differ (here none, and the planted one)
    lo, hi = 0x3A7FFFF0, 0x3A800010              # around 2^-10, where codes underflow to 0
    diffs = 0
    for u in range(lo, hi):
        f = f32(u)
        diffs += int(oracle.e4m3_encode(np.array([f], np.float32))[0] != oracle.e4m3_encode_fields(f))
    assert diffs == 0
    assert oracle.crosscheck_encoders(lo, hi, 1) == diffs
    assert oracle.crosscheck_encoders_planted(lo, hi, lo + 7, 1) == diffs + 1
