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
