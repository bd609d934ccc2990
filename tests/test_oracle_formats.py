"""Pins for the oracle's number formats and its 16-element block quantizer.

The E2M1 and E4M3 encoders are pinned to hand-derived tables (tests/golden/) and, for
E4M3, to torch's own float8_e4m3fn conversion; the block rule is pinned by closed forms
(exactly representable blocks round-trip, zero blocks, saturation, scale rounding).
"""
import math
import struct

import numpy as np
import pytest
import torch

from conftest import read_golden


def _hexf(s: str) -> float:
    if s in ("inf", "-inf"):
        return float(s)
    return float.fromhex(s)


def test_e2m1_decode_matches_golden(oracle_mod):
    rows = read_golden("e2m1_values.txt")
    codes = np.array([int(c, 16) for c, _ in rows], np.uint8)
    want = np.array([float(v) for _, v in rows])
    got = oracle_mod.e2m1_decode(codes)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_e2m1_encode_matches_golden(oracle_mod):
    rows = read_golden("e2m1_rne.txt")
    x = np.array([_hexf(a) for a, _ in rows], np.float32)
    want = np.array([int(c, 16) for _, c in rows], np.uint8)
    got = oracle_mod.e2m1_encode(x)
    bad = [(rows[i][0], hex(got[i]), rows[i][1]) for i in np.nonzero(got != want)[0]]
    assert not bad, bad


def test_e2m1_encode_is_nearest_and_monotone(oracle_mod):
    # Dense sweep of binary32 values in [0, 8): every result is a nearest representable
    # magnitude, and the code sequence never decreases.
    x = np.linspace(0.0, 8.0, 200001, dtype=np.float32)
    c = oracle_mod.e2m1_encode(x)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    dist = np.abs(x.astype(np.float64)[:, None] - mags[None, :])
    got = np.abs(x - oracle_mod.e2m1_decode(c))
    assert np.all(got <= dist.min(axis=1) + 0.0)
    assert np.all(np.diff(c.astype(np.int32)) >= 0)
    # odd symmetry: encode(-x) = encode(x) | 8
    assert np.array_equal(oracle_mod.e2m1_encode(-x[1:]), c[1:] | 8)


def test_e4m3_decode_matches_torch(oracle_mod):
    b = np.arange(256, dtype=np.uint8)
    got = oracle_mod.e4m3_decode(b)
    want = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and got[0x7E] == 448.0


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    # All midpoints between neighbouring finite codes, their binary32 neighbours, the
    # codes themselves and a random sample, up to 464 where torch stops rounding to 448.
    vals = oracle_mod.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    pts = np.concatenate([vals, mids]).astype(np.float32)
    pts = np.concatenate([pts, np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    rng = np.random.default_rng(0)
    pts = np.concatenate([pts, rng.uniform(0, 464, 100000).astype(np.float32),
                          np.exp2(rng.uniform(-14, 8.8, 100000)).astype(np.float32)])
    pts = pts[(pts >= 0) & (pts <= 464)]
    pts = np.concatenate([pts, -pts])
    got = oracle_mod.e4m3_encode(pts)
    want = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(pts[i]), hex(got[i]), hex(want[i])) for i in bad[:10]]


def test_e4m3_encode_matches_golden_and_saturates(oracle_mod):
    rows = read_golden("e4m3_rne.txt")
    x = np.array([_hexf(a) for a, _ in rows], np.float32)
    want = np.array([int(c, 16) for _, c in rows], np.uint8)
    got = oracle_mod.e4m3_encode(x)
    bad = [(rows[i][0], hex(got[i]), rows[i][1]) for i in np.nonzero(got != want)[0]]
    assert not bad, bad
    big = np.array([465, 1000, 3e38, np.inf], np.float32)
    assert np.all(oracle_mod.e4m3_encode(big) == 0x7E)


def _exact_block(rng, scale_byte):
    codes = rng.integers(0, 16, 16).astype(np.uint8)
    codes[rng.integers(0, 16)] = 7 | (8 * rng.integers(0, 2))  # absmax = 6 * s
    return codes


def test_block_roundtrip_of_representable_values(oracle_mod):
    # x_i = e2m1(c_i) * s with max |c| = 6 and s an E4M3 value: a = 6s, a/6 = s exactly,
    # and x_i / s = e2m1(c_i) exactly, so the codes and the scale byte come back.
    rng = np.random.default_rng(1)
    dec = oracle_mod.e2m1_decode(np.arange(16, dtype=np.uint8))
    for sb in list(range(1, 0x7F)):
        s = oracle_mod.e4m3_decode(np.array([sb], np.uint8))[0]
        codes = _exact_block(rng, sb)
        x = (dec[codes] * s).astype(np.float32)
        assert np.array_equal(x.astype(np.float64), dec[codes] * s)  # exact in binary32
        c, b = oracle_mod.quant_block16(x[None, :])
        assert b[0] == sb
        # -0 and +0 both decode to 0: compare values, and signs for the non-zeros
        assert np.array_equal(dec[c[0]], dec[codes])


def test_block_zero_tiny_and_saturating(oracle_mod):
    c, b = oracle_mod.quant_block16(np.zeros((1, 16), np.float32))
    assert b[0] == 0 and not c.any()
    # absmax / 6 at most half the smallest subnormal scale (2^-10): scale byte 0, codes 0
    x = np.full((1, 16), 6 * 2.0 ** -10, np.float32)
    c, b = oracle_mod.quant_block16(x)
    assert b[0] == 0 and not c.any()
    # absmax > 2688 = 448 * 6: the scale saturates at 448 and the largest element at 6
    x = np.zeros((1, 16), np.float32)
    x[0, 3] = 5000.0
    x[0, 5] = -448.0
    c, b = oracle_mod.quant_block16(x)
    assert b[0] == 0x7E and c[0, 3] == 0x7 and c[0, 5] == 0xA  # -448/448 = -1 -> 0xA


def test_block_scale_rounds_down_then_element_saturates(oracle_mod):
    # a = 6.375: a/6 = 1.0625 is a tie between E4M3 1.0 and 1.125 -> 1.0 (even);
    # 6.375 / 1.0 = 6.375 rounds (saturating) to 6 -> code 7; 3.25/1 -> 3 (code 5).
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.375
    x[0, 1] = 3.25
    x[0, 2] = -0.2
    c, b = oracle_mod.quant_block16(x)
    assert b[0] == 0x38
    assert c[0, 0] == 7 and c[0, 1] == 5 and c[0, 2] == 0x8


def test_block_element_division_is_binary32(oracle_mod):
    # scale s = 1.125 (absmax 6.75): 0.84375 / 1.125 = 0.75 exactly -> tie -> 1.0 (code 2);
    # the element just below gives a quotient below 0.75 -> 0.5 (code 1).
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.75
    x[0, 1] = 0.84375
    x[0, 2] = np.nextafter(np.float32(0.84375), np.float32(0))
    c, b = oracle_mod.quant_block16(x)
    assert b[0] == 0x39
    assert c[0, 1] == 2 and c[0, 2] == 1
