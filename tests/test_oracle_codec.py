"""Pins for the oracle's scalar codecs (bf16 rounding, OCP E4M3).

The pages name FP8 e4m3 and bf16 outputs but print no codec, so the oracle's
codec is pinned against (a) closed-form code points from the published OCP
E4M3 definition (tests/golden/e4m3_codes.txt), (b) an independent library
routine (torch's CPU float8_e4m3fn / bfloat16 conversions) and (c) structural
invariants (round trip, ties to even, saturation).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _torch_e4m3_code(v: float) -> int:
    return int(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def test_e4m3_golden_code_points():
    n = 0
    with open(os.path.join(GOLDEN, "e4m3_codes.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            code_s, val_s = line.split()[:2]
            code = int(code_s, 16)
            got = oracle.e4m3_decode(code)
            if val_s == "nan":
                assert math.isnan(got)
                continue
            want = float(val_s)
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (code_s, got, want)
            assert oracle.e4m3_encode(want) == code, code_s
            n += 1
    assert n >= 15


def test_e4m3_decode_all_codes_match_library():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if math.isnan(lib[c]):
            assert math.isnan(got) and (c & 0x7F) == 0x7F
        else:
            assert got == lib[c] and math.copysign(1, got) == math.copysign(1, lib[c]), c


def test_e4m3_units_are_value_times_512():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_units(c) == oracle.e4m3_decode(c) * 512.0


def test_e4m3_round_trip_every_finite_code():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def test_e4m3_ties_go_to_even_code():
    # every midpoint between adjacent finite codes, both signs
    for c in range(0, 0x7E):
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        mid = (lo + hi) / 2.0  # exact in binary32: both have <= 4 significant bits
        assert np.float32(mid) == mid
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even, (hex(c), mid)
        assert oracle.e4m3_encode(-mid) == (even | 0x80) if mid != 0 else True
        # just off the midpoint goes to the nearer code
        below = float(np.nextafter(np.float32(mid), np.float32(-1)))
        above = float(np.nextafter(np.float32(mid), np.float32(1000)))
        assert oracle.e4m3_encode(below) == c
        assert oracle.e4m3_encode(above) == c + 1


def test_e4m3_saturates_at_448():
    for v in (448.0, 449.0, 463.99, 464.0, 480.0, 500.0, 1e6, 3e38):
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE


def test_e4m3_sign_of_zero_kept():
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-9) == 0x80
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00  # exact tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(-(2.0 ** -10)) == 0x80


def test_e4m3_encode_matches_library_on_every_bf16_value():
    # all finite bf16 values below the library's NaN threshold (464)
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    f = ((bits << 16).view(np.float32))
    f = f[np.isfinite(f) & (np.abs(f) < 464.0)]
    lib = torch.from_numpy(f.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    enc = np.array([oracle.e4m3_encode(float(v)) for v in f], dtype=np.uint8)
    assert np.array_equal(enc, lib)


def test_e4m3_encode_matches_library_on_random_floats():
    g = np.random.default_rng(7)
    v = (g.standard_normal(20000) * np.exp(g.uniform(-12, 6, 20000))).astype(np.float32)
    v = v[np.abs(v) < 464.0]
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    enc = np.array([oracle.e4m3_encode(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(enc, lib)


def test_e4m3_normal_relative_error_bound():
    g = np.random.default_rng(3)
    v = g.uniform(2.0 ** -6, 448.0, 5000).astype(np.float32)
    for x in v:
        d = oracle.e4m3_decode(oracle.e4m3_encode(float(x)))
        assert abs(d - x) <= 2.0 ** -4 * abs(x)


def test_bf16_rounding_matches_library():
    g = np.random.default_rng(11)
    f = np.concatenate([
        g.standard_normal(20000).astype(np.float32) * np.float32(1e3),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.0e38, 1e-40, 65504.0], np.float32),
    ])
    lib = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(x)) for x in f], dtype=np.uint16)
    assert np.array_equal(got, lib)


def test_bf16_widening_exact():
    for b in (0x0000, 0x8000, 0x3F80, 0xBF80, 0x7F7F, 0x0001, 0x4049):
        want = float(np.array([b << 16], dtype=np.uint32).view(np.float32)[0])
        assert oracle.bf16_to_f32(b) == want


@pytest.mark.parametrize("b", [0x3F80, 0x3F81, 0x4000])
def test_bf16_ties_to_even(b):
    # exact midpoint above b: ties go to the even pattern
    lo = oracle.bf16_to_f32(b)
    hi = oracle.bf16_to_f32(b + 1)
    mid = (lo + hi) / 2
    assert oracle.f32_to_bf16(mid) == (b if b % 2 == 0 else b + 1)
