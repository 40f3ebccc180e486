"""Pins for the oracle's dynamic quantisers (per-token INT8/FP8, Block-FP8).

Definitions (plainest reading of the formats named in "Helion in vLLM: A
Unified Route to Tunable Linear Kernels", section "What the integration
changes"): s = amax / Qmax as a correctly rounded binary32 division, q = the
correctly rounded quotient x / s rounded to the target grid (INT8: half-even,
clamp +-127; FP8: clamp +-448 then nearest e4m3, ties to even), amax = 0 gives
s = 0 and q = +0.

Pins: hand-worked rows (tests/golden/quant_rows.txt); exhaustive bf16 sweeps
where the scale is exactly 1 so the result reduces to a library rounding;
exact-rational checks of the division; invariants.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def _f32(x: Fraction) -> np.float32:
    # nearest binary32 to an exact rational.  Fraction -> float is correctly
    # rounded to binary64, and binary64 -> binary32 after it is innocuous for a
    # quotient of two binary32 values (53 >= 2*24 + 2), so this is the
    # correctly rounded binary32 quotient.
    return np.float32(float(x))


def _lib_int8(v: np.ndarray) -> np.ndarray:
    return np.clip(np.round(v.astype(np.float64)), -127, 127).astype(np.int8)  # numpy rounds half to even


def _lib_e4m3(v: np.ndarray) -> np.ndarray:
    v = np.clip(v.astype(np.float32), -448.0, 448.0)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_golden_rows():
    n = 0
    with open(os.path.join(GOLDEN, "quant_rows.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            fmt_s, row_s, s_s, q_s = [t.strip() for t in line.split("|")]
            fmt = oracle.FMT_INT8 if fmt_s == "int8" else oracle.FMT_FP8
            x = _bf16([float(t) for t in row_s.split()])[None, :]
            q, s = oracle.quantize_per_token(fmt, x)
            assert s[0] == float(s_s), line
            if fmt == oracle.FMT_INT8:
                want = np.array([int(t) for t in q_s.split()], np.int8).view(np.uint8)
            else:
                want = np.array([int(t, 16) for t in q_s.split()], np.uint8)
            assert np.array_equal(q[0], want), (line, q[0], want)
            n += 1
    assert n >= 6


def _all_finite_bf16(limit: float) -> np.ndarray:
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    keep = np.isfinite(f) & (np.abs(f) <= limit)
    return bits[keep].astype(np.uint16)


def test_exhaustive_bf16_sweep_fp8_unit_scale():
    # rows [448, v]: amax = 448 so s = 1 exactly and q(v) = e4m3(v)
    vb = _all_finite_bf16(448.0)
    x = np.stack([np.full_like(vb, 0x43E0), vb], axis=1)  # 0x43E0 = 448.0 in bf16
    q, s = oracle.quantize_per_token(oracle.FMT_FP8, x)
    assert np.all(s == 1.0)
    v = (vb.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(q[:, 0], np.full(len(vb), 0x7E, np.uint8))
    assert np.array_equal(q[:, 1], _lib_e4m3(v))


def test_exhaustive_bf16_sweep_int8_unit_scale():
    # rows [127, v]: s = 1 exactly and q(v) = round-half-even(v)
    vb = _all_finite_bf16(127.0)
    x = np.stack([np.full_like(vb, 0x42FE), vb], axis=1)  # 0x42FE = 127.0 in bf16
    q, s = oracle.quantize_per_token(oracle.FMT_INT8, x)
    assert np.all(s == 1.0)
    v = (vb.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(q[:, 1].view(np.int8), _lib_int8(v))


@pytest.mark.parametrize("fmt,qmax", [(oracle.FMT_INT8, 127), (oracle.FMT_FP8, 448)])
def test_division_is_exact_ieee_quotient(fmt, qmax):
    # random rows with awkward scales: every q must be the rounding of the
    # correctly rounded quotient fl(x / fl(amax / Qmax)).
    g = torch.Generator().manual_seed(123)
    x = (torch.randn(24, 96, generator=g) * torch.exp(torch.randn(24, 1, generator=g) * 3)).to(torch.bfloat16)
    q, s = oracle.quantize_per_token(fmt, x)
    xf = x.to(torch.float32).numpy()
    for r in range(x.shape[0]):
        amax = float(np.max(np.abs(xf[r])))
        s_ref = _f32(Fraction(amax) / qmax)
        assert s[r] == s_ref
        quot = np.array([_f32(Fraction(float(v)) / Fraction(float(s_ref))) for v in xf[r]], np.float32)
        want = _lib_int8(quot).view(np.uint8) if fmt == oracle.FMT_INT8 else _lib_e4m3(quot)
        assert np.array_equal(q[r], want), r


def test_division_differs_from_reciprocal_multiply_somewhere():
    # the pin above is not vacuous: x * fl(1/s) differs from fl(x/s) on these
    # inputs for some element, so a reciprocal-multiply oracle would fail it.
    g = torch.Generator().manual_seed(123)
    x = (torch.randn(24, 96, generator=g) * torch.exp(torch.randn(24, 1, generator=g) * 3)).to(torch.bfloat16)
    xf = x.to(torch.float32).numpy()
    diff = 0
    for r in range(x.shape[0]):
        s = np.float32(np.max(np.abs(xf[r]))) / np.float32(127)
        diff += int(np.sum((xf[r] / s) != (xf[r] * (np.float32(1) / s))))
    assert diff > 0


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_amax_zero_rows(fmt):
    x = _bf16([[0.0, -0.0, 0.0, 0.0], [1.0, -2.0, 0.0, 0.5]])
    q, s = oracle.quantize_per_token(fmt, x)
    assert s[0] == 0.0 and not math.copysign(1, s[0]) < 0
    assert np.all(q[0] == 0)
    assert s[1] > 0


@pytest.mark.parametrize("fmt,qmax", [(oracle.FMT_INT8, 127), (oracle.FMT_FP8, 448)])
def test_quantiser_invariants_on_workload_rows(fmt, qmax):
    w = synth.WORKLOADS["fp8_attn"]
    x = synth.activations(w, 32, seed=0)
    q, s = oracle.quantize_per_token(fmt, x)
    xf = x.to(torch.float32).numpy()
    for r in range(32):
        amax = np.max(np.abs(xf[r]))
        assert amax > 0
        if fmt == oracle.FMT_INT8:
            qi = q[r].view(np.int8).astype(np.float64)
            assert np.max(np.abs(qi)) == qmax
            # |x - q s| <= s/2 (plus the quotient's own rounding)
            err = np.abs(xf[r] - qi * s[r])
            assert np.all(err <= s[r] * (0.5 + 127 * 2.0 ** -23))
        else:
            dec = np.array([oracle.e4m3_decode(int(c)) for c in q[r]])
            assert np.max(np.abs(dec)) == qmax
            v = xf[r] / s[r]
            normal = np.abs(v) >= 2.0 ** -6
            assert np.all(np.abs(dec - v)[normal] <= 2.0 ** -4 * np.abs(v[normal]) + 1e-6)
            assert np.all(np.abs(dec - v)[~normal] <= 2.0 ** -10 + 1e-9)


def test_saturation_from_division_overshoot():
    # scan amax values: the amax element itself maps to +-Qmax exactly even
    # when amax / fl(amax/Qmax) rounds above Qmax.
    overshoot = 0
    for bits in range(0x3F80, 0x4780, 7):
        amax = float(np.array([bits << 16], np.uint32).view(np.float32)[0])
        for fmt, qmax in ((oracle.FMT_INT8, 127), (oracle.FMT_FP8, 448)):
            x = _bf16([[amax, -amax, amax / 3]])
            q, s = oracle.quantize_per_token(fmt, x)
            if np.float32(amax) / s[0] > qmax:
                overshoot += 1
            if fmt == oracle.FMT_INT8:
                assert q[0, 0].view(np.int8) == 127 and q[0, 1].view(np.int8) == -127
            else:
                assert q[0, 0] == 0x7E and q[0, 1] == 0xFE
    assert overshoot > 0  # the scan does exercise the clamp


def test_block_quant_1x128_groups():
    # groups of 128 along K have independent scales: row-major [rows][cols/128]
    g = torch.Generator().manual_seed(5)
    x = torch.randn(3, 384, generator=g)
    x[:, 128:256] *= 1000.0
    x = x.to(torch.bfloat16)
    q, s = oracle.quantize_block(x, 1, 128)
    assert s.shape == (3, 3)
    xf = x.to(torch.float32).numpy()
    for r in range(3):
        for gi in range(3):
            blk = xf[r, gi * 128:(gi + 1) * 128]
            s_ref = _f32(Fraction(float(np.max(np.abs(blk)))) / 448)
            assert s[r, gi] == s_ref
            quot = np.array([_f32(Fraction(float(v)) / Fraction(float(s_ref))) for v in blk], np.float32)
            assert np.array_equal(q[r, gi * 128:(gi + 1) * 128], _lib_e4m3(quot))


def test_block_quant_128x128_layout_and_ragged_edge():
    # 300 x 384 -> 3 x 3 blocks (last block row holds 44 rows); each block gets
    # a distinct known amax so a transposed or mis-strided index fails.
    g = torch.Generator().manual_seed(6)
    x = torch.rand(300, 384, generator=g) * 0.5
    amax = np.zeros((3, 3))
    for bi in range(3):
        for bj in range(3):
            val = float(2 ** (bi * 3 + bj - 4))
            r = min(bi * 128 + 7 * bj, 299)
            x[r, bj * 128 + 5 * bi] = -val if (bi + bj) % 2 else val
            amax[bi, bj] = max(val, 0.5)
    x = x.to(torch.bfloat16)
    q, s = oracle.quantize_block(x, 128, 128)
    assert s.shape == (3, 3)
    xf = x.to(torch.float32).numpy()
    for bi in range(3):
        for bj in range(3):
            blk = xf[bi * 128:min(bi * 128 + 128, 300), bj * 128:(bj + 1) * 128]
            a = float(np.max(np.abs(blk)))
            assert a == pytest.approx(amax[bi, bj], rel=1e-2)
            assert s[bi, bj] == _f32(Fraction(a) / 448)
            quot = (blk / s[bi, bj]).astype(np.float32)  # binary32 quotients
            assert np.array_equal(q[bi * 128:min(bi * 128 + 128, 300), bj * 128:(bj + 1) * 128],
                                  _lib_e4m3(quot))


def test_block_quant_zero_block():
    x = torch.zeros(128, 256)
    x[:, 128:] = 1.0
    q, s = oracle.quantize_block(x.to(torch.bfloat16), 128, 128)
    assert s[0, 0] == 0.0 and np.all(q[:, :128] == 0)
    assert s[0, 1] == np.float32(1.0) / np.float32(448.0)
    assert np.all(q[:, 128:] == 0x7E)
