"""Pin of the oracle's epilogue: the order and rounding of the scale / bias steps.

Reading (plainest, of the formula the page "Helion in vLLM: A Unified Route to
Tunable Linear Kernels" implies for its per-token formats in "What the
integration changes": the product is scaled by the activation scale, then by
the weight scale, then the bias is added): each step is a separately rounded
binary32 operation, left to right,

    y0 = RN32(acc)            (FP8: the exact sum in 2^-18 units, then the exact
                               power-of-two scaling)
    y1 = RN32(y0 * s_a[m])
    y2 = RN32(y1 * s_w[n])
    y3 = RN32(y2 + bias[n])
    C  = RN_bf16(y3)

The reference here is built from exact rationals and a rounding routine
written from the definition of round-to-nearest, ties-to-even (nothing of the
oracle, numpy's float32 arithmetic or torch's conversions is used for it).
The second test shows the pin has teeth: for each plausible other order
(the scales multiplied together first, the weight scale first, the bias added
by a fused multiply-add) it finds inputs on which that order gives a different
bf16 result, and checks that the oracle gives the left-to-right one there.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def round_binary(x: Fraction, p: int) -> Fraction:
    """x rounded to the nearest binary float with p significant bits, ties to
    the even significand (exponent range unbounded: callers stay normal)."""
    if x == 0:
        return Fraction(0)
    neg = x < 0
    a = -x if neg else x
    # e = floor(log2(a)), exactly
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    unit = Fraction(2) ** (e - p + 1)          # weight of the last kept bit
    scaled = a / unit                          # in [2^(p-1), 2^p)
    q, r = divmod(scaled.numerator, scaled.denominator)
    twice = 2 * r
    if twice > scaled.denominator or (twice == scaled.denominator and q % 2 == 1):
        q += 1
    out = q * unit
    return -out if neg else out


def rn32(x: Fraction) -> Fraction:
    if x != 0:
        assert Fraction(2) ** -126 <= abs(x) < Fraction(2) ** 128, "outside the binary32 normal range"
    return round_binary(x, 24)


def rn_bf16(x: Fraction) -> Fraction:
    return round_binary(x, 8)


def f32_frac(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def bf16_frac(bits) -> Fraction:
    return Fraction(float(oracle.bf16_bits_to_f32(np.array([bits], np.uint16))[0]))


def left_to_right(acc_units: int, unit: Fraction, sa: Fraction, sw: Fraction, bias):
    y = rn32(Fraction(acc_units)) * unit       # FP8: exact power-of-two scaling
    y = rn32(y * sa)
    y = rn32(y * sw)
    if bias is not None:
        y = rn32(y + bias)
    return rn_bf16(y)


def test_round_binary_matches_hand_cases():
    # 1 + 2^-24 is a tie between 1 and 1 + 2^-23: goes to even (1)
    assert rn32(1 + Fraction(1, 2 ** 24)) == 1
    # 1 + 3*2^-24 is a tie between 1 + 2^-23 and 1 + 2^-22: goes to even (1 + 2^-22)
    assert rn32(1 + Fraction(3, 2 ** 24)) == 1 + Fraction(1, 2 ** 22)
    assert rn32(Fraction(1, 3)) == Fraction(11184811, 2 ** 25)   # 0x3EAAAAAB
    assert rn_bf16(Fraction(257, 256)) == 1                       # tie -> even
    assert rn_bf16(Fraction(259, 256)) == Fraction(260, 256)      # tie -> even (odd below)
    assert rn_bf16(-Fraction(385, 256)) == -Fraction(384, 256)


def _problem(fmt, M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g))).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    aq, sa = oracle.quantize_per_token(fmt, a)
    wq, sw = oracle.quantize_per_token(fmt, w)
    return aq, sa, wq, sw, b


def _units(fmt, codes: np.ndarray) -> np.ndarray:
    if fmt == oracle.FMT_INT8:
        return codes.view(np.int8).astype(np.int64)
    lut = np.array([oracle.e4m3_units(c) for c in range(256)], np.int64)
    return lut[codes]


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
@pytest.mark.parametrize("with_bias", [True, False])
def test_epilogue_is_left_to_right_separately_rounded(fmt, with_bias):
    M, N, K = 6, 48, 256
    aq, sa, wq, sw, b = _problem(fmt, M, N, K, 21 + fmt)
    bias = b if with_bias else None
    c = oracle.scaled_mm(fmt, aq, sa, wq, sw, bias)
    acc = _units(fmt, aq) @ _units(fmt, wq).T            # exact integers (< 2^53)
    unit = Fraction(1) if fmt == oracle.FMT_INT8 else Fraction(1, 2 ** 18)
    bbits = b.view(torch.int16).numpy().view(np.uint16)
    for m in range(M):
        for n in range(N):
            want = left_to_right(int(acc[m, n]), unit, f32_frac(sa[m]), f32_frac(sw[n]),
                                 bf16_frac(bbits[n]) if with_bias else None)
            assert bf16_frac(c[m, n]) == want, (m, n)


# ----------------------------------------------------------- non-vacuity ----
def _alt_scales_first(acc, sa, sw, bias):
    y = rn32(Fraction(acc))
    y = rn32(y * rn32(sa * sw))
    return rn_bf16(rn32(y + bias))


def _alt_weight_scale_first(acc, sa, sw, bias):
    y = rn32(Fraction(acc))
    y = rn32(rn32(y * sw) * sa)
    return rn_bf16(rn32(y + bias))


def _alt_fused_bias(acc, sa, sw, bias):
    y = rn32(rn32(Fraction(acc)) * sa)
    return rn_bf16(rn32(y * sw + bias))      # one rounding for multiply and add


def _f32_from_bits(u: int) -> np.float32:
    return np.array([u], np.uint32).view(np.float32)[0]


@pytest.mark.parametrize("alt", [_alt_scales_first, _alt_weight_scale_first, _alt_fused_bias])
def test_other_orders_are_distinguishable_and_the_oracle_is_not_them(alt):
    # INT8, K = 128: A row 0 holds the code a at k = 0 only, W row 0 the code
    # w at k = 0 only, so acc = a * w exactly.  The orders differ by about one
    # binary32 ulp, which shows in bf16 only near a bf16 rounding midpoint, so
    # the weight scale is chosen to put the exact result next to one: with a
    # random midpoint T and bias b, s_w = RN32((T - b) / RN32(acc * s_a)).
    # Among such inputs, find one on which the alternative rounds to another
    # bf16 value than the left-to-right order, then run the oracle on it.
    rng = np.random.default_rng(5)
    found = None
    for _ in range(4000):
        a = int(rng.integers(1, 128))
        w = int(rng.integers(1, 128)) * (1 if rng.random() < 0.5 else -1)
        sa = f32_frac(_f32_from_bits(int(rng.integers(0x3B000000, 0x3D000000))))   # ~2e-3 .. 3e-2
        bb = int(rng.integers(0x3C00, 0x3E80)) | (0x8000 if rng.random() < 0.5 else 0)  # bf16 bias
        bias = bf16_frac(bb)
        sig = int(rng.integers(128, 256)) * 2 + 1                                      # 9-bit odd significand
        T = Fraction(sig, 2 ** 9) * Fraction(2) ** int(rng.integers(-3, 3)) * (1 if rng.random() < 0.5 else -1)
        y1 = rn32(Fraction(a * w) * sa)
        sw = rn32((T - bias) / y1)
        if sw <= 0:
            continue
        ref = left_to_right(a * w, Fraction(1), sa, sw, bias)
        if alt(a * w, sa, sw, bias) != ref:
            found = (a, w, sa, sw, bb, ref)
            break
    assert found is not None, "no input separates the two orders"
    a, w, sa, sw, bb, ref = found
    aq = np.zeros((1, 128), np.uint8)
    wq = np.zeros((1, 128), np.uint8)
    aq[0, 0] = np.uint8(a)
    wq[0, 0] = np.int8(w).view(np.uint8)
    bias_t = torch.from_numpy(np.array([bb], np.uint16).view(np.int16)).view(torch.bfloat16)
    c = oracle.scaled_mm(oracle.FMT_INT8, aq, np.array([float(sa)], np.float32), wq,
                         np.array([float(sw)], np.float32), bias_t)
    assert bf16_frac(c[0, 0]) == ref
    assert bf16_frac(c[0, 0]) != alt(a * w, sa, sw, bias)
