"""Pins of the oracle's block-scaled formats: MXFP8 and NVFP4 codecs, their
quantisers and the block-scaled GEMM.

The page "Helion in vLLM: A Unified Route to Tunable Linear Kernels"
(introduction) lists NVFP4 among the formats vLLM's quantized linear layers
serve, and gives no definition.  The oracle follows the formats' public
definitions (OCP Microscaling Formats v1.0 for MXFP8 and the E2M1 element type;
NVIDIA's two-level NVFP4 scaling for the E4M3 block scale and the per-tensor
decode scale), with the readings stated in ``oracle/qlin_oracle.c``.

What pins it, independently of its code:
  - hand-derived code points and round-to-nearest ties (``tests/golden/``);
  - every element code is checked against a brute-force search for the
    nearest representable value (ties to the even code), not against the
    oracle's own rounding routine;
  - the MXFP8 scale is checked by its defining property, amax / X in
    [2^8, 2^9), plus closed-form special cases (saturation, amax = 0, the
    clamp at 2^-127, the largest bf16);
  - the GEMMs are replayed from exact rationals with a rounding routine written
    from the definition of round-to-nearest-even; a non-vacuity check shows
    that a different epilogue order would have been caught.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from test_oracle_epilogue_order import rn32, rn_bf16, round_binary

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(vals) -> torch.Tensor:
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def _exact(x: torch.Tensor) -> list[Fraction]:
    return [Fraction(float(v)) for v in x.float().reshape(-1)]


E4M3_MAG = [(c, Fraction(oracle.e4m3_decode(c))) for c in range(0x7F)]   # every finite magnitude code
E2M1_MAG = [(c, Fraction(oracle.e2m1_decode(c))) for c in range(8)]


def nearest_code(v: Fraction, table) -> int:
    """Brute force: the magnitude code closest to |v|, ties to the even code."""
    a = abs(v)
    best, bd = None, None
    for c, m in table:
        d = abs(a - m)
        if bd is None or d < bd or (d == bd and c % 2 == 0 and best % 2 == 1):
            best, bd = c, d
    return best


# ---------------------------------------------------------------- codecs ----
def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_e2m1_golden_code_points_and_ties():
    for row in _golden("e2m1_codes.txt"):
        if row[0] == "decode":
            code, val = int(row[1], 16), float(row[2])
            got = oracle.e2m1_decode(code)
            assert got == val and np.signbit(got) == np.signbit(val), row
        else:
            v, code = float(row[1]), int(row[2], 16)
            assert oracle.e2m1_encode(v) == code, row


def test_e8m0_golden_code_points():
    for code, lg, *_ in _golden("e8m0_codes.txt"):
        assert oracle.e8m0_decode(int(code, 16)) == 2.0 ** int(lg)
    assert np.isnan(oracle.e8m0_decode(0xFF))


def test_e2m1_encode_is_the_nearest_value_on_a_dense_grid():
    for i in range(-1400, 1401):
        v = i / 200.0                                         # step 0.005 over [-7, 7]
        code = oracle.e2m1_encode(v)
        assert code & 7 == nearest_code(Fraction(v), E2M1_MAG), v
        assert (code >> 3) == (1 if np.signbit(v) else 0)


# ------------------------------------------------------------------ MXFP8 ----
def _mx_rows(seed, rows=6, cols=256):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    # per-block magnitudes over a wide range, some outliers, some zeros
    mag = torch.exp2(torch.randint(-40, 40, (rows, cols // 32), generator=g).float())
    x = x * mag.repeat_interleave(32, dim=1)
    x[0, 5] *= 300.0
    x[1, 32:64] = 0.0
    x[2, :32] = torch.tensor([-0.0] * 32)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mxfp8_scale_property_and_nearest_codes(seed):
    x = _mx_rows(seed)
    q, sf = oracle.quantize_mxfp8(x)
    xs = x.float().numpy()
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 32):
            blk = [Fraction(float(v)) for v in xs[r, 32 * b:32 * b + 32]]
            amax = max(abs(v) for v in blk)
            if amax == 0:
                assert sf[r, b] == 0 and not q[r, 32 * b:32 * b + 32].any()
                continue
            X = Fraction(oracle.e8m0_decode(int(sf[r, b])))
            if Fraction(2) ** -119 <= amax:                   # clamp inactive
                assert 256 <= amax / X < 512, (r, b)
            for i, v in enumerate(blk):
                code = int(q[r, 32 * b + i])
                assert code & 0x7F == nearest_code(v / X, E4M3_MAG), (r, b, i)
                assert (code >> 7) == (1 if np.signbit(xs[r, 32 * b + i]) else 0)


def test_mxfp8_closed_form_blocks():
    x = torch.zeros(6, 32)
    x[0] = 1.0                                   # amax 1: X = 2^-8, code of 256
    x[1, 0], x[1, 1:] = 500.0, 3.0               # amax 500: X = 1, 500 saturates to 448
    x[2, 0] = 448.0                              # exact largest E4M3
    x[3] = 0.0                                   # amax 0
    xb = x.to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16).copy()
    bits[4, :] = 0
    bits[4, 0] = 0x0001                          # smallest bf16 subnormal 2^-133: e clamps to -127
    bits[5, 0] = 0x7F7F                          # largest bf16 (2 - 2^-7) 2^127: e = 119
    q, sf = oracle.quantize_mxfp8(bits)
    assert sf[0, 0] == 127 - 8 and np.all(q[0] == 0x78)
    assert sf[1, 0] == 127 and q[1, 0] == 0x7E and q[1, 1] == 0x44   # 3.0 = (1 + 4/8) * 2^1
    assert sf[2, 0] == 127 and q[2, 0] == 0x7E
    assert sf[3, 0] == 0 and not q[3].any()
    assert sf[4, 0] == 0 and q[4, 0] == 0x08 and not q[4, 1:].any()   # 2^-133 / 2^-127 = 2^-6
    assert sf[5, 0] == 127 + 119 and q[5, 0] == 0x7E                  # 510 saturates


def test_mxfp8_block_indexing():
    # block b of row r holds magnitude 2^(b + 3r): a transposed or shifted
    # scale index would put the wrong exponent on some block
    x = torch.zeros(3, 8 * 32)
    for r in range(3):
        for b in range(8):
            x[r, 32 * b:32 * b + 32] = 1.5 * 2.0 ** (b + 3 * r)
    q, sf = oracle.quantize_mxfp8(x.to(torch.bfloat16))
    for r in range(3):
        for b in range(8):
            assert sf[r, b] == 127 + (b + 3 * r) - 8
    assert np.all(q == 0x7C)                     # 1.5 * 2^8 = 384


# ------------------------------------------------------------------ NVFP4 ----
def _e4m3_of(t: Fraction) -> int:
    return nearest_code(t, E4M3_MAG)             # t >= 0 here; saturates at 448 by nearness


@pytest.mark.parametrize("seed,g", [(0, 1.0 / 448), (1, 0.01171875), (2, 3.7e-3), (3, 1.0)])
def test_nvfp4_block_scale_and_nearest_codes(seed, g):
    x = _mx_rows(seed, rows=5, cols=128)
    x = (x.float() / x.float().abs().amax() * 40.0).to(torch.bfloat16)
    q, sf = oracle.quantize_nvfp4(x, g)
    gf = Fraction(float(np.float32(g)))
    xs = x.float().numpy()
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 16):
            blk = [Fraction(float(v)) for v in xs[r, 16 * b:16 * b + 16]]
            amax = max(abs(v) for v in blk)
            t = rn32(amax / 6) if amax else Fraction(0)
            t = rn32(t / gf) if t else Fraction(0)
            assert sf[r, b] == _e4m3_of(t), (r, b)
            s = Fraction(oracle.e4m3_decode(int(sf[r, b])))
            d = rn32(s * gf) if s else Fraction(0)
            for i, v in enumerate(blk):
                byte = int(q[r, 8 * b + i // 2])
                code = (byte >> (4 * (i % 2))) & 0xF
                if d == 0:
                    assert code == 0
                    continue
                qv = rn32(v / d) if v else Fraction(0)
                assert code & 7 == nearest_code(qv, E2M1_MAG), (r, b, i)
                assert (code >> 3) == (1 if np.signbit(xs[r, 16 * b + i]) else 0)


def test_nvfp4_worked_block_and_packing():
    x = torch.zeros(3, 16)
    x[0, :4] = torch.tensor([6.0, 3.0, -1.5, 0.5])
    x[1, 0] = 2.0                                 # only element 0: low nibble of byte 0
    q, sf = oracle.quantize_nvfp4(x.to(torch.bfloat16), 1.0)
    assert sf[0, 0] == 0x38                       # amax 6: t = 1, scale code of 1.0
    assert q[0, 0] == 0x57 and q[0, 1] == 0x1B and not q[0, 2:].any()
    assert sf[1, 0] == 0x2B                       # amax 2: t = 1/3 -> nearest E4M3 1.375 * 2^-2 (0x2B)
    s = oracle.e4m3_decode(0x2B)
    assert q[1, 0] == oracle.e2m1_encode(np.float32(2.0) / np.float32(s)) and q[1, 0] == 0x07
    assert sf[2, 0] == 0 and not q[2].any()       # amax 0
    # saturating block scale: a tiny g makes t exceed 448
    q, sf = oracle.quantize_nvfp4(x[:1].to(torch.bfloat16), 1e-4)
    assert sf[0, 0] == 0x7E


# ---------------------------------------------------------------- GEMMs ----
def _dec_e4m3(c):
    return Fraction(oracle.e4m3_decode(int(c)))


def _mx_case(seed, M=3, N=4, K=64):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g)
    w = torch.randn(N, K, generator=g)
    a *= torch.exp2(torch.randint(-6, 7, (M, K // 32), generator=g).float()).repeat_interleave(32, 1)
    w *= torch.exp2(torch.randint(-6, 7, (N, K // 32), generator=g).float()).repeat_interleave(32, 1)
    return a.to(torch.bfloat16), w.to(torch.bfloat16)


@pytest.mark.parametrize("seed", range(6))
def test_mxfp8_gemm_replayed_from_exact_rationals(seed):
    a, w = _mx_case(seed)
    bias = (torch.randn(4, generator=torch.Generator().manual_seed(99 + seed))).to(torch.bfloat16)
    aq, asf = oracle.quantize_mxfp8(a)
    wq, wsf = oracle.quantize_mxfp8(w)
    c = oracle.gemm_block_scaled(oracle.FMT_MXFP8, aq, asf, wq, wsf, bias=bias)
    bb = _exact(bias)
    M, K = aq.shape
    for m in range(M):
        for n in range(wq.shape[0]):
            acc = sum(_dec_e4m3(aq[m, k]) * _dec_e4m3(wq[n, k])
                      * Fraction(oracle.e8m0_decode(int(asf[m, k // 32])))
                      * Fraction(oracle.e8m0_decode(int(wsf[n, k // 32]))) for k in range(K))
            y = rn32(acc) if acc else Fraction(0)
            y = rn32(y + bb[n]) if y + bb[n] else Fraction(0)
            ref = rn_bf16(y)
            got = Fraction(float(oracle.bf16_bits_to_f32(c[m:m + 1, n:n + 1])[0, 0]))
            assert got == ref, (m, n)


def test_mxfp8_gemm_one_hot_closed_form():
    K = 96
    aq = np.zeros((1, K), np.uint8)
    wq = np.zeros((1, K), np.uint8)
    aq[0, 70], wq[0, 70] = 0x46, 0xC4            # 3.5 = 1.75 * 2^1, -3 = -1.5 * 2^1 (block 2)
    asf = np.array([[127, 127, 130]], np.uint8)   # block 2: 2^3
    wsf = np.array([[127, 127, 125]], np.uint8)   # block 2: 2^-2
    c = oracle.gemm_block_scaled(oracle.FMT_MXFP8, aq, asf, wq, wsf)
    assert oracle.bf16_bits_to_f32(c)[0, 0] == 3.5 * -3.0 * 2.0 ** 3 * 2.0 ** -2


def _nv_case(seed, M=3, N=4, K=64):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g) * torch.exp2(torch.randint(-3, 4, (M, K // 16), generator=g).float()
                                                    ).repeat_interleave(16, 1)
    w = torch.randn(N, K, generator=g) * 0.05
    return a.to(torch.bfloat16), w.to(torch.bfloat16)


def _nv_exact(aq, asf, wq, wsf, m, n):
    K = aq.shape[1] * 2

    def el(row, k):
        return Fraction(oracle.e2m1_decode((int(row[k // 2]) >> (4 * (k % 2))) & 0xF))

    return sum(el(aq[m], k) * el(wq[n], k) * _dec_e4m3(asf[m, k // 16]) * _dec_e4m3(wsf[n, k // 16])
               for k in range(K))


@pytest.mark.parametrize("seed", range(6))
def test_nvfp4_gemm_replayed_from_exact_rationals(seed):
    a, w = _nv_case(seed)
    g_a = float(np.float32(a.float().abs().max() / 2688.0))
    g_w = float(np.float32(w.float().abs().max() / 2688.0))
    bias = (torch.randn(4, generator=torch.Generator().manual_seed(7 + seed)) * 0.1).to(torch.bfloat16)
    aq, asf = oracle.quantize_nvfp4(a, g_a)
    wq, wsf = oracle.quantize_nvfp4(w, g_w)
    c = oracle.gemm_block_scaled(oracle.FMT_NVFP4, aq, asf, wq, wsf, g_a, g_w, bias=bias)
    bb, ga, gw = _exact(bias), Fraction(g_a), Fraction(g_w)
    for m in range(aq.shape[0]):
        for n in range(wq.shape[0]):
            acc = _nv_exact(aq, asf, wq, wsf, m, n)
            y = rn32(acc) if acc else Fraction(0)
            y = rn32(y * ga) if y else Fraction(0)
            y = rn32(y * gw) if y else Fraction(0)
            y = rn32(y + bb[n]) if y + bb[n] else Fraction(0)
            got = Fraction(float(oracle.bf16_bits_to_f32(c[m:m + 1, n:n + 1])[0, 0]))
            assert got == rn_bf16(y), (m, n)


def test_nvfp4_epilogue_order_has_teeth():
    """Multiplying the two per-tensor scales together first would round
    differently.  Random inputs almost never show it at bf16 (the two orders
    differ by an fp32 ulp), so g_w is chosen to put the product next to a bf16
    rounding midpoint; among such inputs find three where the orders disagree
    and check that the oracle takes the stated left-to-right order there."""
    K = 32
    rng = np.random.default_rng(5)
    midpoint = Fraction(1) + Fraction(1, 256)          # halfway between two bf16 values
    found = 0
    for _ in range(4000):
        aq = rng.integers(0, 256, size=(1, K // 2), dtype=np.uint8)
        wq = rng.integers(0, 256, size=(1, K // 2), dtype=np.uint8)
        asf = rng.integers(0x28, 0x50, size=(1, 2), dtype=np.uint8)
        wsf = rng.integers(0x28, 0x50, size=(1, 2), dtype=np.uint8)
        acc = _nv_exact(aq, asf, wq, wsf, 0, 0)
        if acc == 0:
            continue
        g_a = float(np.float32(rng.uniform(0.3, 3.0)))
        y1 = rn32(rn32(acc) * Fraction(g_a))
        g_w = float(rn32(midpoint / y1) * (1 + Fraction(int(rng.integers(-3, 4)), 1 << 24)))
        g_w = float(np.float32(g_w))
        if g_w <= 0:
            continue
        ltr = rn_bf16(rn32(y1 * Fraction(g_w)))
        alt = rn_bf16(rn32(rn32(acc) * rn32(Fraction(g_a) * Fraction(g_w))))
        if ltr == alt:
            continue
        c = oracle.gemm_block_scaled(oracle.FMT_NVFP4, aq, asf, wq, wsf, g_a, g_w)
        assert Fraction(float(oracle.bf16_bits_to_f32(c)[0, 0])) == ltr
        found += 1
        if found == 3:
            break
    assert found == 3, "no input separates the two epilogue orders"


def test_nvfp4_gemm_block_indexing():
    # distinct block scales per (row, block): a transposed or shifted scale
    # index changes the exact result
    K = 64
    aq = np.full((2, K // 2), 0x22, np.uint8)     # every element 1.0
    wq = np.full((1, K // 2), 0x22, np.uint8)
    asf = np.array([[0x30, 0x38, 0x40, 0x48], [0x31, 0x39, 0x41, 0x49]], np.uint8)
    wsf = np.array([[0x38, 0x40, 0x48, 0x50]], np.uint8)
    c = oracle.gemm_block_scaled(oracle.FMT_NVFP4, aq, asf, wq, wsf)
    for m in range(2):
        want = sum(16 * oracle.e4m3_decode(int(asf[m, b])) * oracle.e4m3_decode(int(wsf[0, b])) for b in range(4))
        assert oracle.bf16_bits_to_f32(c)[m, 0] == float(rn_bf16(rn32(Fraction(want))))


def test_round_binary_helper_is_round_to_nearest_even():
    # the rounding routine the replays use, on hand-checked values
    assert round_binary(Fraction(3, 2), 1) == 2          # 1.5 -> tie -> even significand (2)
    assert round_binary(Fraction(5, 2), 2) == 2          # 2.5 -> tie between 2 and 3 -> 2
    assert round_binary(Fraction(7, 2), 2) == 4          # 3.5 -> tie between 3 and 4 -> 4
