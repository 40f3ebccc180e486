"""Pins for the oracle's scaled GEMM (INT8, FP8 per-token/per-channel, Block-FP8).

Definitions (plainest reading; the page "Helion in vLLM: A Unified Route to
Tunable Linear Kernels", section "What the integration changes", names the
formats and strategies but prints no formula):
  C[m,n] = bf16( (fp32(sum_k A_q[m,k] W_q[n,k]) * s_a[m]) * s_w[n] + bias[n] )
  Block-FP8: C[m,n] = bf16( sum_kb P_kb[m,n] * s_a[m,kb] * s_w[n//128,kb] )

Pins: the INT8 accumulators against numpy's integer matmul (exact); outputs
against a float64 library matmul of operands dequantised by torch's own e4m3
decoder and against exact rational arithmetic on tiny inputs (within one bf16
ulp of the exact value); one-hot and constant closed forms; the sampled-index
path against the dense one; row independence.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth


def _dequant_e4m3(q: np.ndarray) -> np.ndarray:
    return torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _bf16_f(c_bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f32(c_bits).astype(np.float64)


def _within_one_bf16_ulp(c_bits: np.ndarray, exact: np.ndarray):
    got = _bf16_f(c_bits)
    # one bf16 ulp at |exact| (8 significant bits), with a floor for tiny values
    ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(exact), 1e-30))[1] - 8)
    bad = np.abs(got - exact) > ulp
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], exact[bad][:5])


def _quantized_problem(fmt, M, N, K, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g))).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16) if bias else None
    if fmt == oracle.FMT_FP8_BLOCK:
        aq, sa = oracle.quantize_block(a, 1, 128)
        wq, sw = oracle.quantize_block(w, 128, 128)
        b = None
    else:
        aq, sa = oracle.quantize_per_token(fmt, a)
        wq, sw = oracle.quantize_per_token(fmt, w)
    return aq, sa, wq, sw, b


@pytest.mark.parametrize("M,N,K", [(5, 48, 256), (17, 130, 384), (1, 16, 128)])
def test_int8_accumulators_equal_integer_matmul(M, N, K):
    aq, sa, wq, sw, b = _quantized_problem(oracle.FMT_INT8, M, N, K, 1)
    c, acc = oracle.scaled_mm(oracle.FMT_INT8, aq, sa, wq, sw, b, want_acc=True)
    ref = aq.view(np.int8).astype(np.int64) @ wq.view(np.int8).astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), ref)


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
@pytest.mark.parametrize("M,N,K", [(7, 40, 256), (33, 136, 512)])
def test_per_token_output_vs_float64_library_matmul(fmt, M, N, K):
    aq, sa, wq, sw, b = _quantized_problem(fmt, M, N, K, 2)
    c = oracle.scaled_mm(fmt, aq, sa, wq, sw, b)
    if fmt == oracle.FMT_INT8:
        da, dw = aq.view(np.int8).astype(np.float64), wq.view(np.int8).astype(np.float64)
    else:
        da, dw = _dequant_e4m3(aq), _dequant_e4m3(wq)
    exact = (torch.from_numpy(da) @ torch.from_numpy(dw).T).numpy()  # exact: < 2^53 in 2^-18 units
    exact = exact * sa.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    exact = exact + b.to(torch.float64).numpy()[None, :]
    _within_one_bf16_ulp(c, exact)


@pytest.mark.parametrize("M,N,K", [(3, 256, 384), (9, 384, 256), (1, 128, 128)])
def test_block_output_vs_float64_library_matmul(M, N, K):
    aq, sa, wq, sw, _ = _quantized_problem(oracle.FMT_FP8_BLOCK, M, N, K, 3)
    c = oracle.scaled_mm(oracle.FMT_FP8_BLOCK, aq, sa, wq, sw)
    da, dw = torch.from_numpy(_dequant_e4m3(aq)), torch.from_numpy(_dequant_e4m3(wq))
    exact = np.zeros((M, N))
    for kb in range(K // 128):
        p = (da[:, kb * 128:(kb + 1) * 128] @ dw[:, kb * 128:(kb + 1) * 128].T).numpy()
        s_w_cols = np.repeat(sw[:, kb].astype(np.float64), 128)[:N]
        exact += p * sa[:, kb].astype(np.float64)[:, None] * s_w_cols[None, :]
    _within_one_bf16_ulp(c, exact)


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8, oracle.FMT_FP8_BLOCK])
def test_tiny_brute_force_exact_rationals(fmt):
    M, N, K = 2, 16, 256 if fmt != oracle.FMT_FP8_BLOCK else 256
    aq, sa, wq, sw, b = _quantized_problem(fmt, M, N, K, 4 + fmt)
    c = oracle.scaled_mm(fmt, aq, sa, wq, sw, b)

    def val(code):
        if fmt == oracle.FMT_INT8:
            return Fraction(int(np.uint8(code).view(np.int8)))
        return Fraction(oracle.e4m3_units(int(code)), 512)

    exact = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            if fmt == oracle.FMT_FP8_BLOCK:
                tot = Fraction(0)
                for kb in range(K // 128):
                    p = sum(val(aq[m, k]) * val(wq[n, k]) for k in range(kb * 128, kb * 128 + 128))
                    tot += p * Fraction(float(sa[m, kb])) * Fraction(float(sw[n // 128, kb]))
            else:
                p = sum(val(aq[m, k]) * val(wq[n, k]) for k in range(K))
                tot = p * Fraction(float(sa[m])) * Fraction(float(sw[n]))
                if b is not None:
                    tot += Fraction(float(b[n].float()))
            exact[m, n] = float(tot)
    _within_one_bf16_ulp(c, exact)


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_one_hot_closed_form(fmt):
    # A row m has one non-zero at k0, W row n one non-zero at k0: C = a*w*s_a*s_w
    M, N, K = 4, 32, 256
    aq = np.zeros((M, K), np.uint8)
    wq = np.zeros((N, K), np.uint8)
    one = 0x38 if fmt == oracle.FMT_FP8 else 1           # e4m3 1.0 / int8 1
    two = 0x40 if fmt == oracle.FMT_FP8 else 2           # e4m3 2.0 / int8 2
    aq[1, 200] = two
    wq[5, 200] = one
    wq[6, 201] = one                                     # different k: no overlap
    sa = np.array([1, 0.5, 1, 1], np.float32)
    sw = np.full(N, 0.25, np.float32)
    c = oracle.scaled_mm(fmt, aq, sa, wq, sw)
    f = _bf16_f(c)
    assert f[1, 5] == 2 * 0.5 * 0.25
    f[1, 5] = 0
    assert np.all(f == 0)


def test_block_one_hot_closed_form_selects_the_right_scales():
    M, N, K = 2, 256, 384
    aq = np.zeros((M, K), np.uint8)
    wq = np.zeros((N, K), np.uint8)
    aq[1, 300] = 0x40                                    # 2.0 in K-block 2
    wq[200, 300] = 0x38                                  # 1.0, weight block row 1
    sa = np.arange(1, M * 3 + 1, dtype=np.float32).reshape(M, 3)
    sw = np.arange(1, 2 * 3 + 1, dtype=np.float32).reshape(2, 3) * 0.5
    c = oracle.scaled_mm(oracle.FMT_FP8_BLOCK, aq, sa, wq, sw)
    f = _bf16_f(c)
    assert f[1, 200] == 2.0 * sa[1, 2] * sw[1, 2]
    f[1, 200] = 0
    assert np.all(f == 0)


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_constant_rows_closed_form(fmt):
    M, N, K = 3, 16, 512
    code_a = 3 if fmt == oracle.FMT_INT8 else 0x44          # 3 / e4m3 3.0
    code_w = 0xFE if fmt == oracle.FMT_INT8 else 0xB0       # -2 / e4m3 -0.5
    val_a = 3.0
    val_w = -2.0 if fmt == oracle.FMT_INT8 else -0.5
    aq = np.full((M, K), code_a, np.uint8)
    wq = np.full((N, K), code_w, np.uint8)
    sa = np.array([0.5, 1.0, 2.0], np.float32)
    sw = np.full(N, 0.125, np.float32)
    c = oracle.scaled_mm(fmt, aq, sa, wq, sw)
    want = K * val_a * val_w * sa[:, None].astype(np.float64) * 0.125
    assert np.array_equal(_bf16_f(c), np.broadcast_to(want, (M, N)))


def test_bias_only_when_activation_row_is_zero():
    # amax = 0 row -> s_a = 0, q = 0 -> C row is exactly bf16(bias)
    w = synth.WORKLOADS["fp8_attn"]
    a = synth.activations(w, 3, seed=0)[:, :256].clone()
    a[1] = 0
    wt = synth.normal((64, 256), 0.02, 9)
    b = synth.normal((64,), 0.1, 10)
    aq, sa = oracle.quantize_per_token(oracle.FMT_FP8, a)
    wq, sw = oracle.quantize_per_token(oracle.FMT_FP8, wt)
    c = oracle.scaled_mm(oracle.FMT_FP8, aq, sa, wq, sw, b)
    assert sa[1] == 0
    assert np.array_equal(c[1], synth.bf16_bits(b))


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8, oracle.FMT_FP8_BLOCK])
def test_sampled_indices_equal_dense_slice(fmt):
    aq, sa, wq, sw, b = _quantized_problem(fmt, 20, 384, 256, 8)
    dense = oracle.scaled_mm(fmt, aq, sa, wq, sw, b)
    mi = np.array([19, 0, 7, 7])
    ni = np.array([383, 0, 129, 255, 5])
    samp = oracle.scaled_mm(fmt, aq, sa, wq, sw, b, m_idx=mi, n_idx=ni)
    assert np.array_equal(samp, dense[np.ix_(mi, ni)])


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8, oracle.FMT_FP8_BLOCK])
def test_rows_do_not_depend_on_batch(fmt):
    aq, sa, wq, sw, b = _quantized_problem(fmt, 40, 256, 256, 9)
    full = oracle.scaled_mm(fmt, aq, sa, wq, sw, b)
    part = oracle.scaled_mm(fmt, aq[:16].copy(), sa[:16].copy(), wq, sw, b)
    assert np.array_equal(full[:16], part)


def test_int8_worst_case_accumulator_fits_int32():
    # 127 * 127 * 6144 < 2^31: the extreme K of the workloads stays in range
    K = 6144
    aq = np.full((1, K), 127, np.uint8)
    wq = np.full((2, K), 0x81, np.uint8)  # -127
    c, acc = oracle.scaled_mm(oracle.FMT_INT8, aq, np.ones(1, np.float32), wq, np.ones(2, np.float32),
                              want_acc=True)
    assert acc[0, 0] == -127 * 127 * K
