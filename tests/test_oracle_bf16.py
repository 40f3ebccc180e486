"""Pins for the oracle's bf16 GEMM (the matmul of the page "[Kernel][Perf] Add
Hopper (SM90) tuned config for batch-invariant persistent matmul", section
"Summary": bf16 activations [M, K] times bf16 weights [N, K], fp32
accumulation, bf16 out).

Definition: C[m,n] = bf16( fp32( sum_k a[m,k] w[n,k] ) + bias[n] ).

Pins: exact rationals on tiny inputs (the exact sum rounded to binary32 by a
rounding routine written from the definition, then the bias and the bf16
rounding); a float64 library matmul; closed forms (one-hot, constant rows);
the sampled-index path against the dense one; row independence.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from test_oracle_epilogue_order import bf16_frac, rn32, rn_bf16


def _bf(x):
    return x.to(torch.bfloat16)


def _frac_bf16(t):
    return [Fraction(float(v)) for v in t.float().reshape(-1).tolist()]


def test_tiny_exact_rationals():
    g = torch.Generator().manual_seed(11)
    M, N, K = 3, 16, 128
    a = _bf(torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g)))
    w = _bf(torch.randn(N, K, generator=g) * 0.05)
    b = _bf(torch.randn(N, generator=g) * 0.1)
    c = oracle.gemm_bf16(a, w, b)
    fa = [_frac_bf16(a[m]) for m in range(M)]
    fw = [_frac_bf16(w[n]) for n in range(N)]
    fb = _frac_bf16(b)
    for m in range(M):
        for n in range(N):
            exact = sum(x * y for x, y in zip(fa[m], fw[n]))
            want = rn_bf16(rn32(rn32(exact) + fb[n]))
            # the binary64 k-order sum is within K * 2^-53 of the exact one; with
            # these magnitudes it rounds to the same binary32 value
            assert bf16_frac(c[m, n]) == want, (m, n)


def test_float64_library_matmul():
    g = torch.Generator().manual_seed(12)
    M, N, K = 9, 40, 512
    a = _bf(torch.randn(M, K, generator=g))
    w = _bf(torch.randn(N, K, generator=g) * 0.02)
    c = oracle.bf16_bits_to_f32(oracle.gemm_bf16(a, w)).astype(np.float64)
    ref = (a.double() @ w.double().T).numpy()
    ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(ref), 1e-30))[1] - 8)
    assert np.all(np.abs(c - ref) <= ulp)


def test_closed_forms():
    K = 256
    # one-hot: a[1, 200] = 3, w[5, 200] = -0.5, everything else 0
    a = torch.zeros(2, K, dtype=torch.bfloat16)
    w = torch.zeros(8, K, dtype=torch.bfloat16)
    a[1, 200] = 3.0
    w[5, 200] = -0.5
    c = oracle.bf16_bits_to_f32(oracle.gemm_bf16(a, w))
    assert c[1, 5] == -1.5 and np.count_nonzero(c) == 1
    # constant rows: C = K * a * w exactly; bias added after
    a = torch.full((3, K), 0.25, dtype=torch.bfloat16)
    w = torch.full((4, K), -2.0, dtype=torch.bfloat16)
    b = torch.tensor([1.0, 0.0, -1.0, 64.0], dtype=torch.bfloat16)
    c = oracle.bf16_bits_to_f32(oracle.gemm_bf16(a, w, b))
    assert np.array_equal(c, np.broadcast_to(np.float32(K * 0.25 * -2.0) + b.float().numpy(), (3, 4)))


def test_sampled_indices_and_row_independence():
    g = torch.Generator().manual_seed(13)
    a = _bf(torch.randn(20, 256, generator=g))
    w = _bf(torch.randn(130, 256, generator=g) * 0.02)
    b = _bf(torch.randn(130, generator=g) * 0.1)
    dense = oracle.gemm_bf16(a, w, b)
    mi, ni = np.array([19, 0, 7]), np.array([129, 0, 64, 5])
    assert np.array_equal(oracle.gemm_bf16(a, w, b, m_idx=mi, n_idx=ni), dense[np.ix_(mi, ni)])
    assert np.array_equal(oracle.gemm_bf16(a[:5].contiguous(), w, b), dense[:5])
