"""Batch invariance (page "[Kernel][Perf] Add Hopper (SM90) tuned config for
batch-invariant persistent matmul", section "Test Plan": deterministic outputs
across batch sizes) and the seeded mixed serving stream.

The same first 16 token rows are embedded in batches of many sizes M; their
output rows must be bitwise identical to the M=16 result under the variant the
dispatch table picks for each M and under every forced variant that exists for
that M (with the shape's fixed K segmentation).  The mixed stream is 1000 seeded
calls across the five shapes with M mostly small, each checked against the
oracle on a sample of rows and columns."""
import os
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_parity, bits_u8, bits_u16, gpu_gemm, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TABLE = os.path.join(ROOT, "quantized_linear_layers_group_b200", "tables", "b200.qlt")

PLAIN, SPLITK, SWAPAB, SWAPAB_SPLITK, PAIR = 1, 2, 3, 4, 5
M_SET = [1, 2, 3, 5, 8, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 255, 256, 257, 511, 512, 700, 1023,
         1024, 1025, 2047, 2048]


@pytest.fixture(scope="module", autouse=True)
def table():
    from quantized_linear_layers_group_b200 import qlin

    qlin.qlin_dispatch_table_load(TABLE)
    yield
    qlin.qlin_dispatch_table_clear()


def _forced(fmt):
    out = [(PLAIN, 128), (SPLITK, 128), (SWAPAB, 16), (SWAPAB, 64), (SWAPAB_SPLITK, 32)]
    if fmt != oracle.FMT_FP8_BLOCK:
        out += [(PLAIN, 256), (SPLITK, 256), (PAIR, 256)]
    return out


@pytest.mark.parametrize("name", ["fp8_vocab", "int8_square"])
def test_first_rows_bitwise_identical_across_batch_sizes_and_variants(name):
    from quantized_linear_layers_group_b200 import qlin

    w = synth.WORKLOADS[name]
    wt = synth.weights(w, 0)
    wq, sw = gpu_quantize(w.fmt, wt.cuda(), True)
    fixed = synth.activations(w, 16, seed=42)
    S = qlin.qlin_dispatch_query(w.fmt, 16, w.N, w.K)["k_segments"]

    def run(M, variant=0, tile=0):
        a = synth.invariance_batch(w, M, fixed, seed=0)
        aq, sa = gpu_quantize(w.fmt, a.cuda(), False)
        c = gpu_gemm(w.fmt, aq, sa, wq, sw, None, variant, tile, S if variant else 0)
        return bits_u16(c[: min(M, 16)])

    ref = run(16)
    # the reference rows themselves match the oracle
    rwq, rsw = oracle_quantize(w.fmt, wt, True)
    raq, rsa = oracle_quantize(w.fmt, fixed, False)
    cols = np.arange(0, w.N, 7)
    assert_parity(w.fmt, ref[:, cols], oracle.scaled_mm(w.fmt, raq, rsa, rwq, rsw, None, n_idx=cols), name)
    checked = 0
    for M in M_SET:
        r = min(M, 16)
        got = run(M)
        assert np.array_equal(got, ref[:r]), f"{name}: AUTO differs at M={M}"
        for var, tile in _forced(w.fmt):
            try:
                got = run(M, var, tile)
            except qlin.QlinError:
                continue  # variant not offered for this shape / M
            assert np.array_equal(got, ref[:r]), f"{name}: variant {var} tile {tile} differs at M={M}"
            checked += 1
    assert checked > 50


def test_mixed_serving_stream():
    from quantized_linear_layers_group_b200 import qlin

    stream = synth.mixed_stream(1000, seed=0)
    prepared = {}
    gpu_time = 0.0
    roof_time = 0.0
    g = np.random.default_rng(3)
    for i, (name, M) in enumerate(stream):
        w = synth.WORKLOADS[name]
        if name not in prepared:
            wt = synth.weights(w, 0)
            wq, sw = gpu_quantize(w.fmt, wt.cuda(), True)
            rwq, rsw = oracle_quantize(w.fmt, wt, True)
            torch.cuda.synchronize()
            assert np.array_equal(bits_u8(wq), rwq)
            b = synth.bias(w, 0)
            prepared[name] = (wq, sw, rwq, rsw, b, None if b is None else b.cuda())
        wq, sw, rwq, rsw, b, bd = prepared[name]
        a = synth.activations(w, M, seed=10_000 + i)
        ad = a.cuda()
        aq, sa = gpu_quantize(w.fmt, ad, False)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        c = gpu_gemm(w.fmt, aq, sa, wq, sw, bd)
        torch.cuda.synchronize()
        gpu_time += time.perf_counter() - t0
        roof_time += max((M * w.K + w.N * w.K) / 6550.4e9, 2.0 * M * w.N * w.K / 2751.2e12)
        rows = np.unique(np.concatenate([[0, M - 1], g.integers(0, M, 2)]))
        cols = np.unique(np.concatenate([g.integers(0, w.N, 512), [w.N - 1]]))
        raq, rsa = oracle_quantize(w.fmt, a[torch.from_numpy(rows)], False)
        assert np.array_equal(bits_u8(aq)[rows], raq), f"call {i} {name} M={M}: codes differ"
        ref = oracle.scaled_mm(w.fmt, raq, rsa, rwq, rsw, b, n_idx=cols)
        sub = c[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()]
        assert_parity(w.fmt, bits_u16(sub), ref, f"call {i} {name} M={M}")
    assert qlin.qlin_sync_status() == 0
    print(f"mixed stream: 1000 calls, host-timed GPU time {gpu_time * 1e3:.1f} ms "
          f"(sum of rooflines {roof_time * 1e3:.2f} ms)")
