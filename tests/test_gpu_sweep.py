"""The offline sweep that writes the dispatch table, run on tiny shapes.

The page "Helion in vLLM: A Unified Route to Tunable Linear Kernels" makes the
GEMM variant part of the per-shape tuning ("Algorithm choice becomes part of
tuning", in "What the integration changes"), and the page "[Kernel][Perf] Add
Hopper (SM90) tuned config for batch-invariant persistent matmul" keys such
tables by device and M bucket and requires outputs that do not change with the
batch size ("Test Plan").  This test builds the sweep, runs it in its quick
mode (buckets 1, 16, 256) on three small shapes, loads the table it writes and
checks the rules that keep batch invariance in it: one K segmentation per
(format, N, K); every selected variant bitwise equal to the plain variant with
that segmentation; and, under AUTO dispatch through the table, the first 16
rows of C bitwise identical at every M (including M between and beyond the
buckets), and within the parity bar of the oracle.
"""
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_parity, bits_u16, check_status, gpu_gemm, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu

SHAPES = [(oracle.FMT_FP8, 512, 1024), (oracle.FMT_FP8_BLOCK, 256, 768), (oracle.FMT_INT8, 256, 512)]
NAMES = {oracle.FMT_INT8: "int8", oracle.FMT_FP8: "fp8", oracle.FMT_FP8_BLOCK: "fp8_block"}


def _read_table(path):
    entries = []
    with open(path) as f:
        for line in f:
            if line.startswith("entry"):
                t = line.split("#")[0].split()
                entries.append((t[1], int(t[2]), int(t[3]), int(t[4]), t[5], int(t[6]), int(t[7])))
    return entries


@pytest.fixture(scope="module")
def table(tmp_path_factory):
    from quantized_linear_layers_group_b200 import build, qlin

    exe = build.build_sweep()
    out = str(tmp_path_factory.mktemp("sweep") / "tiny.qlt")
    args = [exe, "--quick", out] + [f"{NAMES[f]}:{n}:{k}" for f, n, k in SHAPES]
    r = subprocess.run(args, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    qlin.qlin_dispatch_table_load(out)
    yield out, r.stdout
    qlin.qlin_dispatch_table_clear()


def test_table_has_one_segmentation_per_shape_and_every_bucket(table):
    path, log = table
    entries = _read_table(path)
    for fmt, N, K in SHAPES:
        mine = [e for e in entries if (e[0], e[1], e[2]) == (NAMES[fmt], N, K)]
        assert sorted(e[3] for e in mine) == [1, 16, 256], mine
        if fmt != oracle.FMT_INT8:  # INT8 sums are exact: its segmentation is free per bucket
            assert len({e[6] for e in mine}) == 1, mine
    assert "S=" in log  # the sweep printed its per-segmentation totals


def test_selected_variants_equal_plain_with_the_same_segmentation(table):
    from quantized_linear_layers_group_b200 import qlin

    path, _ = table
    var_of = {v: k for k, v in qlin.VARIANT_NAMES.items()}
    for fmt_s, N, K, m_max, var_s, tile, S in _read_table(path):
        fmt = {v: k for k, v in NAMES.items()}[fmt_s]
        M = m_max
        g = torch.Generator().manual_seed(N + K + M)
        a = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
        w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
        aq, sa = gpu_quantize(fmt, a, False)
        wq, sw = gpu_quantize(fmt, w, True)
        c_sel = gpu_gemm(fmt, aq, sa, wq, sw, None, variant=var_of[var_s], tile_n=tile, k_segments=S)
        c_pl = gpu_gemm(fmt, aq, sa, wq, sw, None, variant=qlin.QLIN_VAR_PLAIN, tile_n=128, k_segments=S)
        torch.cuda.synchronize()
        assert np.array_equal(bits_u16(c_sel), bits_u16(c_pl)), (fmt_s, N, K, M, var_s, tile, S)
    check_status()


@pytest.mark.parametrize("shape", SHAPES)
def test_auto_dispatch_through_the_table_is_batch_invariant(table, shape):
    fmt, N, K = shape
    g = torch.Generator().manual_seed(7)
    fixed = torch.randn(16, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    wq, sw = gpu_quantize(fmt, w.cuda(), True)
    rwq, rsw = oracle_quantize(fmt, w, True)
    first = None
    for M in (16, 1, 5, 17, 100, 256, 300):      # M = 16 first: its rows are the reference
        a = torch.randn(M, K, generator=g).to(torch.bfloat16)
        r = min(M, 16)
        a[:r] = fixed[:r]
        aq, sa = gpu_quantize(fmt, a.cuda(), False)
        c = bits_u16(gpu_gemm(fmt, aq, sa, wq, sw, None))
        if first is None:
            first = c[:16].copy()
        assert np.array_equal(c[:r], first[:r]), f"M={M}: rows 0..{r - 1} changed with the batch size"
        raq, rsa = oracle_quantize(fmt, a, False)
        rows = np.arange(min(M, 20))
        assert_parity(fmt, c[rows], oracle.scaled_mm(fmt, raq, rsa, rwq, rsw, None, m_idx=rows), f"M={M}")
    check_status()
