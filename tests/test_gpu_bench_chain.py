"""Parity of the configuration the benchmark times.

bench.HotPath issues, per M of a workload's sweep, the activation quantiser
and then the scaled GEMM, both with QLIN_PDL (the GEMM starts while the
quantiser runs and streams weights before its dependency wait), captured into
CUDA graphs back to back, with the weights rotating over many copies and the
activations over several sets.  A misplaced dependency wait would only show in
exactly this chained configuration, so these tests capture the graphs through
the benchmark's own code, poison every output, replay every graph of the
rotation, and compare the codes and scales bit-exact and C on sampled rows and
columns with the oracle (the parity bar: bit-exact for INT8, the FP8
tolerance otherwise).
"""
import os

import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from helpers import assert_parity, bits_u8, bits_u16, check_status, oracle_quantize

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TABLE = os.path.join(ROOT, "quantized_linear_layers_group_b200", "tables", "b200.qlt")


def _rows(M, k=16, seed=0):
    if M <= k:
        return np.arange(M)
    g = np.random.default_rng(seed + M)
    return np.array(sorted(set(g.choice(M, k - 3, replace=False).tolist()) | {0, M // 2, M - 1}))


def _cols(N, k=3072, seed=2):
    if N <= k:
        return None
    g = np.random.default_rng(seed)
    return np.array(sorted(set(g.choice(N, k - 256, replace=False).tolist()) | set(range(128)) |
                           set(range(N - 128, N))))


@pytest.mark.parametrize("name", bench.ALL_WORKLOADS)
def test_graph_captured_pdl_chain_matches_oracle(name):
    from quantized_linear_layers_group_b200 import qlin

    qlin.qlin_dispatch_table_load(TABLE)
    try:
        w = synth.WORKLOADS[name]
        dev = torch.device("cuda", 0)
        stream = torch.cuda.Stream(dev)
        with torch.cuda.stream(stream):
            hp = bench.HotPath(w, list(w.m_values), dev)
            graphs = hp.capture_graphs(stream)
            for M in hp.ms:
                hp.c[M].fill_(float("nan"))
                hp.a_q[M].fill_(0x7F)
                hp.s_a[M].fill_(float("nan"))
            torch.cuda.synchronize()
            for g in graphs + graphs[:1]:
                g.replay()
            torch.cuda.synchronize()
            check_status()
        wt = synth.weights(w, 0)
        b = synth.bias(w, 0)
        rwq, rsw = oracle_quantize(w.fmt, wt, True)
        ni = _cols(w.N)
        for M in hp.ms:
            a = synth.activations(w, M, seed=0)
            raq, rsa = oracle_quantize(w.fmt, a, False)
            assert np.array_equal(bits_u8(hp.a_q[M]), raq), f"{name} M={M}: activation codes"
            assert np.array_equal(hp.s_a[M].cpu().numpy().view(np.uint32), rsa.view(np.uint32)), \
                f"{name} M={M}: activation scales"
            mi = _rows(M)
            ref = oracle.scaled_mm(w.fmt, raq, rsa, rwq, rsw, b, m_idx=mi, n_idx=ni)
            sub = hp.c[M][torch.from_numpy(mi).cuda()]
            if ni is not None:
                sub = sub[:, torch.from_numpy(ni).cuda()]
            assert_parity(w.fmt, bits_u16(sub), ref, f"{name} M={M} (graph-captured PDL chain)")
        del graphs, hp
        torch.cuda.empty_cache()
    finally:
        qlin.qlin_dispatch_table_clear()


@pytest.mark.parametrize("name", ["fp8_attn", "int8_square", "mxfp8_attn"])
def test_end_to_end_step_returns_the_device_results(name):
    """The benchmark's end-to-end step (activations copied in on one stream,
    kernels on another, C copied out on a third, ordered by events, steps
    overlapping) must hand back, in pinned host memory, exactly the C that the
    graph-captured step computes from the same activations."""
    from quantized_linear_layers_group_b200 import qlin

    qlin.qlin_dispatch_table_load(TABLE)
    try:
        w = synth.WORKLOADS[name]
        dev = torch.device("cuda", 0)
        stream = torch.cuda.Stream(dev)
        with torch.cuda.stream(stream):
            hp = bench.HotPath(w, list(w.m_values), dev)
            hp.step(stream, act_set=0)  # activation set 0 holds the same inputs as the host copies
            torch.cuda.synchronize()
            want = {M: bits_u16(hp.c[M]).copy() for M in hp.ms}
            for _ in range(3):  # overlapping steps: copy-in of one step runs under the kernels of the last
                hp.step_e2e(stream)
            hp.e2e_join(stream)
            torch.cuda.synchronize()
            check_status()
        for M in hp.ms:
            got = hp.c_host[M].view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(got, want[M]), f"{name} M={M}: end-to-end C differs from the device step"
        del hp
        torch.cuda.empty_cache()
    finally:
        qlin.qlin_dispatch_table_clear()
