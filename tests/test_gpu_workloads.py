"""GPU parity at the full workload sizes, through the C ABI with the dispatch
table loaded (the configuration bench.py times).

Every quantised operand is compared bit-exact with the oracle's; GEMM outputs
are compared on all columns of a row sample (plus a column sample for the
151936-wide lm_head), where the oracle computes each entry on its own."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_parity, bits_u8, bits_u16, check_status, gpu_gemm, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TABLE = os.path.join(ROOT, "quantized_linear_layers_group_b200", "tables", "b200.qlt")


@pytest.fixture(scope="module", autouse=True)
def table():
    from quantized_linear_layers_group_b200 import qlin

    qlin.qlin_dispatch_table_load(TABLE)
    yield
    qlin.qlin_dispatch_table_clear()


class Weights:
    """Quantised weight on both sides (checked bit-exact), cached per workload."""
    cache = {}

    @classmethod
    def get(cls, name):
        if name not in cls.cache:
            w = synth.WORKLOADS[name]
            wt = synth.weights(w, 0)
            b = synth.bias(w, 0)
            wq, sw = gpu_quantize(w.fmt, wt.cuda(), True)
            rwq, rsw = oracle_quantize(w.fmt, wt, True)
            torch.cuda.synchronize()
            assert np.array_equal(bits_u8(wq), rwq), f"{name}: W codes differ"
            assert np.array_equal(sw.cpu().numpy().view(np.uint32), rsw.view(np.uint32)), f"{name}: s_w differ"
            cls.cache[name] = (wq, sw, rwq, rsw, b, None if b is None else b.cuda())
        return cls.cache[name]


def _row_sample(M, k=24, seed=0):
    if M <= k:
        return np.arange(M)
    g = np.random.default_rng(seed + M)
    pick = set(g.choice(M, k - 4, replace=False).tolist()) | {0, 1, M - 2, M - 1}
    return np.array(sorted(pick))


def _col_sample(N, k=4096, seed=1):
    if N <= k:
        return None
    g = np.random.default_rng(seed)
    pick = set(g.choice(N, k - 256, replace=False).tolist()) | set(range(N - 128, N)) | set(range(128))
    return np.array(sorted(pick))


def run_workload(name, M, seed=0):
    w = synth.WORKLOADS[name]
    wq, sw, rwq, rsw, b, bd = Weights.get(name)
    a = synth.activations(w, M, seed=seed)
    aq, sa = gpu_quantize(w.fmt, a.cuda(), False)
    c = gpu_gemm(w.fmt, aq, sa, wq, sw, bd)
    torch.cuda.synchronize()
    check_status()
    raq, rsa = oracle_quantize(w.fmt, a, False)
    assert np.array_equal(bits_u8(aq), raq), f"{name} M={M}: activation codes differ"
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), rsa.view(np.uint32)), f"{name} M={M}: s_a differ"
    mi = _row_sample(M)
    ni = _col_sample(w.N)
    ref = oracle.scaled_mm(w.fmt, raq, rsa, rwq, rsw, b, m_idx=mi, n_idx=ni)
    sub = c[torch.from_numpy(mi).cuda()]
    if ni is not None:
        sub = sub[:, torch.from_numpy(ni).cuda()]
    got = bits_u16(sub)
    assert_parity(w.fmt, got, ref, f"{name} M={M}")
    return c


def test_int8_smoke_full():
    # INT8 W8A8 M=16 N=K=2048: every output bit-exact
    run_workload("int8_smoke", 16)


@pytest.mark.parametrize("M", synth.WORKLOADS["fp8_attn"].m_values)
def test_fp8_attention_projection(M):
    run_workload("fp8_attn", M)


@pytest.mark.parametrize("M", synth.WORKLOADS["fp8_block_down"].m_values)
def test_block_fp8_down_projection(M):
    run_workload("fp8_block_down", M)


@pytest.mark.parametrize("M", synth.WORKLOADS["lm_head"].m_values)
def test_lm_head(M):
    run_workload("lm_head", M)


def test_lm_head_m1_every_column():
    w = synth.WORKLOADS["lm_head"]
    wq, sw, rwq, rsw, b, bd = Weights.get("lm_head")
    a = synth.activations(w, 1, seed=7)
    aq, sa = gpu_quantize(w.fmt, a.cuda(), False)
    c = gpu_gemm(w.fmt, aq, sa, wq, sw, bd)
    raq, rsa = oracle_quantize(w.fmt, a, False)
    ref = oracle.scaled_mm(w.fmt, raq, rsa, rwq, rsw, b)
    assert_parity(w.fmt, bits_u16(c), ref, "lm_head M=1 all columns")


@pytest.mark.parametrize("M", [1, 37, 64, 333, 2048])
def test_fp8_vocab_and_int8_square(M):
    run_workload("fp8_vocab", M)
    run_workload("int8_square", M)
