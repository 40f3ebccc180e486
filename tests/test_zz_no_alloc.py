"""The no-allocation GEMM entry point (qlin_scaled_mm_noalloc).

Some callers cannot allocate device memory: a kernel plugin inside a serving
engine that owns the whole memory pool may not call cudaMalloc behind the
engine's back.  They cannot pass a Split-K workspace, so this entry point takes
its Split-K scratch from a fixed device array inside the library.  These tests
check, through the C ABI, that it gives bitwise the same output as
qlin_scaled_mm with a caller workspace (Split-K reduces in a fixed order, so
the two must agree bit for bit, which is within every tolerance the other
tests use), and that both are within the parity bar of the oracle, on two
calls in a row (the second call reuses the array the first one left dirty);
that the cluster Split-K mode is accepted; that M = 0 is a no-op; and that a
configuration needing more scratch than the fixed maximum is refused.  This
file is collected last, so that a run that stops at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_parity, bits_u16, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu


def _operands(fmt, M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = None if fmt == oracle.FMT_FP8_BLOCK else (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    a_q, s_a = gpu_quantize(fmt, a.cuda(), False)
    w_q, s_w = gpu_quantize(fmt, w.cuda(), True)
    ref = oracle_quantize(fmt, a, False) + oracle_quantize(fmt, w, True)
    return a_q, s_a, w_q, s_w, None if b is None else b.cuda(), b, ref


def _oracle_c(fmt, ref, b, rows):
    raq, rsa, rwq, rsw = ref
    return oracle.scaled_mm(fmt, raq, rsa, rwq, rsw, b, m_idx=rows)


@pytest.mark.parametrize("flags_name", ["none", "cluster"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(flags_name):
    from quantized_linear_layers_group_b200 import qlin

    flags = qlin.QLIN_SPLITK_CLUSTER if flags_name == "cluster" else 0
    # both calls use a Split-K variant, so both go through the scratch array
    # (with the cluster flag the Swap-AB call reduces in a cluster instead)
    calls = [(oracle.FMT_FP8, 16, 4096, 2048, qlin.QLIN_VAR_SWAPAB_SPLITK, 16, 4),
             (oracle.FMT_INT8, 200, 512, 768, qlin.QLIN_VAR_SPLITK, 128, 3),
             (oracle.FMT_FP8_BLOCK, 40, 1024, 1536, qlin.QLIN_VAR_SWAPAB_SPLITK, 64, 3)]
    for i, (fmt, M, N, K, var, tile, S) in enumerate(calls):
        a_q, s_a, w_q, s_w, b_dev, b, ref = _operands(fmt, M, N, K, seed=100 + i)
        nbytes = qlin.qlin_scaled_mm_workspace_size(fmt, M, N, K, var, tile, S)
        assert 0 < nbytes <= qlin.QLIN_NOALLOC_SCRATCH_BYTES
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        want = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        qlin.qlin_scaled_mm(fmt, a_q, s_a, w_q, s_w, b_dev, want, ws, variant=var, tile_n=tile, k_segments=S)
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        qlin.qlin_scaled_mm_noalloc(fmt, a_q, s_a, w_q, s_w, b_dev, out, variant=var, tile_n=tile, k_segments=S,
                                    flags=flags)
        torch.cuda.synchronize()
        assert qlin.qlin_sync_status() == 0
        assert np.array_equal(bits_u16(out), bits_u16(want)), f"noalloc call {i}: not bitwise equal"
        rows = np.unique(np.r_[0, M - 1, np.arange(0, M, 7)])
        assert_parity(fmt, bits_u16(out)[rows], _oracle_c(fmt, ref, b, rows), f"noalloc call {i} vs oracle")


def test_noalloc_m0_is_a_noop():
    from quantized_linear_layers_group_b200 import qlin

    # M = 0 returns OK even for a configuration whose scratch need exceeds the maximum
    e = torch.empty(0, 2048, dtype=torch.uint8, device="cuda")
    w = torch.empty(16384, 2048, dtype=torch.uint8, device="cuda")
    s = torch.ones(16384, dtype=torch.float32, device="cuda")
    c = torch.empty(0, 16384, dtype=torch.bfloat16, device="cuda")
    qlin.qlin_scaled_mm_noalloc(oracle.FMT_FP8, e, s, w, s, None, c, variant=qlin.QLIN_VAR_SWAPAB_SPLITK,
                                tile_n=64, k_segments=8, M=0)


def test_noalloc_refuses_configurations_beyond_the_scratch_maximum():
    from quantized_linear_layers_group_b200 import qlin

    # Swap-AB + Split-K over 128 tiles of 128x64 with 8 segments needs 32 MiB
    M, N, K = 64, 16384, 2048
    need = qlin.qlin_scaled_mm_workspace_size(oracle.FMT_FP8, M, N, K, qlin.QLIN_VAR_SWAPAB_SPLITK, 64, 8)
    assert need > qlin.QLIN_NOALLOC_SCRATCH_BYTES
    a = torch.zeros(M, K, dtype=torch.uint8, device="cuda")
    w = torch.zeros(N, K, dtype=torch.uint8, device="cuda")
    s = torch.ones(max(M, N), dtype=torch.float32, device="cuda")
    c = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qlin.QlinError) as e:
        qlin.qlin_scaled_mm_noalloc(oracle.FMT_FP8, a, s, w, s, None, c, variant=qlin.QLIN_VAR_SWAPAB_SPLITK,
                                    tile_n=64, k_segments=8)
    assert e.value.status == qlin.QLIN_ERR_WORKSPACE
