"""Failure detection on the GPU without a fault: every device-side wait is
bounded.  A self-test kernel waits on an mbarrier that nothing arrives on; the
wait gives up after its limit, records QLIN_ERR_DEVICE_TIMEOUT and returns, the
host reads the status through qlin_sync_status, and the context stays usable
for the next GEMM."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_parity, bits_u16, gpu_gemm, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    from quantized_linear_layers_group_b200 import qlin

    assert qlin.qlin_sync_status() == qlin.QLIN_OK
    qlin.qlin_selftest_wait_timeout(20000)  # 20 ms
    assert qlin.qlin_sync_status() == qlin.QLIN_ERR_DEVICE_TIMEOUT
    assert qlin.qlin_sync_status() == qlin.QLIN_OK  # reading clears it
    # the context is intact: a GEMM right after still matches the oracle
    fmt = oracle.FMT_FP8
    g = torch.Generator().manual_seed(0)
    a = torch.randn(9, 512, generator=g).to(torch.bfloat16)
    w = (torch.randn(256, 512, generator=g) * 0.02).to(torch.bfloat16)
    aq, sa = gpu_quantize(fmt, a.cuda(), False)
    wq, sw = gpu_quantize(fmt, w.cuda(), True)
    c = gpu_gemm(fmt, aq, sa, wq, sw, None)
    assert qlin.qlin_sync_status() == qlin.QLIN_OK
    raq, rsa = oracle_quantize(fmt, a, False)
    rwq, rsw = oracle_quantize(fmt, w, True)
    assert_parity(fmt, bits_u16(c), oracle.scaled_mm(fmt, raq, rsa, rwq, rsw, None), "after timeout")


def test_timeout_on_a_side_stream_is_reported_there():
    from quantized_linear_layers_group_b200 import qlin

    s = torch.cuda.Stream()
    qlin.qlin_selftest_wait_timeout(5000, s)
    assert qlin.qlin_sync_status(s) == qlin.QLIN_ERR_DEVICE_TIMEOUT
    assert qlin.qlin_sync_status() == qlin.QLIN_OK


def test_workspace_tickets_are_rezeroed_after_a_timeout():
    # A GEMM whose bounded wait gives up can leave a Split-K ticket
    # half-counted.  Simulated on the host (no GPU fault): non-zero ticket
    # words are planted in a workspace, a timeout is raised by the self-test
    # kernel, and linear.check_device_status must report it and re-zero the
    # tickets, so the next Split-K call on that workspace is correct again.
    from quantized_linear_layers_group_b200 import linear, qlin

    fmt = oracle.FMT_FP8
    M, N, K = 16, 512, 1024
    g = torch.Generator().manual_seed(3)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    aq, sa = gpu_quantize(fmt, a.cuda(), False)
    wq, sw = gpu_quantize(fmt, w.cuda(), True)
    var, tile, S = qlin.QLIN_VAR_SWAPAB_SPLITK, 16, 4
    ws = linear.Workspace(qlin.qlin_scaled_mm_workspace_size(fmt, M, N, K, var, tile, S))
    ws.buf[: 4 * 64].view(torch.int32).fill_(1)  # a half-counted ticket on every tile of this shape
    qlin.qlin_selftest_wait_timeout(5000)
    with pytest.raises(qlin.QlinError) as e:
        linear.check_device_status(workspaces=[ws])
    assert e.value.status == qlin.QLIN_ERR_DEVICE_TIMEOUT
    assert int(ws.buf[:65536].count_nonzero()) == 0
    c = gpu_gemm(fmt, aq, sa, wq, sw, None, variant=var, tile_n=tile, k_segments=S, workspace=ws.buf)
    linear.check_device_status(workspaces=[ws])
    raq, rsa = oracle_quantize(fmt, a, False)
    rwq, rsw = oracle_quantize(fmt, w, True)
    assert_parity(fmt, bits_u16(c), oracle.scaled_mm(fmt, raq, rsa, rwq, rsw, None), "after ticket reset")
    assert int(ws.buf[:65536].count_nonzero()) == 0  # the call left its tickets at zero
