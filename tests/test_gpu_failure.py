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
