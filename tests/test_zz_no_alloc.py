"""The no-allocation GEMM entry point (qlin_scaled_mm_noalloc).

Callers that cannot allocate device memory -- a plugin inside a serving engine
that owns the whole memory pool, or code running during CUDA graph capture --
use this entry point instead of passing a workspace; its Split-K scratch is a
fixed device array inside the library.  These tests check, through the C ABI,
that it gives the same output as qlin_scaled_mm with a caller workspace on two
calls in a row (the second call reuses the array the first one left dirty),
and that a configuration needing more scratch than the fixed maximum is
refused.  This file is collected last so that a run that stops at the first
failure has already run every other test.
"""
import pytest
import torch

import oracle
from helpers import assert_parity, bits_u16, gpu_quantize

pytestmark = pytest.mark.gpu


def _operands(fmt, M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16).cuda()
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
    b = None if fmt == oracle.FMT_FP8_BLOCK else (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16).cuda()
    a_q, s_a = gpu_quantize(fmt, a, False)
    w_q, s_w = gpu_quantize(fmt, w, True)
    return a_q, s_a, w_q, s_w, b


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    from quantized_linear_layers_group_b200 import qlin

    # both calls use a Split-K variant, so both go through the scratch array
    calls = [(oracle.FMT_FP8, 16, 4096, 2048, qlin.QLIN_VAR_SWAPAB_SPLITK, 16, 4),
             (oracle.FMT_INT8, 200, 512, 768, qlin.QLIN_VAR_SPLITK, 128, 3)]
    for i, (fmt, M, N, K, var, tile, S) in enumerate(calls):
        a_q, s_a, w_q, s_w, b = _operands(fmt, M, N, K, seed=100 + i)
        nbytes = qlin.qlin_scaled_mm_workspace_size(fmt, M, N, K, var, tile, S)
        assert 0 < nbytes <= qlin.QLIN_NOALLOC_SCRATCH_BYTES
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        qlin.qlin_scaled_mm(fmt, a_q, s_a, w_q, s_w, b, ref, ws, variant=var, tile_n=tile, k_segments=S)
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        qlin.qlin_scaled_mm_noalloc(fmt, a_q, s_a, w_q, s_w, b, out, variant=var, tile_n=tile, k_segments=S)
        torch.cuda.synchronize()
        assert qlin.qlin_sync_status() == 0
        assert_parity(fmt, bits_u16(out), bits_u16(ref), f"noalloc call {i}")


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
