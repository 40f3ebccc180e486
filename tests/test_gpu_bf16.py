"""GPU parity of the bf16 batch-invariant matmul (qlin_matmul_bf16) against
the oracle's bf16 GEMM, the workload of the page "[Kernel][Perf] Add Hopper
(SM90) tuned config for batch-invariant persistent matmul".

Every variant (plain 128/256-column tiles, CTA pairs, Swap-AB 16/32/64,
Split-K through the workspace and through a cluster) is compared with the
oracle within the FP8 tolerance |d| <= 1e-2 |ref| + 1e-3 (fp32 accumulation
against a binary64 sum, then one bf16 rounding), with ragged M, N and K;
variants that share a K segmentation must agree bitwise, and the first rows of
C must not change with the batch size ("Test Plan": deterministic outputs
across batch sizes).  The five (N, K) shapes of the page's sweep are checked at
full size on sampled rows and columns.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_fp_parity, bits_u16, check_status

pytestmark = pytest.mark.gpu

PLAIN, SPLITK, SWAPAB, SWAPAB_SPLITK, PAIR = 1, 2, 3, 4, 5


def _mm(a, w, bias=None, variant=0, tile_n=0, S=0, flags=0):
    from quantized_linear_layers_group_b200 import qlin

    M, K = a.shape
    N = w.shape[0]
    c = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    nbytes = qlin.qlin_scaled_mm_workspace_size(qlin.QLIN_FMT_BF16, M, N, K, variant, tile_n, S)
    ws = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=a.device) if nbytes else None
    qlin.qlin_matmul_bf16(a, w, bias, c, ws, variant=variant, tile_n=tile_n, k_segments=S, flags=flags)
    return c


def _inputs(M, N, K, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16) if bias else None
    return a, w, b


CASES = [  # (variant, tile_n, S, flags)
    (PLAIN, 128, 1, 0), (PLAIN, 256, 1, 0), (PLAIN, 128, 4, 0), (PAIR, 256, 1, 0),
    (SWAPAB, 16, 1, 0), (SWAPAB, 32, 4, 0), (SWAPAB, 64, 1, 0),
    (SPLITK, 128, 4, 0), (SWAPAB_SPLITK, 16, 4, 0), (SWAPAB_SPLITK, 32, 2, 4),
]


@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (37, 528, 2048), (300, 1040, 1024)])
@pytest.mark.parametrize("case", CASES)
def test_variants_match_oracle(M, N, K, case):
    variant, tile_n, S, flags = case
    if variant in (SWAPAB, SWAPAB_SPLITK) and M > 64:
        pytest.skip("Swap-AB serves M <= 64")
    a, w, b = _inputs(M, N, K, seed=M + N + K)
    c = _mm(a.cuda(), w.cuda(), b.cuda(), variant, tile_n, S, flags)
    torch.cuda.synchronize()
    check_status()
    assert_fp_parity(bits_u16(c), oracle.gemm_bf16(a, w, b), f"bf16 M={M} N={N} K={K} {case}")


def test_variants_with_one_segmentation_agree_bitwise_and_rows_do_not_depend_on_M():
    N, K, S = 640, 2048, 4
    g = torch.Generator().manual_seed(5)
    fixed = torch.randn(16, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
    ref = None
    for M in (16, 1, 7, 33, 64, 129, 300):
        a = torch.randn(M, K, generator=g).to(torch.bfloat16)
        r = min(M, 16)
        a[:r] = fixed[:r]
        ad = a.cuda()
        outs = [bits_u16(_mm(ad, w, None, PLAIN, 128, S)), bits_u16(_mm(ad, w, None, SPLITK, 128, S))]
        if M <= 64:
            outs += [bits_u16(_mm(ad, w, None, SWAPAB_SPLITK, 16 if M <= 16 else 64, S)),
                     bits_u16(_mm(ad, w, None, SWAPAB, 64, S))]
        for o in outs[1:]:
            assert np.array_equal(o, outs[0]), f"M={M}: variants differ"
        if ref is None:
            ref = outs[0][:16].copy()
        assert np.array_equal(outs[0][:r], ref[:r]), f"M={M}: rows changed with the batch size"
    check_status()


@pytest.mark.parametrize("name", ["bf16_vocab", "bf16_down", "bf16_attn", "bf16_lm_head", "bf16_square"])
@pytest.mark.parametrize("M", [1, 64, 2048])
def test_full_size_shapes_auto_dispatch(name, M):
    from quantized_linear_layers_group_b200 import qlin
    import os

    table = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                         "quantized_linear_layers_group_b200", "tables", "b200.qlt")
    qlin.qlin_dispatch_table_load(table)
    try:
        w = synth.WORKLOADS[name]
        a = synth.activations(w, M, seed=0)
        wt = synth.weights(w, 0)
        c = _mm(a.cuda(), wt.cuda())
        torch.cuda.synchronize()
        check_status()
        g = np.random.default_rng(M)
        mi = np.unique(np.r_[0, M - 1, g.choice(M, min(M, 20), replace=False)])
        ni = None if w.N <= 4096 else np.unique(np.r_[np.arange(128), np.arange(w.N - 128, w.N),
                                                     g.choice(w.N, 3000, replace=False)])
        ref = oracle.gemm_bf16(a, wt, None, m_idx=mi, n_idx=ni)
        sub = c[torch.from_numpy(mi).cuda()]
        if ni is not None:
            sub = sub[:, torch.from_numpy(ni).cuda()]
        assert_fp_parity(bits_u16(sub), ref, f"{name} M={M}")
    finally:
        qlin.qlin_dispatch_table_clear()
