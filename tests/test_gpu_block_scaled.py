"""GPU parity of the block-scaled formats (MXFP8, NVFP4) against the oracle.

NVFP4 is listed among vLLM's linear-layer formats on the page "Helion in vLLM:
A Unified Route to Tunable Linear Kernels" (introduction); both formats follow
their public definitions (readings in ``oracle/qlin_oracle.c``).

  - quantisers: codes and scale factors bit-exact against the oracle, over
    ragged row counts, strided input, zero / negative-zero / subnormal /
    saturating blocks and a wide spread of block magnitudes;
  - GEMM (tcgen05 block-scaled MMA, scale factors in TMEM): on the oracle's
    codes and scales, within |d| <= 1e-2 |ref| + 1e-3 of the oracle's GEMM,
    for plain, Split-K and Swap-AB (32 / 64) tiles, ragged M and N, with and
    without bias; every variant with the same K segmentation bitwise equal;
    AUTO dispatch (Swap-AB at small M, plain above) batch-invariant: the first
    rows of C do not change with M;
  - the chain (GPU quantiser -> GPU GEMM) at the attention-projection shape
    N = 4096, K = 2048, sampled rows against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import (assert_fp_parity, bits_u8, bits_u16, check_status, gpu_block_scaled_mm, sf_tile, sf_untile)

pytestmark = pytest.mark.gpu

MX, NV = oracle.FMT_MXFP8, oracle.FMT_NVFP4


def _q():
    from quantized_linear_layers_group_b200 import qlin

    return qlin


def _wide(rows, cols, seed, spread=30):
    """bf16 rows whose 16-element blocks span 2^-spread .. 2^spread, with
    outliers, an all-zero block, a negative-zero block and subnormals."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    mag = torch.exp2(torch.randint(-spread, spread + 1, (rows, cols // 16), generator=g).float())
    x = x * mag.repeat_interleave(16, dim=1)
    if rows > 2 and cols >= 64:
        x[0, 7] *= 900.0
        x[1, 16:32] = 0.0
        x[2, 32:64] = -0.0
    xb = x.to(torch.bfloat16)
    if rows > 3 and cols >= 128:
        bits = xb.view(torch.int16)
        bits[3, 96:128] = torch.arange(1, 33, dtype=torch.int16)   # bf16 subnormals
    return xb


def _gpu_quantize(fmt, x_dev, g=None):
    qlin = _q()
    rows, cols = x_dev.shape
    qcols = cols // 2 if fmt == NV else cols
    q = torch.empty(rows, qcols, dtype=torch.uint8, device="cuda")
    sf = torch.zeros(qlin.block_scaled_sf_bytes(fmt, rows, cols), dtype=torch.uint8, device="cuda")
    gt = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
    qlin.qlin_quantize_block_scaled(fmt, x_dev, q, sf, gt)
    return q, sf, gt


def _nsf(fmt, cols):
    return cols // (16 if fmt == NV else 32)


@pytest.mark.parametrize("rows,cols", [(1, 128), (5, 384), (130, 256), (300, 2048), (64, 4096)])
def test_mxfp8_quantiser_bit_exact(rows, cols):
    x = _wide(rows, cols, seed=rows + cols)
    q, sf, _ = _gpu_quantize(MX, x.cuda())
    torch.cuda.synchronize()
    check_status()
    rq, rsf = oracle.quantize_mxfp8(x)
    assert np.array_equal(bits_u8(q), rq)
    assert np.array_equal(sf_untile(bits_u8(sf), rows, _nsf(MX, cols)), rsf)


@pytest.mark.parametrize("rows,cols,g", [(1, 128, 1.0), (5, 384, 0.0123), (130, 256, 3.1e-7), (300, 2048, 0.5),
                                         (64, 4096, 448.0)])
def test_nvfp4_quantiser_bit_exact(rows, cols, g):
    x = _wide(rows, cols, seed=7 * rows + cols, spread=12)
    g = float(np.float32(g))
    q, sf, _ = _gpu_quantize(NV, x.cuda(), g)
    torch.cuda.synchronize()
    check_status()
    rq, rsf = oracle.quantize_nvfp4(x, g)
    assert np.array_equal(bits_u8(q), rq)
    assert np.array_equal(sf_untile(bits_u8(sf), rows, _nsf(NV, cols)), rsf)


def test_quantisers_read_strided_rows():
    qlin = _q()
    rows, cols, ld = 40, 256, 384
    big = _wide(rows, ld, seed=3)
    xs = big.cuda()[:, :cols]
    for fmt, g in ((MX, None), (NV, 0.01)):
        qcols = cols // 2 if fmt == NV else cols
        q = torch.empty(rows, qcols, dtype=torch.uint8, device="cuda")
        sf = torch.zeros(qlin.block_scaled_sf_bytes(fmt, rows, cols), dtype=torch.uint8, device="cuda")
        gt = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
        qlin.qlin_quantize_block_scaled(fmt, xs, q, sf, gt, ld_x=ld)
        torch.cuda.synchronize()
        rq, rsf = (oracle.quantize_mxfp8(big[:, :cols].contiguous()) if fmt == MX
                   else oracle.quantize_nvfp4(big[:, :cols].contiguous(), np.float32(g)))
        assert np.array_equal(bits_u8(q), rq)
        assert np.array_equal(sf_untile(bits_u8(sf), rows, _nsf(fmt, cols)), rsf)
    check_status()


# ------------------------------------------------------------------- GEMM
def _operands(fmt, M, N, K, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g)
    a[:, torch.randperm(K, generator=g)[: max(1, K // 100)]] *= 20.0          # outlier channels
    a = a.to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16) if bias else None
    if fmt == MX:
        aq, asf = oracle.quantize_mxfp8(a)
        wq, wsf = oracle.quantize_mxfp8(w)
        ga = gw = None
    else:
        ga = float(np.float32(a.float().abs().max() / 2688.0))
        gw = float(np.float32(w.float().abs().max() / 2688.0))
        aq, asf = oracle.quantize_nvfp4(a, ga)
        wq, wsf = oracle.quantize_nvfp4(w, gw)
    return a, w, b, aq, asf, wq, wsf, ga, gw


def _dev_ops(fmt, aq, asf, wq, wsf, ga, gw, b):
    t = lambda v: torch.from_numpy(np.ascontiguousarray(v)).cuda()
    gad = None if ga is None else torch.tensor([ga], dtype=torch.float32, device="cuda")
    gwd = None if gw is None else torch.tensor([gw], dtype=torch.float32, device="cuda")
    return (t(aq), t(sf_tile(asf)), t(wq), t(sf_tile(wsf)), gad, gwd, None if b is None else b.cuda())


def _ref(fmt, aq, asf, wq, wsf, ga, gw, b, m_idx=None):
    return oracle.gemm_block_scaled(fmt, aq, asf, wq, wsf, 1.0 if ga is None else ga, 1.0 if gw is None else gw,
                                    bias=b, m_idx=m_idx)


@pytest.mark.parametrize("fmt", [MX, NV], ids=["mxfp8", "nvfp4"])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (29, 384, 1024), (64, 272, 768), (77, 384, 1024),
                                   (300, 272, 768), (129, 128, 2048)])
def test_gemm_matches_oracle(fmt, M, N, K):
    if fmt == NV and K % 256:
        K = 1024
    qlin = _q()
    a, w, b, aq, asf, wq, wsf, ga, gw = _operands(fmt, M, N, K, seed=M + N + K, bias=(M % 2 == 1))
    d = _dev_ops(fmt, aq, asf, wq, wsf, ga, gw, b)
    ref = _ref(fmt, aq, asf, wq, wsf, ga, gw, b)
    c_plain = gpu_block_scaled_mm(fmt, d[0], d[1], d[2], d[3], d[6], d[4], d[5], variant=qlin.QLIN_VAR_PLAIN,
                                  k_segments=1)
    torch.cuda.synchronize()
    check_status()
    assert_fp_parity(bits_u16(c_plain), ref, f"fmt {fmt} plain S=1")
    kblocks = (K // 2 if fmt == NV else K) // 128
    run = lambda v, t, S: bits_u16(gpu_block_scaled_mm(fmt, d[0], d[1], d[2], d[3], d[6], d[4], d[5], variant=v,
                                                       tile_n=t, k_segments=S))
    swap_tiles = [t for t in (32, 64) if M <= t]  # Swap-AB: one activation tile
    for t in swap_tiles:  # bitwise the plain tile's result
        assert np.array_equal(run(qlin.QLIN_VAR_SWAPAB, t, 1), bits_u16(c_plain)), f"Swap-AB {t} S=1"
    for S in (2, 4):
        if kblocks % S:
            continue
        cp = run(qlin.QLIN_VAR_PLAIN, 128, S)
        assert_fp_parity(cp, ref, f"fmt {fmt} S={S}")
        for v, t in [(qlin.QLIN_VAR_SPLITK, 128)] + [(qlin.QLIN_VAR_SWAPAB, t) for t in swap_tiles] + \
                [(qlin.QLIN_VAR_SWAPAB_SPLITK, t) for t in swap_tiles]:
            assert np.array_equal(run(v, t, S), cp), f"S={S}: variant {v} tile {t} differs from plain"
    check_status()


@pytest.mark.parametrize("fmt", [MX, NV], ids=["mxfp8", "nvfp4"])
def test_gemm_rows_do_not_depend_on_M(fmt):
    N, K = 384, 1024
    a, w, b, aq, asf, wq, wsf, ga, gw = _operands(fmt, 300, N, K, seed=11)
    first = None
    for M in (16, 1, 7, 130, 300):
        d = _dev_ops(fmt, aq[:M], asf[:M], wq, wsf, ga, gw, b)
        c = bits_u16(gpu_block_scaled_mm(fmt, d[0], d[1], d[2], d[3], d[6], d[4], d[5]))
        torch.cuda.synchronize()
        r = min(M, 16)
        if first is None:
            first = c[:16].copy()
        assert np.array_equal(c[:r], first[:r]), f"M={M}"
    check_status()


@pytest.mark.parametrize("fmt", [MX, NV], ids=["mxfp8", "nvfp4"])
@pytest.mark.parametrize("M", [1, 2048])
def test_quantise_then_gemm_attention_projection(fmt, M):
    """Full attention-projection shape: GPU quantiser then GPU GEMM, sampled
    rows (all N columns) against the oracle on the oracle's own codes."""
    qlin = _q()
    N, K = 4096, 2048
    g = torch.Generator().manual_seed(M)
    a = torch.randn(M, K, generator=g)
    a[:, torch.randperm(K, generator=g)[: K // 100]] *= 20.0
    a = a.to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    ga = float(np.float32(a.float().abs().max() / 2688.0)) if fmt == NV else None
    gw = float(np.float32(w.float().abs().max() / 2688.0)) if fmt == NV else None
    aq, asf, gad = _gpu_quantize(fmt, a.cuda(), ga)
    wq, wsf, gwd = _gpu_quantize(fmt, w.cuda(), gw)
    c = gpu_block_scaled_mm(fmt, aq, asf, wq, wsf, b.cuda(), gad, gwd, flags=qlin.QLIN_PDL)
    torch.cuda.synchronize()
    check_status()
    rows = np.unique(np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 6)])
    if fmt == MX:
        raq, rasf = oracle.quantize_mxfp8(a[rows].contiguous())
        rwq, rwsf = oracle.quantize_mxfp8(w)
    else:
        raq, rasf = oracle.quantize_nvfp4(a[rows].contiguous(), ga)
        rwq, rwsf = oracle.quantize_nvfp4(w, gw)
    assert np.array_equal(bits_u8(aq)[rows], raq)
    ref = _ref(fmt, raq, rasf, rwq, rwsf, ga, gw, b)
    assert_fp_parity(bits_u16(c)[rows], ref, f"fmt {fmt} M={M}")


@pytest.mark.parametrize("fmt", [MX, NV], ids=["mxfp8", "nvfp4"])
def test_shipped_table_dispatch_is_batch_invariant(fmt):
    """The shipped dispatch table's entries for the attention projection
    (Swap-AB Split-K at small M, plain tiles above, one K segmentation):
    the first 16 rows of C are bitwise the same at every M, and match the
    oracle."""
    import os

    qlin = _q()
    table = os.path.join(os.path.dirname(qlin.__file__), "tables", "b200.qlt")
    qlin.qlin_dispatch_table_load(table)
    try:
        N, K = 4096, 2048
        a, w, b, aq, asf, wq, wsf, ga, gw = _operands(fmt, 600, N, K, seed=21)
        segs = {qlin.qlin_dispatch_query(fmt, M, N, K)["k_segments"] for M in (1, 64, 128, 600)}
        assert len(segs) == 1 and all(qlin.qlin_dispatch_query(fmt, M, N, K)["from_table"] for M in (1, 600))
        first = None
        for M in (16, 1, 5, 33, 64, 100, 600):
            d = _dev_ops(fmt, aq[:M], asf[:M], wq, wsf, ga, gw, b)
            c = bits_u16(gpu_block_scaled_mm(fmt, d[0], d[1], d[2], d[3], d[6], d[4], d[5], flags=qlin.QLIN_PDL))
            torch.cuda.synchronize()
            r = min(M, 16)
            if first is None:
                first = c[:16].copy()
                assert_fp_parity(first, _ref(fmt, aq[:16], asf[:16], wq, wsf, ga, gw, b), f"fmt {fmt}")
            assert np.array_equal(c[:r], first[:r]), f"M={M}"
        check_status()
    finally:
        qlin.qlin_dispatch_table_clear()
