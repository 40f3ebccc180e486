"""GPU parity of the scaled GEMM (every format x variant) against the oracle.

INT8: bf16 output and int32 accumulators bit-exact.  FP8 / Block-FP8:
|C_gpu - C_ref| <= 1e-2 |C_ref| + 1e-3 elementwise.  The GPU operands come
from the GPU quantisers and are first checked bit-exact against the oracle's,
so these are end-to-end checks of the hot path.  Sizes span several tiles in
both dimensions with ragged tails."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_parity, bits_u8, bits_u16, check_status, gpu_gemm, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu

PLAIN, SPLITK, SWAPAB, SWAPAB_SPLITK, PAIR = 1, 2, 3, 4, 5
FMTS = [oracle.FMT_INT8, oracle.FMT_FP8, oracle.FMT_FP8_BLOCK]


def _problem(fmt, M, N, K, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g))).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16) if bias and fmt != oracle.FMT_FP8_BLOCK else None
    return a, w, b


class Prepared:
    """Quantised operands on both sides, checked bit-exact against each other."""

    def __init__(self, fmt, a, w, b):
        self.fmt = fmt
        self.a, self.w, self.b = a, w, b
        self.a_q, self.s_a = gpu_quantize(fmt, a.cuda(), False)
        self.w_q, self.s_w = gpu_quantize(fmt, w.cuda(), True)
        self.b_dev = None if b is None else b.cuda()
        self.ra_q, self.rs_a = oracle_quantize(fmt, a, False)
        self.rw_q, self.rs_w = oracle_quantize(fmt, w, True)
        torch.cuda.synchronize()
        assert np.array_equal(bits_u8(self.a_q), self.ra_q)
        assert np.array_equal(self.s_a.cpu().numpy().view(np.uint32), self.rs_a.view(np.uint32))
        assert np.array_equal(bits_u8(self.w_q), self.rw_q)
        assert np.array_equal(self.s_w.cpu().numpy().view(np.uint32), self.rs_w.view(np.uint32))

    def reference(self, m_idx=None, n_idx=None, want_acc=False):
        return oracle.scaled_mm(self.fmt, self.ra_q, self.rs_a, self.rw_q, self.rs_w, self.b, m_idx=m_idx,
                                n_idx=n_idx, want_acc=want_acc)

    def run(self, variant=0, tile_n=0, k_segments=0, out_i32=False, flags=0):
        c = gpu_gemm(self.fmt, self.a_q, self.s_a, self.w_q, self.s_w, self.b_dev, variant, tile_n, k_segments,
                     out_i32, flags=flags)
        torch.cuda.synchronize()
        return c


def _variants(fmt, K):
    """(variant, tile_n, k_segments) combinations that exist for a format."""
    kb = K // 128
    segs = [s for s in (1, 2, 3, 4) if kb % s == 0]
    out = []
    for s in segs:
        out.append((PLAIN, 128, s))
        if fmt != oracle.FMT_FP8_BLOCK and (fmt == oracle.FMT_INT8 or s == 1):
            out.append((PLAIN, 256, s))
            out.append((PAIR, 256, s))
        for t in (16, 32, 64):
            out.append((SWAPAB, t, s))
        if s > 1:
            out.append((SPLITK, 128, s))
            if fmt != oracle.FMT_FP8_BLOCK:
                out.append((SPLITK, 256, s))
            for t in (16, 64):
                out.append((SWAPAB_SPLITK, t, s))
    return out


SHAPES = [(1, 256, 256), (7, 384, 384), (65, 512, 1024), (130, 384, 512), (300, 640, 768)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_every_variant_matches_oracle(fmt, M, N, K):
    p = Prepared(fmt, *_problem(fmt, M, N, K, seed=M * 7 + N + K + fmt))
    ref = p.reference()
    for var, tile, s in _variants(fmt, K):
        c = p.run(var, tile, s)
        assert_parity(fmt, bits_u16(c), ref, f"fmt={fmt} M={M} N={N} K={K} var={var} tile={tile} S={s}")
    check_status()


@pytest.mark.parametrize("M,N,K", [(5, 272, 384), (129, 400, 256), (64, 1024, 2048)])
def test_int8_accumulators_bit_exact(M, N, K):
    fmt = oracle.FMT_INT8
    p = Prepared(fmt, *_problem(fmt, M, N, K, seed=11))
    _, acc = p.reference(want_acc=True)
    for var, tile, s in _variants(fmt, K):
        c = p.run(var, tile, s, out_i32=True)
        got = c.cpu().numpy()
        assert np.array_equal(got, acc), f"acc mismatch var={var} tile={tile} S={s}"


@pytest.mark.parametrize("fmt", FMTS)
def test_variants_bitwise_identical_for_fixed_segmentation(fmt):
    # the fixed-order reduction makes every variant give the same bits for a
    # given k_segments (the property batch invariance rests on)
    M, N, K = 48, 512, 1024
    p = Prepared(fmt, *_problem(fmt, M, N, K, seed=5))
    for s in (1, 2, 4):
        outs = {}
        for var, tile, ss in _variants(fmt, K):
            if ss != s:
                continue
            outs[(var, tile)] = bits_u16(p.run(var, tile, s))
        keys = list(outs)
        for k in keys[1:]:
            assert np.array_equal(outs[keys[0]], outs[k]), f"S={s}: {keys[0]} vs {k}"


CLUSTER_MAX = {16: 8, 32: 4, 64: 4}


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(3, 640, 1024), (40, 3072, 3072), (64, 25600, 1024)])
def test_cluster_splitk_matches_workspace_splitk_and_oracle(fmt, M, N, K):
    # Swap-AB Split-K through a thread-block cluster (segments reduced in the
    # shared memory of rank 0) against the workspace reduction: bitwise equal,
    # and within the parity bar of the oracle.  N=25600 gives every cluster
    # several tiles (the per-tile exchange runs through many phases); M=40
    # gives several tiles along M for the narrow tiles.
    from quantized_linear_layers_group_b200 import qlin

    p = Prepared(fmt, *_problem(fmt, M, N, K, seed=M + N + fmt))
    rows = np.unique(np.r_[0, M - 1, np.arange(0, M, 5)])
    ref = p.reference(m_idx=rows)
    racc = p.reference(m_idx=rows, want_acc=True)[1] if fmt == oracle.FMT_INT8 else None
    kb = K // 128
    checked = 0
    for tile in (16, 32, 64):
        for s in range(2, CLUSTER_MAX[tile] + 1):
            if kb % s:
                continue
            got = bits_u16(p.run(SWAPAB_SPLITK, tile, s, flags=qlin.QLIN_SPLITK_CLUSTER))
            want = bits_u16(p.run(SWAPAB_SPLITK, tile, s))
            assert np.array_equal(got, want), f"cluster vs workspace: fmt={fmt} tile={tile} S={s}"
            same_s = bits_u16(p.run(PLAIN, 128, s))
            assert np.array_equal(got, same_s), f"cluster vs plain: fmt={fmt} tile={tile} S={s}"
            if fmt == oracle.FMT_INT8:
                acc = p.run(SWAPAB_SPLITK, tile, s, out_i32=True, flags=qlin.QLIN_SPLITK_CLUSTER).cpu().numpy()
                assert np.array_equal(acc[rows], racc), f"INT8 accumulators tile={tile} S={s}"
            assert_parity(fmt, got[rows], ref, f"cluster fmt={fmt} M={M} N={N} K={K} tile={tile} S={s}")
            checked += 1
    assert checked >= 3
    check_status()


@pytest.mark.parametrize("fmt", FMTS)
def test_auto_dispatch_matches_oracle(fmt):
    N, K = 512, 768
    for M in (1, 16, 40, 64, 65, 200):
        p = Prepared(fmt, *_problem(fmt, M, N, K, seed=M))
        assert_parity(fmt, bits_u16(p.run()), p.reference(), f"auto M={M}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(3, 256, 128), (70, 384, 128), (5, 256, 8192), (140, 256, 8192)])
def test_extreme_depths(fmt, M, N, K):
    # one 128-wide K block (no pipelining across K), and a deep K of 64 blocks
    # (the shared-memory ring wraps several times; up to 8 segments)
    p = Prepared(fmt, *_problem(fmt, M, N, K, seed=K + M + fmt))
    ref = p.reference()
    kb = K // 128
    for var, tile, s in [(PLAIN, 128, 1), (SWAPAB, 16, 1), (SWAPAB, 64, 1)] + \
            ([(PAIR, 256, 1)] if fmt != oracle.FMT_FP8_BLOCK else []) + \
            ([(SPLITK, 128, 8), (SWAPAB_SPLITK, 16, 8), (PLAIN, 128, 8)] if kb % 8 == 0 else []):
        c = p.run(var, tile, s)
        assert_parity(fmt, bits_u16(c), ref, f"fmt={fmt} M={M} N={N} K={K} var={var} tile={tile} S={s}")
    check_status()


def test_zero_activation_row_gives_bias():
    fmt = oracle.FMT_FP8
    a, w, b = _problem(fmt, 9, 256, 256, seed=3)
    a[4] = 0
    p = Prepared(fmt, a, w, b)
    c = bits_u16(p.run(SWAPAB, 16, 1))
    assert np.array_equal(c[4], synth.bf16_bits(b))
    c = bits_u16(p.run(PLAIN, 128, 2))
    assert np.array_equal(c[4], synth.bf16_bits(b))


def test_empty_batch_is_a_no_op():
    from quantized_linear_layers_group_b200 import qlin

    w = torch.zeros(256, 256, dtype=torch.uint8, device="cuda")
    s = torch.ones(256, dtype=torch.float32, device="cuda")
    c = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    a = torch.empty(0, 256, dtype=torch.uint8, device="cuda")
    qlin.qlin_scaled_mm(qlin.QLIN_FMT_FP8, a, s, w, s, None, c, M=0)
    torch.cuda.synchronize()


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
@pytest.mark.parametrize("M,N,K", [(300, 25600, 1024), (1100, 4096, 2048), (2048, 4096, 2048), (129, 272, 640)])
def test_pair_tiles_match_single_cta_tiles_and_oracle(fmt, M, N, K):
    # 256-row tiles on CTA pairs (cta_group::2): every cluster walks several
    # tiles (N=25600: 200 tiles on at most 74 pairs), the last pair's second
    # CTA may hold no rows at all (M=1100, 129: an odd number of 128-row
    # halves), and N tails inside the second CTA's half of a W tile (N=272).
    # Bitwise equal to the one-CTA 256-column tiles with the same K
    # segmentation, within the parity bar of the oracle on a row sample.
    p = Prepared(fmt, *_problem(fmt, M, N, K, seed=M + N + K + 3 * fmt))
    rows = np.unique(np.r_[0, 1, 127, 128, 255, 256, M - 1, np.arange(0, M, max(1, M // 24))])
    rows = rows[rows < M]
    segs = [1] if fmt == oracle.FMT_FP8 or (K // 128) % 4 else [1, 4]
    for s in segs:
        got = bits_u16(p.run(PAIR, 256, s))
        want = bits_u16(p.run(PLAIN, 256, s))
        assert np.array_equal(got, want), f"pair vs plain: fmt={fmt} M={M} N={N} K={K} S={s}"
        assert_parity(fmt, got[rows], p.reference(m_idx=rows), f"pair fmt={fmt} M={M} N={N} K={K} S={s}")
    if fmt == oracle.FMT_INT8:
        acc = p.run(PAIR, 256, 1, out_i32=True).cpu().numpy()
        assert np.array_equal(acc[rows], p.reference(m_idx=rows, want_acc=True)[1])
    check_status()
