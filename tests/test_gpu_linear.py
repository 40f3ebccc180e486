"""GPU parity of qlin_linear, the whole layer in one call: dynamic activation
quantisation followed by the scaled GEMM.  With QLIN_FUSED, Swap-AB
configurations whose work units fit the kernel's resident activation operand
have the GEMM quantise its own activation rows (one kernel); its C, codes and
scales must be bitwise those of the default two-kernel path (the stand-alone
quantiser, then the GEMM), and the codes / scales bit-exact and C within the
parity bar against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_parity, bits_u8, bits_u16, check_status, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu

PLAIN, SPLITK, SWAPAB, SWAPAB_SPLITK = 1, 2, 3, 4
FMTS = [oracle.FMT_INT8, oracle.FMT_FP8, oracle.FMT_FP8_BLOCK]
FUSED_MAX_KB = {16: 32, 32: 16, 64: 8}  # K blocks per unit the resident operand holds


def _inputs(fmt, M, N, K, seed, pad=0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K + pad, generator=g) * torch.exp(torch.randn(M, 1, generator=g))).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16) if fmt != oracle.FMT_FP8_BLOCK else None
    return x, w, b


class Layer:
    def __init__(self, fmt, w, b):
        self.fmt = fmt
        self.w_q, self.s_w = gpu_quantize(fmt, w.cuda(), True)
        self.rw_q, self.rs_w = oracle_quantize(fmt, w, True)
        torch.cuda.synchronize()
        assert np.array_equal(bits_u8(self.w_q), self.rw_q)
        self.b = b
        self.b_dev = None if b is None else b.cuda()
        self.N, self.K = w.shape

    def run(self, x_dev, K, variant, tile, S, flags=0, out_i32=False):
        from quantized_linear_layers_group_b200 import qlin

        M = x_dev.shape[0]
        a_q = torch.full((M, K), 0x5A, dtype=torch.uint8, device="cuda")  # outputs: start from junk
        if self.fmt == oracle.FMT_FP8_BLOCK:
            s_a = torch.full((M, K // 128), -1.0, dtype=torch.float32, device="cuda")
        else:
            s_a = torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
        c = torch.empty(M, self.N, dtype=torch.int32 if out_i32 else torch.bfloat16, device="cuda")
        nb = qlin.qlin_scaled_mm_workspace_size(self.fmt, M, self.N, K, variant, tile, S)
        ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
        qlin.qlin_linear(self.fmt, x_dev, a_q, s_a, self.w_q, self.s_w, self.b_dev, c, ws, variant=variant,
                         tile_n=tile, k_segments=S, K=K, ld_x=x_dev.stride(0),
                         flags=flags | (qlin.QLIN_OUT_I32ACC if out_i32 else 0))
        torch.cuda.synchronize()
        return c, a_q, s_a


def _check_against_unfused_and_oracle(layer, x, x_dev, K, variant, tile, S, rows=None, cols=None, what=""):
    from quantized_linear_layers_group_b200 import qlin

    c, a_q, s_a = layer.run(x_dev, K, variant, tile, S, flags=qlin.QLIN_FUSED)
    c2, a_q2, s_a2 = layer.run(x_dev, K, variant, tile, S)
    assert np.array_equal(bits_u16(c), bits_u16(c2)), f"{what}: C differs from the two-kernel path"
    assert np.array_equal(bits_u8(a_q), bits_u8(a_q2)), f"{what}: codes differ from the quantiser's"
    assert np.array_equal(s_a.cpu().numpy().view(np.uint32), s_a2.cpu().numpy().view(np.uint32)), \
        f"{what}: scales differ from the quantiser's"
    xs = x[:, :K].contiguous()
    ra_q, rs_a = oracle_quantize(layer.fmt, xs, False)
    assert np.array_equal(bits_u8(a_q), ra_q), f"{what}: codes differ from the oracle"
    assert np.array_equal(s_a.cpu().numpy().view(np.uint32), rs_a.view(np.uint32)), f"{what}: scales vs oracle"
    ref = oracle.scaled_mm(layer.fmt, ra_q, rs_a, layer.rw_q, layer.rs_w, layer.b, m_idx=rows, n_idx=cols)
    got = bits_u16(c)
    if rows is not None:
        got = got[rows]
    if cols is not None:
        got = got[:, cols]
    assert_parity(layer.fmt, got, ref, what)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 5, 16, 37, 64])
def test_fused_layer_matches_two_kernel_path_and_oracle(fmt, M):
    N, K = 384, 1024
    x, w, b = _inputs(fmt, M, N, K, seed=100 + M + fmt)
    layer = Layer(fmt, w, b)
    x_dev = x.cuda()
    checked = 0
    for tile in (16, 32, 64):
        for S in (1, 2, 4, 8):
            var = SWAPAB if S == 1 else SWAPAB_SPLITK
            if (K // 128) // S > FUSED_MAX_KB[tile]:
                continue
            _check_against_unfused_and_oracle(layer, x, x_dev, K, var, tile, S,
                                              what=f"fmt={fmt} M={M} tile={tile} S={S}")
            checked += 1
    assert checked >= 8
    check_status()


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_layer_several_units_per_cta(fmt):
    # 320 weight tiles x 2 activation tiles: every CTA quantises several units
    # in turn (the next unit's rows while the current one is in its epilogue)
    M, N, K = 20, 40960, 2048
    x, w, b = _inputs(fmt, M, N, K, seed=7 + fmt)
    layer = Layer(fmt, w, b)
    cols = np.unique(np.r_[np.arange(0, N, 37), N - 1])
    for tile, S in ((16, 1), (16, 2), (32, 2)):
        if fmt == oracle.FMT_FP8_BLOCK and S == 1:
            continue  # 16 K blocks of Block-FP8 per unit: fine, but keep the case count down
        _check_against_unfused_and_oracle(layer, x, x.cuda(), K, SWAPAB if S == 1 else SWAPAB_SPLITK, tile, S,
                                          cols=cols, what=f"fmt={fmt} tile={tile} S={S}")
    check_status()


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_layer_strided_activations(fmt):
    M, N, K = 9, 256, 768
    x, w, b = _inputs(fmt, M, N, K, seed=3, pad=64)  # row stride K + 64 elements
    layer = Layer(fmt, w, b)
    x_dev = x.cuda()
    for tile, S in ((16, 1), (16, 3), (32, 2)):
        _check_against_unfused_and_oracle(layer, x, x_dev, K, SWAPAB if S == 1 else SWAPAB_SPLITK, tile, S,
                                          what=f"strided fmt={fmt} tile={tile} S={S}")


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_fused_layer_rows_with_scales_outside_the_reciprocal_range(fmt):
    # Row scales amax / Qmax below 2^-68 or above 2^92 take the IEEE division
    # instead of the reciprocal and its correction step, in the fused kernel's
    # register-resident path (first unit of a CTA) as in the quantiser.
    M, N, K = 8, 256, 1024
    x, w, b = _inputs(fmt, M, N, K, seed=41 + fmt)
    row_exp = [-80, -70, -58, 0, 96, 103, 110, None]  # None: an all-zero row
    xf = x.float()
    for r, e in enumerate(row_exp):
        xf[r] = 0.0 if e is None else torch.ldexp(xf[r] / xf[r].abs().max(), torch.tensor(float(e)))
    x = xf.to(torch.bfloat16)
    assert torch.isfinite(x.float()).all()
    layer = Layer(fmt, w, b)
    x_dev = x.cuda()
    for tile, S in ((16, 1), (32, 2), (64, 1)):
        _check_against_unfused_and_oracle(layer, x, x_dev, K, SWAPAB if S == 1 else SWAPAB_SPLITK, tile, S,
                                          what=f"extreme scales fmt={fmt} tile={tile} S={S}")
    check_status()


def test_fused_int8_accumulators_bit_exact():
    from quantized_linear_layers_group_b200 import qlin

    fmt = oracle.FMT_INT8
    M, N, K = 23, 640, 2048
    x, w, b = _inputs(fmt, M, N, K, seed=21)
    layer = Layer(fmt, w, b)
    ra_q, rs_a = oracle_quantize(fmt, x, False)
    _, acc = oracle.scaled_mm(fmt, ra_q, rs_a, layer.rw_q, layer.rs_w, b, want_acc=True)
    for tile, S in ((16, 1), (32, 4), (64, 2)):
        c, _, _ = layer.run(x.cuda(), K, SWAPAB if S == 1 else SWAPAB_SPLITK, tile, S, out_i32=True,
                            flags=qlin.QLIN_FUSED)
        assert np.array_equal(c.cpu().numpy(), acc), f"tile={tile} S={S}"


def test_fused_layer_zero_rows_and_auto_dispatch():
    from quantized_linear_layers_group_b200 import qlin

    fmt = oracle.FMT_FP8
    M, N, K = 12, 512, 2048
    x, w, b = _inputs(fmt, M, N, K, seed=5)
    x[3] = 0  # a zero row: scale 0, codes 0, C row = bias
    layer = Layer(fmt, w, b)
    c, a_q, s_a = layer.run(x.cuda(), K, 0, 0, 0)
    assert float(s_a[3]) == 0.0 and int(a_q[3].abs().sum()) == 0
    assert np.array_equal(bits_u16(c)[3], b.view(torch.int16).numpy().view(np.uint16))
    _check_against_unfused_and_oracle(layer, x, x.cuda(), K, 0, 0, 0, what="auto")
    assert qlin.qlin_sync_status() == 0


def test_quantized_linear_module_runs_quantiser_then_pdl_gemm():
    # QuantizedLinear's default: qlin_linear with QLIN_PDL (the stand-alone
    # quantiser, then the GEMM as its programmatic dependent)
    from quantized_linear_layers_group_b200 import linear

    fmt = oracle.FMT_FP8
    M, N, K = 4, 1024, 2048
    x, w, b = _inputs(fmt, M, N, K, seed=9)
    mod = linear.QuantizedLinear(fmt, w.cuda(), b.cuda())
    c = mod(x.cuda())
    torch.cuda.synchronize()
    ra_q, rs_a = oracle_quantize(fmt, x, False)
    rw_q, rs_w = oracle_quantize(fmt, w, True)
    assert_parity(fmt, bits_u16(c), oracle.scaled_mm(fmt, ra_q, rs_a, rw_q, rs_w, b), "module")


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_layer_on_cta_pair_tiles(fmt):
    # qlin_linear with the 256x256 CTA-pair tiles (the quantiser, then the
    # pair GEMM; QLIN_FUSED does not apply to plain tiles and is ignored):
    # codes and scales bit-exact, C bitwise equal to one-CTA 256-column tiles
    # and within the parity bar of the oracle, with a strided x and a tail of
    # rows and columns.
    PAIR = 5
    M, N, K = 300, 528, 1024
    x, w, b = _inputs(fmt, M, N, K, seed=21 + fmt, pad=64)
    layer = Layer(fmt, w, b)
    x_dev = x.cuda()
    rows = np.unique(np.r_[0, 127, 128, 255, 256, M - 1, np.arange(0, M, 11)])
    c_pair, a_q, s_a = layer.run(x_dev, K, PAIR, 256, 1)
    c_plain, _, _ = layer.run(x_dev, K, PLAIN, 256, 1)
    assert np.array_equal(bits_u16(c_pair), bits_u16(c_plain)), "pair vs one-CTA tiles"
    ra_q, rs_a = oracle_quantize(fmt, x[:, :K].contiguous(), False)
    assert np.array_equal(bits_u8(a_q), ra_q)
    assert np.array_equal(s_a.cpu().numpy().view(np.uint32), rs_a.view(np.uint32))
    ref = oracle.scaled_mm(fmt, ra_q, rs_a, layer.rw_q, layer.rs_w, layer.b, m_idx=rows)
    assert_parity(fmt, bits_u16(c_pair)[rows], ref, f"pair layer fmt={fmt}")
    from quantized_linear_layers_group_b200 import qlin
    c_fl, _, _ = layer.run(x_dev, K, PAIR, 256, 1, flags=qlin.QLIN_FUSED)
    assert np.array_equal(bits_u16(c_fl), bits_u16(c_pair)), "QLIN_FUSED on pair tiles"
    check_status()
