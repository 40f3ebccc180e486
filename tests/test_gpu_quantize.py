"""GPU parity of the quantisation kernels against the oracle: bit-exact codes and
scales (INT8 / FP8 per-token, Block-FP8 1x128 groups and 128x128 blocks)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import bits_u8, check_status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from quantized_linear_layers_group_b200 import qlin
    return qlin


def _gpu_per_token(lib, fmt, x):
    xd = x.cuda()
    rows, cols = x.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    lib.qlin_quantize_per_token(fmt, xd, q, s)
    torch.cuda.synchronize()
    return bits_u8(q), s.cpu().numpy()


def _gpu_block(lib, x, block_rows):
    xd = x.cuda()
    rows, cols = x.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty((rows + block_rows - 1) // block_rows, cols // 128, dtype=torch.float32, device="cuda")
    lib.qlin_quantize_block(xd, block_rows, q, s)
    torch.cuda.synchronize()
    return bits_u8(q), s.cpu().numpy()


def _assert_same(q_gpu, s_gpu, q_ref, s_ref, what):
    assert np.array_equal(s_gpu.view(np.uint32), s_ref.view(np.uint32)), f"{what}: scales differ"
    if not np.array_equal(q_gpu, q_ref):
        bad = np.argwhere(q_gpu != q_ref)
        raise AssertionError(f"{what}: {len(bad)} codes differ, first {bad[:5].tolist()} "
                             f"gpu={q_gpu[tuple(bad[:5].T)]} ref={q_ref[tuple(bad[:5].T)]}")


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
@pytest.mark.parametrize("wname,M", [("int8_smoke", 16), ("fp8_attn", 1), ("fp8_attn", 333),
                                     ("fp8_block_down", 64), ("fp8_attn", 2048)])
def test_per_token_workload_rows(lib, fmt, wname, M):
    x = synth.activations(synth.WORKLOADS[wname], M, seed=0)
    qg, sg = _gpu_per_token(lib, fmt, x)
    qr, sr = oracle.quantize_per_token(fmt, x)
    _assert_same(qg, sg, qr, sr, f"{wname} M={M}")
    check_status()


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_per_token_exhaustive_bf16(lib, fmt):
    # every finite bf16 value paired with the format's Qmax so the scale is 1
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    qmax = 127.0 if fmt == oracle.FMT_INT8 else 448.0
    vb = bits[np.isfinite(f) & (np.abs(f) <= qmax)].astype(np.uint16)
    head = np.uint16(0x42FE if fmt == oracle.FMT_INT8 else 0x43E0)
    x_bits = np.stack([np.full_like(vb, head)] + [vb] * 7, axis=1)  # 8 columns (16-byte rows)
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
    qg, sg = _gpu_per_token(lib, fmt, x)
    qr, sr = oracle.quantize_per_token(fmt, x)
    assert np.all(sg == 1.0)
    _assert_same(qg, sg, qr, sr, "exhaustive")


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_per_token_random_magnitudes_and_edges(lib, fmt):
    g = torch.Generator().manual_seed(17)
    x = torch.randn(67, 2056, generator=g) * torch.exp(torch.randn(67, 1, generator=g) * 4)
    x[3] = 0.0                      # amax = 0
    x[4] = -0.0
    x[5, :] = -7.0                  # all -amax
    x[6] = 0.0
    x[6, 1000] = 3e-5               # single non-zero
    x[7, ::2] = 1e-30               # subnormal-range quotients
    x = x.to(torch.bfloat16)
    qg, sg = _gpu_per_token(lib, fmt, x)
    qr, sr = oracle.quantize_per_token(fmt, x)
    _assert_same(qg, sg, qr, sr, "random")
    assert sg[3] == 0 and np.all(qg[3] == 0) and np.all(qg[4] == 0)


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
@pytest.mark.parametrize("cols", [8, 136, 8192, 8200, 12288])
def test_per_token_column_counts(lib, fmt, cols):
    # register-resident paths up to 8192 columns, two-pass path above
    x = synth.normal((9, cols), 1.0, cols)
    qg, sg = _gpu_per_token(lib, fmt, x)
    qr, sr = oracle.quantize_per_token(fmt, x)
    _assert_same(qg, sg, qr, sr, f"cols={cols}")


def test_per_token_strided_input(lib):
    x = synth.normal((20, 512), 1.0, 3)
    xd = x.cuda()
    sub = xd[:, 128:384]                       # ld_x = 512, cols = 256
    q = torch.empty(20, 256, dtype=torch.uint8, device="cuda")
    s = torch.empty(20, dtype=torch.float32, device="cuda")
    lib.qlin_quantize_per_token(oracle.FMT_FP8, sub, q, s)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_per_token(oracle.FMT_FP8, x[:, 128:384].contiguous())
    _assert_same(bits_u8(q), s.cpu().numpy(), qr, sr, "strided")


@pytest.mark.parametrize("rows,cols", [(1, 128), (37, 6144), (2048, 6144), (5, 16384)])
def test_group128_activations(lib, rows, cols):
    w = synth.WORKLOADS["fp8_block_down"]
    x = synth.activations(w, rows, seed=1) if cols == 6144 else synth.normal((rows, cols), 3.0, 5)
    qg, sg = _gpu_block(lib, x, 1)
    qr, sr = oracle.quantize_block(x, 1, 128)
    _assert_same(qg, sg, qr, sr, f"group128 {rows}x{cols}")


@pytest.mark.parametrize("rows,cols", [(128, 128), (300, 384), (2048, 6144)])
def test_block128_weights(lib, rows, cols):
    x = synth.normal((rows, cols), 0.02, rows + cols)
    if cols > 128:
        x[:, 128:256] = 0  # an all-zero block column
    qg, sg = _gpu_block(lib, x, 128)
    qr, sr = oracle.quantize_block(x, 128, 128)
    _assert_same(qg, sg, qr, sr, f"block128 {rows}x{cols}")
    check_status()


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_per_token_division_across_scale_magnitudes(lib, fmt):
    # rows whose amax spans 2^-100 .. 2^120 (both sides of the fast-quotient
    # range of scales), filled with values concentrated near the target grid's
    # rounding boundaries; codes and scales must equal the oracle's, which
    # divides with IEEE binary32 division.
    g = torch.Generator().manual_seed(99)
    rows, cols = 2048, 136
    e = torch.linspace(-100, 120, rows)
    amax = torch.exp2(e.round())[:, None] * (1 + torch.rand(rows, 1, generator=g))
    qmax = 127.0 if fmt == oracle.FMT_INT8 else 448.0
    # quotients near half-integers (INT8) / e4m3 midpoints (FP8) and plain random ones
    u = torch.rand(rows, cols, generator=g)
    near = (torch.floor(u * qmax) + 0.5) / qmax
    mix = torch.where(torch.rand(rows, cols, generator=g) < 0.5, near, u)
    sign = torch.where(torch.rand(rows, cols, generator=g) < 0.5, -1.0, 1.0)
    x = (sign * mix * amax).to(torch.bfloat16)
    x[:, 0] = amax[:, 0].to(torch.bfloat16)
    qg, sg = _gpu_per_token(lib, fmt, x)
    qr, sr = oracle.quantize_per_token(fmt, x)
    _assert_same(qg, sg, qr, sr, "division sweep")


def test_group128_division_across_scale_magnitudes(lib):
    g = torch.Generator().manual_seed(7)
    rows, cols = 512, 1024
    grp = torch.exp2(torch.randint(-90, 110, (rows, cols // 128), generator=g).float())
    x = (torch.randn(rows, cols, generator=g) * grp.repeat_interleave(128, dim=1)).to(torch.bfloat16)
    qg, sg = _gpu_block(lib, x, 1)
    qr, sr = oracle.quantize_block(x, 1, 128)
    _assert_same(qg, sg, qr, sr, "group division sweep")


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
@pytest.mark.parametrize("rows", [1, 511, 513, 2049, 4100])
def test_per_token_every_row_split(lib, fmt, rows):
    # 8, 2 and 1 warps per row are chosen by the row count: cover each and the edges
    x = synth.normal((rows, 2048), 1.0, rows)
    qg, sg = _gpu_per_token(lib, fmt, x)
    qr, sr = oracle.quantize_per_token(fmt, x)
    _assert_same(qg, sg, qr, sr, f"rows={rows}")


@pytest.mark.parametrize("rows", [1, 600, 3000])
def test_group128_every_row_split(lib, rows):
    x = synth.normal((rows, 6144), 2.0, rows + 1)
    qg, sg = _gpu_block(lib, x, 1)
    qr, sr = oracle.quantize_block(x, 1, 128)
    _assert_same(qg, sg, qr, sr, f"group rows={rows}")


@pytest.mark.parametrize("rows", [3, 700, 2500])
@pytest.mark.parametrize("cols", [640, 1152, 4224, 6272])
def test_group128_odd_group_counts(lib, rows, cols):
    # 5, 9, 33 and 49 groups per row: a row's last slot of 8 groups per warp is
    # partly empty, for each warps-per-row choice the row count leads to
    x = synth.normal((rows, cols), 1.5, rows * 7 + cols)
    qg, sg = _gpu_block(lib, x, 1)
    qr, sr = oracle.quantize_block(x, 1, 128)
    _assert_same(qg, sg, qr, sr, f"group rows={rows} cols={cols}")


def _markstein_rows(fmt, binades):
    """Rows [amax, x...] for every amax significand in the given binades: the
    row's x values are every bf16 significand at every exponent from amax's
    down to 21 binades below it (where the quotient x / s leaves the range of
    non-zero codes), both signs, |x| <= amax; unused slots are +0."""
    rel = 22
    L = 8 + 2 * 128 * rel                     # a multiple of 8 (16-byte rows)
    rows = []
    for eb in binades:                        # unbiased exponent of amax
        EA = eb + 127
        for ma in range(128):
            amax = (EA << 7) | ma
            r = np.zeros(L, np.uint16)
            r[0] = amax
            i = 1
            for d in range(rel):
                E = EA - d
                for mx in range(128):
                    if d == 0 and mx > ma:
                        continue
                    v = (E << 7) | mx
                    r[i] = v
                    r[i + 1] = v | 0x8000
                    i += 2
            rows.append(r)
    return np.stack(rows)


@pytest.mark.parametrize("fmt", [oracle.FMT_INT8, oracle.FMT_FP8])
def test_per_token_quotient_exhaustive_over_significands(lib, fmt):
    # The quantisers form x / s as one reciprocal of s plus Markstein's
    # correction step where s lies in [2^-68, 2^92], and as an IEEE division
    # elsewhere.  A quotient's rounding depends only on the significands of
    # amax (hence of s = amax / Qmax) and of x and on their exponent gap, so
    # every amax significand x every x significand x every gap that can give a
    # non-zero code, in the binade amax in [1, 2), covers the whole fast range
    # up to its edges; the edges themselves are covered by every amax of the
    # five binades around each of 2^-68 * Qmax and 2^92 * Qmax.  Codes and
    # scales must equal the oracle's (IEEE binary32 division) bit for bit.
    qmax = 127.0 if fmt == oracle.FMT_INT8 else 448.0
    lo = int(np.floor(np.log2(2.0 ** -68 * qmax)))
    hi = int(np.floor(np.log2(2.0 ** 92 * qmax)))
    binades = [0] + list(range(lo - 2, lo + 3)) + list(range(hi - 2, hi + 3))
    x_bits = _markstein_rows(fmt, binades)
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
    qg, sg = _gpu_per_token(lib, fmt, x)
    qr, sr = oracle.quantize_per_token(fmt, x)
    s_edge = sr[128:]
    assert (s_edge < 2.0 ** -68).any() and (s_edge >= 2.0 ** -68).any()      # both sides of the low edge
    assert (s_edge > 2.0 ** 92).any() and (s_edge <= 2.0 ** 92).any()        # and of the high edge
    _assert_same(qg, sg, qr, sr, "quotient exhaustive")
    check_status()
