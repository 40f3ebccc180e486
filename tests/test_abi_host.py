"""Host-only checks of the C ABI (no GPU): the library loads, exports every
symbol include/qlin.h declares, validates arguments before launching
anything, and plans / dispatches shapes as documented."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q():
    from quantized_linear_layers_group_b200 import build

    build.build()
    from quantized_linear_layers_group_b200 import qlin

    return qlin


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "qlin.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^QLIN_API\s+[\w\s\*]+?\b(qlin_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    for name in ("qlin_quantize_per_token", "qlin_quantize_block", "qlin_scaled_mm", "qlin_dispatch_table_load"):
        assert name in syms
    assert len(syms) == 23


def test_library_exports_every_declared_symbol(q):
    import ctypes

    lib = ctypes.CDLL(q.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(_declared_symbols()) == set(q.EXPORTS)
    assert q.qlin_abi_version() == 7


def test_status_strings(q):
    for s in range(0, 11):
        assert q.qlin_status_string(s) and q.qlin_status_string(s) != "unknown status"
    assert q.qlin_status_string(99) == "unknown status"


def _mm(q, **kw):
    args = dict(fmt=1, variant=0, tile_n=0, k_segments=0, M=16, N=256, K=256, a=16, sa=16, w=16, sw=16,
                bias=None, c=16, flags=0, ws=None, wsb=0)
    args.update(kw)
    return q.lib.qlin_scaled_mm(args["fmt"], args["variant"], args["tile_n"], args["k_segments"], args["M"],
                                args["N"], args["K"], args["a"], args["sa"], args["w"], args["sw"], args["bias"],
                                args["c"], args["flags"], args["ws"], args["wsb"], None)


def test_scaled_mm_rejects_bad_arguments_before_launch(q):
    assert _mm(q, fmt=7) == q.QLIN_ERR_INVALID_ARG
    assert _mm(q, N=8) == q.QLIN_ERR_INVALID_ARG
    assert _mm(q, N=250) == q.QLIN_ERR_UNSUPPORTED
    assert _mm(q, K=200) == q.QLIN_ERR_UNSUPPORTED
    assert _mm(q, fmt=2, N=320) == q.QLIN_ERR_UNSUPPORTED
    assert _mm(q, M=-1) == q.QLIN_ERR_INVALID_ARG
    assert _mm(q, variant=9) == q.QLIN_ERR_INVALID_ARG
    assert _mm(q, flags=16) == q.QLIN_ERR_INVALID_ARG          # undefined flag bit
    assert _mm(q, flags=8) == q.QLIN_ERR_INVALID_ARG           # QLIN_FUSED is for qlin_linear
    assert _mm(q, flags=1) == q.QLIN_ERR_INVALID_ARG          # I32 accumulators are INT8 only
    assert _mm(q, fmt=2, bias=16) == q.QLIN_ERR_INVALID_ARG   # Block-FP8 takes no bias
    assert _mm(q, a=None) == q.QLIN_ERR_INVALID_ARG
    assert _mm(q, a=24) == q.QLIN_ERR_ALIGNMENT
    assert _mm(q, c=8) == q.QLIN_ERR_ALIGNMENT
    assert _mm(q, sa=18) == q.QLIN_ERR_ALIGNMENT
    assert _mm(q, M=0) == q.QLIN_OK                            # empty batch: no-op


def test_quantize_rejects_bad_arguments(q):
    L = q.lib
    assert L.qlin_quantize_per_token(2, 16, 4, 64, 64, 16, 16, 0, None) == q.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_per_token(1, 16, 4, 60, 64, 16, 16, 0, None) == q.QLIN_ERR_ALIGNMENT
    assert L.qlin_quantize_per_token(1, 16, 4, 64, 32, 16, 16, 0, None) == q.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_per_token(1, 8, 4, 64, 64, 16, 16, 0, None) == q.QLIN_ERR_ALIGNMENT
    assert L.qlin_quantize_per_token(1, None, 4, 64, 64, 16, 16, 0, None) == q.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_per_token(1, 16, 4, 64, 64, 16, 16, 4, None) == q.QLIN_ERR_INVALID_ARG  # bad flag
    assert L.qlin_quantize_per_token(1, None, 0, 64, 64, None, None, 0, None) == q.QLIN_OK
    assert L.qlin_quantize_block(16, 4, 256, 256, 2, 128, 16, 16, 0, None) == q.QLIN_ERR_UNSUPPORTED
    assert L.qlin_quantize_block(16, 4, 256, 256, 1, 64, 16, 16, 0, None) == q.QLIN_ERR_UNSUPPORTED
    assert L.qlin_quantize_block(16, 4, 200, 200, 1, 128, 16, 16, 0, None) == q.QLIN_ERR_UNSUPPORTED
    assert L.qlin_quantize_block(16, 4, 256, 256, 1, 128, 16, 17, 0, None) == q.QLIN_ERR_ALIGNMENT
    assert L.qlin_quantize_block(16, 4, 256, 256, 1, 128, 16, 16, 8, None) == q.QLIN_ERR_INVALID_ARG


def test_workspace_sizes(q):
    # Swap-AB + Split-K, FP8 N=4096 K=2048 M=16: S=4 segments of 32 tiles of 128x16
    assert q.qlin_scaled_mm_workspace_size(1, 16, 4096, 2048) == 65536 + 4 * 32 * 128 * 16 * 4
    # plain variants need none
    assert q.qlin_scaled_mm_workspace_size(1, 2048, 151936, 2048) == 0
    assert q.qlin_scaled_mm_workspace_size(1, 16, 256, 256, variant=q.QLIN_VAR_PLAIN, tile_n=128,
                                           k_segments=1) == 0
    with pytest.raises(q.QlinError):
        q.qlin_scaled_mm_workspace_size(1, 16, 256, 384, k_segments=2)          # 3 K blocks, 2 segments
    with pytest.raises(q.QlinError):
        q.qlin_scaled_mm_workspace_size(1, 200, 4096, 2048, variant=q.QLIN_VAR_PLAIN, tile_n=256,
                                        k_segments=4)                            # multi-chunk on a 256 tile
    with pytest.raises(q.QlinError):
        q.qlin_scaled_mm_workspace_size(1, 16, 256, 256, variant=q.QLIN_VAR_SWAPAB, tile_n=128)
    # CTA-pair tiles: 256 columns, INT8 / FP8 only, no workspace, no multi-chunk FP8
    assert q.qlin_scaled_mm_workspace_size(1, 2048, 4096, 2048, variant=q.QLIN_VAR_PAIR, k_segments=1) == 0
    assert q.qlin_scaled_mm_workspace_size(0, 300, 2048, 2048, variant=q.QLIN_VAR_PAIR, k_segments=4) == 0
    for fmt, kw in ((1, dict(tile_n=128)), (2, {}), (1, dict(k_segments=2))):
        with pytest.raises(q.QlinError):
            q.qlin_scaled_mm_workspace_size(fmt, 2048, 4096, 2048, variant=q.QLIN_VAR_PAIR, **kw)
    with pytest.raises(q.QlinError):
        q.qlin_scaled_mm_workspace_size(1, 16, 256, 256, variant=6)


def test_builtin_dispatch_rule(q):
    q.qlin_dispatch_table_clear()
    c = q.qlin_dispatch_query(q.QLIN_FMT_FP8, 1, 4096, 2048)
    assert (c["variant"], c["tile_n"], c["k_segments"], c["from_table"]) == (q.QLIN_VAR_SWAPAB_SPLITK, 16, 4, 0)
    c = q.qlin_dispatch_query(q.QLIN_FMT_FP8, 64, 4096, 2048)
    assert (c["variant"], c["tile_n"]) == (q.QLIN_VAR_SWAPAB_SPLITK, 64)
    c = q.qlin_dispatch_query(q.QLIN_FMT_FP8, 2048, 4096, 2048)
    assert (c["variant"], c["tile_n"], c["k_segments"]) == (q.QLIN_VAR_PLAIN, 128, 4)
    c = q.qlin_dispatch_query(q.QLIN_FMT_FP8, 2048, 151936, 2048)
    assert (c["variant"], c["tile_n"], c["k_segments"]) == (q.QLIN_VAR_PLAIN, 256, 1)
    c = q.qlin_dispatch_query(q.QLIN_FMT_FP8_BLOCK, 1, 2048, 6144)
    assert (c["variant"], c["k_segments"]) == (q.QLIN_VAR_SWAPAB_SPLITK, 8)
    # segmentation is a property of the shape, never of M
    for fmt, N, K in ((1, 4096, 2048), (2, 2048, 6144), (1, 12288, 2048), (0, 2048, 2048)):
        segs = {q.qlin_dispatch_query(fmt, M, N, K)["k_segments"] for M in (1, 8, 64, 65, 256, 2048)}
        assert len(segs) == 1


def _write(tmp_path, text):
    p = tmp_path / "t.qlt"
    p.write_text(text)
    return str(p)


def test_table_loader_rejects_bad_files(q, tmp_path):
    with pytest.raises(q.QlinError) as e:
        q.qlin_dispatch_table_load(str(tmp_path / "missing.qlt"))
    assert e.value.status == q.QLIN_ERR_TABLE_IO
    head = "qlin-dispatch 1\ndevice 148 10 0 NVIDIA B200\n"
    bad = [
        "nonsense\n",
        "qlin-dispatch 2\ndevice 148 10 0 NVIDIA B200\n",
        "qlin-dispatch 1\n",                                                    # no device line
        head + "entry fp9 4096 2048 16 swapab 16 4\n",                         # bad format
        head + "entry fp8 4096 2048 16 swapab 128 4\n",                        # tile not allowed for swap
        head + "entry fp8 4096 2048 16 swapab 16 3\n",                         # 16 K blocks, 3 segments
        head + "entry fp8 4096 2048 16 swapab 16 4\nentry fp8 4096 2048 256 plain 128 2\n",  # S differs by M
        head + "entry fp8 4096 2048 16 swapab 16 4\nentry fp8 4096 2048 16 plain 128 4\n",  # duplicate bucket
        head + "entry fp8 4096 2048 256 plain 256 4\n",                        # multi-chunk 256 tile
        head + "entry fp8 4096 2048 16 swapab 16\n",                           # truncated
        head + "entry fp8 4096 2048 2048 pair 128 1\n",                       # pair tiles are 256 wide
        head + "entry fp8_block 2048 6144 2048 pair 256 4\n",                 # no Block-FP8 pair tiles
        head + "entry fp8 4096 2048 2048 pair 256 2\n",                       # multi-chunk 256 tile
    ]
    for text in bad:
        with pytest.raises(q.QlinError) as e:
            q.qlin_dispatch_table_load(_write(tmp_path, text))
        assert e.value.status == q.QLIN_ERR_TABLE_FORMAT, text


def test_pair_entries_pass_the_format_checks(q, tmp_path):
    # a table with CTA-pair entries gets past every format check; only the
    # device guard (which needs a B200) can refuse it here
    text = ("qlin-dispatch 1\ndevice 148 10 0 NVIDIA B200\n"
            "entry fp8 151936 2048 16 swapab 16 1\nentry fp8 151936 2048 2048 pair 256 1\n"
            "entry int8 2048 2048 16 swapab_splitk 16 4\nentry int8 2048 2048 2048 pair 256 4\n")
    try:
        q.qlin_dispatch_table_load(_write(tmp_path, text))
    except q.QlinError as e:
        assert e.status in (q.QLIN_ERR_NO_DEVICE, q.QLIN_ERR_TABLE_DEVICE, q.QLIN_ERR_CUDA), e
    finally:
        q.qlin_dispatch_table_clear()


def test_shipped_table_parses(q, tmp_path):
    # the committed table passes every format check (the device check needs a GPU)
    path = os.path.join(ROOT, "quantized_linear_layers_group_b200", "tables", "b200.qlt")
    if not os.path.exists(path):
        pytest.skip("no table shipped yet")
    try:
        q.qlin_dispatch_table_load(path)
    except q.QlinError as e:
        assert e.status in (q.QLIN_ERR_NO_DEVICE, q.QLIN_ERR_TABLE_DEVICE, q.QLIN_ERR_CUDA), e
    finally:
        q.qlin_dispatch_table_clear()


def _lin(q, **kw):
    args = dict(fmt=1, variant=0, tile_n=0, k_segments=0, M=16, N=256, K=256, x=16, ld=256, a=16, sa=16, w=16,
                sw=16, bias=None, c=16, flags=0, ws=None, wsb=0)
    args.update(kw)
    return q.lib.qlin_linear(args["fmt"], args["variant"], args["tile_n"], args["k_segments"], args["M"], args["N"],
                             args["K"], args["x"], args["ld"], args["a"], args["sa"], args["w"], args["sw"],
                             args["bias"], args["c"], args["flags"], args["ws"], args["wsb"], None)


def test_linear_rejects_bad_arguments_before_launch(q):
    assert _lin(q, fmt=5) == q.QLIN_ERR_INVALID_ARG
    assert _lin(q, ld=128) == q.QLIN_ERR_INVALID_ARG            # row stride below K
    assert _lin(q, ld=260) == q.QLIN_ERR_ALIGNMENT              # rows not 16-byte aligned
    assert _lin(q, x=24) == q.QLIN_ERR_ALIGNMENT
    assert _lin(q, x=None) == q.QLIN_ERR_INVALID_ARG
    assert _lin(q, a=None) == q.QLIN_ERR_INVALID_ARG            # the codes are an output and required
    assert _lin(q, flags=4) == q.QLIN_ERR_INVALID_ARG           # cluster Split-K is a qlin_scaled_mm flag
    assert _lin(q, flags=16) == q.QLIN_ERR_INVALID_ARG
    assert _lin(q, fmt=2, bias=16) == q.QLIN_ERR_INVALID_ARG
    assert _lin(q, K=200, ld=200) == q.QLIN_ERR_UNSUPPORTED
    assert _lin(q, M=0) == q.QLIN_OK


def test_selftest_rejects_bad_limits(q):
    assert q.lib.qlin_selftest_wait_timeout(0, None) == q.QLIN_ERR_INVALID_ARG
    assert q.lib.qlin_selftest_wait_timeout(2000000, None) == q.QLIN_ERR_INVALID_ARG


def test_matmul_bf16_rejects_bad_arguments_before_launch(q):
    def mm(**kw):
        a = dict(variant=0, tile_n=0, k_segments=0, M=16, N=256, K=256, a=16, w=16, bias=None, c=16, flags=0,
                 ws=None, wsb=0)
        a.update(kw)
        return q.lib.qlin_matmul_bf16(a["variant"], a["tile_n"], a["k_segments"], a["M"], a["N"], a["K"], a["a"],
                                      a["w"], a["bias"], a["c"], a["flags"], a["ws"], a["wsb"], None)

    assert mm(K=96) == q.QLIN_ERR_UNSUPPORTED                 # K blocks are 64 bf16 elements
    assert mm(K=32) == q.QLIN_ERR_INVALID_ARG
    assert mm(N=250) == q.QLIN_ERR_UNSUPPORTED
    assert mm(flags=1) == q.QLIN_ERR_INVALID_ARG              # no int32 accumulators for bf16
    assert mm(flags=8) == q.QLIN_ERR_INVALID_ARG
    assert mm(a=None) == q.QLIN_ERR_INVALID_ARG
    assert mm(w=24) == q.QLIN_ERR_ALIGNMENT
    assert mm(bias=17) == q.QLIN_ERR_ALIGNMENT
    assert mm(M=0) == q.QLIN_OK
    # the scaled entry points do not take the bf16 format
    assert _mm(q, fmt=q.QLIN_FMT_BF16) == q.QLIN_ERR_INVALID_ARG
    # K blocks of a bf16 row: K = 192 is three of them, so S = 3 divides it
    assert q.qlin_scaled_mm_workspace_size(q.QLIN_FMT_BF16, 16, 256, 192, q.QLIN_VAR_SWAPAB_SPLITK, 16, 3) > 0


def _bsmm(q, **kw):
    args = dict(fmt=4, variant=0, tile_n=0, k_segments=0, M=16, N=256, K=256, a=16, asf=16, w=16, wsf=16, ga=None,
                gw=None, bias=None, c=16, flags=0, ws=None, wsb=0)
    args.update(kw)
    return q.lib.qlin_block_scaled_mm(args["fmt"], args["variant"], args["tile_n"], args["k_segments"], args["M"],
                                      args["N"], args["K"], args["a"], args["asf"], args["w"], args["wsf"],
                                      args["ga"], args["gw"], args["bias"], args["c"], args["flags"], args["ws"],
                                      args["wsb"], None)


def test_block_scaled_entry_points_reject_bad_arguments_before_launch(q):
    assert _bsmm(q, fmt=1) == q.QLIN_ERR_INVALID_ARG                 # per-token formats: qlin_scaled_mm
    assert _bsmm(q, K=192) == q.QLIN_ERR_UNSUPPORTED                 # MXFP8: K % 128
    assert _bsmm(q, fmt=5, K=384, ga=16, gw=16) == q.QLIN_ERR_UNSUPPORTED   # NVFP4: K % 256
    assert _bsmm(q, fmt=5) == q.QLIN_ERR_INVALID_ARG                 # NVFP4 needs both decode scales
    assert _bsmm(q, ga=16, gw=16) == q.QLIN_ERR_INVALID_ARG          # MXFP8 takes none
    assert _bsmm(q, variant=q.QLIN_VAR_PAIR) == q.QLIN_ERR_UNSUPPORTED
    # tile support is planned without a device: through the workspace query
    import ctypes

    def ws(fmt, variant, tile_n):
        out = ctypes.c_size_t(0)
        return q.lib.qlin_scaled_mm_workspace_size(fmt, variant, tile_n, 0, 16, 256, 256, ctypes.byref(out))

    assert ws(4, q.QLIN_VAR_SWAPAB, 16) == q.QLIN_ERR_UNSUPPORTED     # whole 32-row quadrants only
    assert ws(4, q.QLIN_VAR_SWAPAB, 32) == q.QLIN_OK
    assert ws(4, q.QLIN_VAR_SWAPAB_SPLITK, 64) == q.QLIN_OK
    out = ctypes.c_size_t(0)
    assert q.lib.qlin_scaled_mm_workspace_size(4, q.QLIN_VAR_SWAPAB, 32, 0, 33, 256, 256,
                                               ctypes.byref(out)) == q.QLIN_ERR_UNSUPPORTED  # one activation tile
    assert ws(4, q.QLIN_VAR_PLAIN, 256) == q.QLIN_ERR_UNSUPPORTED
    assert ws(4, q.QLIN_VAR_PLAIN, 128) == q.QLIN_OK
    assert _bsmm(q, variant=9) == q.QLIN_ERR_INVALID_ARG
    assert _bsmm(q, flags=q.QLIN_SPLITK_CLUSTER) == q.QLIN_ERR_INVALID_ARG
    assert _bsmm(q, asf=None) == q.QLIN_ERR_INVALID_ARG
    assert _bsmm(q, asf=24) == q.QLIN_ERR_ALIGNMENT
    assert _bsmm(q, M=0) == q.QLIN_OK
    # the per-token entry points refuse the block-scaled formats
    assert _mm(q, fmt=4) == q.QLIN_ERR_INVALID_ARG
    assert _mm(q, fmt=5) == q.QLIN_ERR_INVALID_ARG
    L = q.lib
    assert L.qlin_quantize_block_scaled(1, 16, 4, 256, 256, None, 16, 16, 0, None) == q.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_block_scaled(4, 16, 4, 192, 192, None, 16, 16, 0, None) == q.QLIN_ERR_UNSUPPORTED
    assert L.qlin_quantize_block_scaled(5, 16, 4, 256, 256, None, 16, 16, 0, None) == q.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_block_scaled(4, 16, 4, 256, 256, 16, 16, 16, 0, None) == q.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_block_scaled(4, 16, 4, 256, 256, None, 16, 24, 0, None) == q.QLIN_ERR_ALIGNMENT
    assert L.qlin_quantize_block_scaled(4, 16, 0, 256, 256, None, 16, 16, 0, None) == q.QLIN_OK


def test_block_scaled_dispatch_rule(q):
    for fmt in (q.QLIN_FMT_MXFP8, q.QLIN_FMT_NVFP4):
        for M in (1, 16, 64, 256, 2048):
            c = q.qlin_dispatch_query(fmt, M, 4096, 2048)
            want = (q.QLIN_VAR_SWAPAB, 32 if M <= 32 else 64) if M <= 64 else (q.QLIN_VAR_PLAIN, 128)
            assert (c["variant"], c["tile_n"], c["k_segments"]) == (*want, 1), (fmt, M, c)
        assert q.qlin_scaled_mm_workspace_size(fmt, 64, 4096, 2048, q.QLIN_VAR_PLAIN) == 0
        ws = q.qlin_scaled_mm_workspace_size(fmt, 64, 4096, 2048, q.QLIN_VAR_SPLITK, 0, 4)
        assert ws == 65536 + 4 * 32 * 128 * 128 * 4
    assert q.block_scaled_sf_bytes(q.QLIN_FMT_MXFP8, 130, 256) == 2 * 2 * 512
    assert q.block_scaled_sf_bytes(q.QLIN_FMT_NVFP4, 130, 256) == 2 * 4 * 512
