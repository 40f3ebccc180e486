"""Shared test helpers: run the CUDA path through the C ABI, run the oracle on
the same seeded inputs, compare.  (Imports the product binding and the oracle
side by side -- tests are the one place allowed to hold both.)"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_REL = 1e-2   # FP8 / Block-FP8 bf16 outputs: |d| <= 1e-2 |ref| + 1e-3
TOL_ABS = 1e-3


def bits_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint8)


def assert_fp_parity(c_gpu_bits: np.ndarray, c_ref_bits: np.ndarray, what: str = ""):
    g = oracle.bf16_bits_to_f32(c_gpu_bits).astype(np.float64)
    r = oracle.bf16_bits_to_f32(c_ref_bits).astype(np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    bad = np.abs(g - r) > TOL_REL * np.abs(r) + TOL_ABS
    if bad.any():
        idx = np.argwhere(bad)[:8]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside |d|<=1e-2|ref|+1e-3; "
                             f"first {idx.tolist()} gpu={g[bad][:8]} ref={r[bad][:8]}")


def assert_parity(fmt: int, c_gpu_bits: np.ndarray, c_ref_bits: np.ndarray, what: str = ""):
    if fmt == oracle.FMT_INT8:
        if not np.array_equal(c_gpu_bits, c_ref_bits):
            bad = np.argwhere(c_gpu_bits != c_ref_bits)
            raise AssertionError(f"{what}: INT8 bf16 output not bit-exact at {len(bad)} places, first "
                                 f"{bad[:8].tolist()}")
    else:
        assert_fp_parity(c_gpu_bits, c_ref_bits, what)


def oracle_quantize(fmt: int, x: torch.Tensor, is_weight: bool):
    if fmt == oracle.FMT_FP8_BLOCK:
        return oracle.quantize_block(x, 128 if is_weight else 1, 128)
    return oracle.quantize_per_token(fmt, x)


def gpu_quantize(fmt: int, x_dev: torch.Tensor, is_weight: bool):
    from quantized_linear_layers_group_b200 import linear

    if is_weight:
        return linear.quantize_weight(fmt, x_dev)
    return linear.quantize_activation(fmt, x_dev)


def gpu_gemm(fmt, a_q, s_a, w_q, s_w, bias_dev, variant=0, tile_n=0, k_segments=0, out_i32=False,
             workspace=None, flags=0):
    from quantized_linear_layers_group_b200 import qlin

    M, K = a_q.shape
    N = w_q.shape[0]
    if out_i32:
        c = torch.empty(M, N, dtype=torch.int32, device=a_q.device)
    else:
        c = torch.empty(M, N, dtype=torch.bfloat16, device=a_q.device)
    nbytes = qlin.qlin_scaled_mm_workspace_size(fmt, M, N, K, variant, tile_n, k_segments)
    ws = None
    if nbytes:
        ws = workspace if workspace is not None and workspace.numel() >= nbytes else \
            torch.zeros(nbytes, dtype=torch.uint8, device=a_q.device)
    qlin.qlin_scaled_mm(fmt, a_q, s_a, w_q, s_w, bias_dev, c, ws, variant=variant, tile_n=tile_n,
                        k_segments=k_segments, flags=flags | (qlin.QLIN_OUT_I32ACC if out_i32 else 0))
    return c


def check_status():
    from quantized_linear_layers_group_b200 import qlin

    st = qlin.qlin_sync_status()
    assert st == 0, f"device status {st}: {qlin.qlin_status_string(st)}"


# ------------------------------------------------------ block-scaled formats
# The GPU keeps scale factors in the tiled layout its tensor cores read (512-byte
# atoms of 128 rows x 4 scales, row r's four bytes at (r%32)*16 + ((r/32)%4)*4);
# the oracle keeps them plain, [rows][K / block].  These two functions only move
# bytes between the layouts.
def _sf_index(rows: int, nsf: int) -> np.ndarray:
    atoms = nsf // 4
    r = np.arange(rows)[:, None]
    j = np.arange(nsf)[None, :]
    return ((r // 128) * atoms + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4


def sf_tile(plain: np.ndarray) -> np.ndarray:
    rows, nsf = plain.shape
    out = np.zeros(-(-rows // 128) * (nsf // 4) * 512, np.uint8)
    out[_sf_index(rows, nsf)] = plain
    return out


def sf_untile(tiled: np.ndarray, rows: int, nsf: int) -> np.ndarray:
    return tiled[_sf_index(rows, nsf)]


def gpu_block_scaled_mm(fmt, a_q, a_sf, w_q, w_sf, bias_dev=None, g_a=None, g_w=None, variant=0, tile_n=0,
                        k_segments=0, flags=0):
    from quantized_linear_layers_group_b200 import qlin

    M = a_q.shape[0]
    N = w_q.shape[0]
    K = a_q.shape[1] * (2 if fmt == qlin.QLIN_FMT_NVFP4 else 1)
    c = torch.empty(M, N, dtype=torch.bfloat16, device=a_q.device)
    nbytes = qlin.qlin_scaled_mm_workspace_size(fmt, M, N, K, variant, tile_n, k_segments)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=a_q.device) if nbytes else None
    qlin.qlin_block_scaled_mm(fmt, a_q, a_sf, w_q, w_sf, bias_dev, c, g_a, g_w, ws, variant=variant, tile_n=tile_n,
                              k_segments=k_segments, flags=flags)
    return c
