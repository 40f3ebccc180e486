"""Thin ctypes binding of the C ABI in include/qlin.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: torch tensors are turned into device pointers, the
current CUDA stream into a ``cudaStream_t`` and a non-OK status into a
``QlinError``.  PyTorch is used for device memory and streams only.

The library ``libqlin.so`` is built in-tree by ``build.py``; if it is missing
this module raises ImportError -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("QLIN_LIB", os.path.join(_HERE, "libqlin.so"))

# ------------------------------------------------------------ enums (qlin.h)
QLIN_OK = 0
QLIN_ERR_INVALID_ARG = 1
QLIN_ERR_UNSUPPORTED = 2
QLIN_ERR_ALIGNMENT = 3
QLIN_ERR_WORKSPACE = 4
QLIN_ERR_TABLE_IO = 5
QLIN_ERR_TABLE_FORMAT = 6
QLIN_ERR_TABLE_DEVICE = 7
QLIN_ERR_CUDA = 8
QLIN_ERR_DEVICE_TIMEOUT = 9
QLIN_ERR_NO_DEVICE = 10

QLIN_FMT_INT8 = 0
QLIN_FMT_FP8 = 1
QLIN_FMT_FP8_BLOCK = 2
QLIN_FMT_BF16 = 3  # qlin_matmul_bf16 (and the workspace-size / dispatch queries)
QLIN_FMT_MXFP8 = 4  # block-scaled: qlin_quantize_block_scaled / qlin_block_scaled_mm
QLIN_FMT_NVFP4 = 5

QLIN_VAR_AUTO = 0
QLIN_VAR_PLAIN = 1
QLIN_VAR_SPLITK = 2
QLIN_VAR_SWAPAB = 3
QLIN_VAR_SWAPAB_SPLITK = 4
QLIN_VAR_PAIR = 5

QLIN_OUT_I32ACC = 1
QLIN_PDL = 2
QLIN_SPLITK_CLUSTER = 4  # Swap-AB Split-K: reduce through a thread-block cluster instead of the workspace
QLIN_FUSED = 8  # qlin_linear: the GEMM quantises its own activation rows where it can (one kernel)

VARIANT_NAMES = {QLIN_VAR_AUTO: "auto", QLIN_VAR_PLAIN: "plain", QLIN_VAR_SPLITK: "splitk",
                 QLIN_VAR_SWAPAB: "swapab", QLIN_VAR_SWAPAB_SPLITK: "swapab_splitk", QLIN_VAR_PAIR: "pair"}

# every symbol include/qlin.h declares
EXPORTS = ("qlin_quantize_per_token", "qlin_quantize_block", "qlin_scaled_mm", "qlin_scaled_mm_noalloc", "qlin_linear",
           "qlin_matmul_bf16", "qlin_moe_route", "qlin_moe_quantize_scatter", "qlin_moe_grouped_mm",
           "qlin_moe_act_quantize", "qlin_moe_combine", "qlin_moe_workspace_size", "qlin_moe_forward",
           "qlin_scaled_mm_workspace_size", "qlin_dispatch_table_load", "qlin_dispatch_table_clear",
           "qlin_dispatch_query", "qlin_status_string", "qlin_sync_status", "qlin_abi_version",
           "qlin_selftest_wait_timeout", "qlin_quantize_block_scaled", "qlin_block_scaled_mm")
QLIN_NOALLOC_SCRATCH_BYTES = 8 << 20


class qlin_config(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int32), ("tile_n", ctypes.c_int32), ("k_segments", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("m_max", ctypes.c_int64), ("from_table", ctypes.c_int32)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class QlinError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libqlin.so not found at {LIB_PATH}; build it with "
                      "`python quantized_linear_layers_group_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)
_vp, _i64, _i32, _u32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_size_t
lib.qlin_quantize_per_token.argtypes = [_i32, _vp, _i64, _i64, _i64, _vp, _vp, _u32, _vp]
lib.qlin_quantize_block.argtypes = [_vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _u32, _vp]
lib.qlin_scaled_mm.argtypes = [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _u32, _vp,
                               _sz, _vp]
lib.qlin_scaled_mm_noalloc.argtypes = [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _u32, _vp]
lib.qlin_linear.argtypes = [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _u32,
                            _vp, _sz, _vp]
lib.qlin_matmul_bf16.argtypes = [_i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _u32, _vp, _sz, _vp]
lib.qlin_quantize_block_scaled.argtypes = [_i32, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _u32, _vp]
lib.qlin_block_scaled_mm.argtypes = [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _u32, _vp, _sz, _vp]
lib.qlin_moe_route.argtypes = [_i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _u32, _vp]
lib.qlin_moe_quantize_scatter.argtypes = [_i64, _i64, _i32, _vp, _vp, _vp, _vp, _u32, _vp]
lib.qlin_moe_grouped_mm.argtypes = [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _u32, _vp]
lib.qlin_moe_act_quantize.argtypes = [_i64, _i64, _vp, _vp, _vp, _u32, _vp]
lib.qlin_moe_combine.argtypes = [_i64, _i64, _i32, _vp, _vp, _vp, _vp, _u32, _vp]
lib.qlin_moe_workspace_size.argtypes = [_i64, _i64, _i64, _i32, _i32, ctypes.POINTER(_sz)]
lib.qlin_moe_forward.argtypes = [_i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _u32, _vp, _sz, _vp]
lib.qlin_scaled_mm_workspace_size.argtypes = [_i32, _i32, _i32, _i32, _i64, _i64, _i64, ctypes.POINTER(_sz)]
lib.qlin_dispatch_table_load.argtypes = [ctypes.c_char_p]
lib.qlin_dispatch_table_clear.argtypes = []
lib.qlin_dispatch_query.argtypes = [_i32, _i64, _i64, _i64, ctypes.POINTER(qlin_config)]
lib.qlin_status_string.argtypes = [_i32]
lib.qlin_status_string.restype = ctypes.c_char_p
lib.qlin_sync_status.argtypes = [_vp]
lib.qlin_selftest_wait_timeout.argtypes = [_u32, _vp]
lib.qlin_abi_version.argtypes = []
for _name in EXPORTS:
    if _name != "qlin_status_string":
        getattr(lib, _name).restype = _i32


def status_string(status: int) -> str:
    return lib.qlin_status_string(status).decode()


def _check(status: int, where: str):
    if status != QLIN_OK:
        raise QlinError(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------- entry points
def qlin_quantize_per_token(fmt: int, x, q_out, scale_out, stream=None, *, flags: int = 0, rows=None, cols=None,
                            ld_x=None):
    """Per-token INT8/FP8 quantisation of bf16 x [rows, cols] into q_out / scale_out."""
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[1] if cols is None else cols
    ld_x = (x.stride(0) if x.dim() == 2 else cols) if ld_x is None else ld_x
    _check(lib.qlin_quantize_per_token(fmt, _ptr(x), rows, cols, ld_x, _ptr(q_out), _ptr(scale_out), flags,
                                       _stream(stream)), "qlin_quantize_per_token")


def qlin_quantize_block(x, block_rows: int, q_out, scale_out, stream=None, *, flags: int = 0, block_cols: int = 128,
                        rows=None, cols=None, ld_x=None):
    """Block-FP8 quantisation (1x128 activation groups or 128x128 weight blocks)."""
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[1] if cols is None else cols
    ld_x = (x.stride(0) if x.dim() == 2 else cols) if ld_x is None else ld_x
    _check(lib.qlin_quantize_block(_ptr(x), rows, cols, ld_x, block_rows, block_cols, _ptr(q_out), _ptr(scale_out),
                                   flags, _stream(stream)), "qlin_quantize_block")


def qlin_scaled_mm_workspace_size(fmt: int, M: int, N: int, K: int, variant: int = QLIN_VAR_AUTO, tile_n: int = 0,
                                  k_segments: int = 0) -> int:
    out = _sz(0)
    _check(lib.qlin_scaled_mm_workspace_size(fmt, variant, tile_n, k_segments, M, N, K, ctypes.byref(out)),
           "qlin_scaled_mm_workspace_size")
    return out.value


def qlin_scaled_mm(fmt: int, a_q, s_a, w_q, s_w, bias, c_out, workspace=None, stream=None, *,
                   variant: int = QLIN_VAR_AUTO, tile_n: int = 0, k_segments: int = 0, flags: int = 0,
                   M=None, N=None, K=None, workspace_bytes=None):
    """C = (A_q W_q^T) * s_a * s_w + bias (bf16), or raw INT8 accumulators with QLIN_OUT_I32ACC."""
    M = a_q.shape[0] if M is None else M
    N = w_q.shape[0] if N is None else N
    K = a_q.shape[1] if K is None else K
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qlin_scaled_mm(fmt, variant, tile_n, k_segments, M, N, K, _ptr(a_q), _ptr(s_a), _ptr(w_q), _ptr(s_w),
                              _ptr(bias), _ptr(c_out), flags, _ptr(workspace), workspace_bytes, _stream(stream)),
           "qlin_scaled_mm")


def qlin_scaled_mm_noalloc(fmt: int, a_q, s_a, w_q, s_w, bias, c_out, stream=None, *, variant: int = QLIN_VAR_AUTO,
                           tile_n: int = 0, k_segments: int = 0, flags: int = 0, M=None, N=None, K=None):
    """qlin_scaled_mm without a workspace, for callers that cannot allocate
    device memory: Split-K scratch comes from the library's fixed device array."""
    M = a_q.shape[0] if M is None else M
    N = w_q.shape[0] if N is None else N
    K = a_q.shape[1] if K is None else K
    _check(lib.qlin_scaled_mm_noalloc(fmt, variant, tile_n, k_segments, M, N, K, _ptr(a_q), _ptr(s_a), _ptr(w_q),
                                      _ptr(s_w), _ptr(bias), _ptr(c_out), flags, _stream(stream)),
           "qlin_scaled_mm_noalloc")


def qlin_linear(fmt: int, x, a_q, s_a, w_q, s_w, bias, c_out, workspace=None, stream=None, *,
                variant: int = QLIN_VAR_AUTO, tile_n: int = 0, k_segments: int = 0, flags: int = 0, M=None, N=None,
                K=None, ld_x=None, workspace_bytes=None):
    """Quantise bf16 x and run the scaled GEMM in one call (one kernel with
    QLIN_FUSED where the configuration allows); a_q / s_a receive the
    activation codes and scales."""
    M = x.shape[0] if M is None else M
    K = x.shape[1] if K is None else K
    N = w_q.shape[0] if N is None else N
    ld_x = (x.stride(0) if x.dim() == 2 else K) if ld_x is None else ld_x
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qlin_linear(fmt, variant, tile_n, k_segments, M, N, K, _ptr(x), ld_x, _ptr(a_q), _ptr(s_a), _ptr(w_q),
                           _ptr(s_w), _ptr(bias), _ptr(c_out), flags, _ptr(workspace), workspace_bytes,
                           _stream(stream)), "qlin_linear")


def qlin_matmul_bf16(a, w, bias, c_out, workspace=None, stream=None, *, variant: int = QLIN_VAR_AUTO,
                     tile_n: int = 0, k_segments: int = 0, flags: int = 0, M=None, N=None, K=None,
                     workspace_bytes=None):
    """C = bf16(fp32(a w^T) + bias) for bf16 a [M, K], w [N, K] (batch-invariant)."""
    M = a.shape[0] if M is None else M
    N = w.shape[0] if N is None else N
    K = a.shape[1] if K is None else K
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qlin_matmul_bf16(variant, tile_n, k_segments, M, N, K, _ptr(a), _ptr(w), _ptr(bias), _ptr(c_out),
                                flags, _ptr(workspace), workspace_bytes, _stream(stream)), "qlin_matmul_bf16")


def block_scaled_sf_bytes(fmt: int, rows: int, cols: int) -> int:
    """Bytes of the tiled scale-factor buffer for a [rows, cols] operand."""
    atoms = cols // (128 if fmt == QLIN_FMT_MXFP8 else 64)
    return -(-rows // 128) * atoms * 512


def qlin_quantize_block_scaled(fmt: int, x, q_out, sf_out, g=None, stream=None, *, flags: int = 0, rows=None,
                               cols=None, ld_x=None):
    """MXFP8 / NVFP4 quantisation of bf16 x [rows, cols]: codes into q_out, tiled
    scale factors into sf_out (NVFP4: g is the fp32 [1] decode scale on the device)."""
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[1] if cols is None else cols
    ld_x = (x.stride(0) if x.dim() == 2 else cols) if ld_x is None else ld_x
    _check(lib.qlin_quantize_block_scaled(fmt, _ptr(x), rows, cols, ld_x, _ptr(g), _ptr(q_out), _ptr(sf_out), flags,
                                          _stream(stream)), "qlin_quantize_block_scaled")


def qlin_block_scaled_mm(fmt: int, a_q, a_sf, w_q, w_sf, bias, c_out, g_a=None, g_w=None, workspace=None,
                         stream=None, *, variant: int = QLIN_VAR_AUTO, tile_n: int = 0, k_segments: int = 0,
                         flags: int = 0, M=None, N=None, K=None, workspace_bytes=None):
    """Block-scaled GEMM: C = bf16(acc + bias) (MXFP8) or bf16((acc*g_a)*g_w + bias) (NVFP4)."""
    M = a_q.shape[0] if M is None else M
    N = w_q.shape[0] if N is None else N
    K = a_q.shape[1] * (2 if fmt == QLIN_FMT_NVFP4 else 1) if K is None else K
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qlin_block_scaled_mm(fmt, variant, tile_n, k_segments, M, N, K, _ptr(a_q), _ptr(a_sf), _ptr(w_q),
                                    _ptr(w_sf), _ptr(g_a), _ptr(g_w), _ptr(bias), _ptr(c_out), flags,
                                    _ptr(workspace), workspace_bytes, _stream(stream)), "qlin_block_scaled_mm")


# ------------------------------------------------------------------- MoE
def qlin_moe_route(logits, topk: int, topk_ids, topk_w, rows, offsets, stream=None, *, flags: int = 0):
    T, E = logits.shape
    _check(lib.qlin_moe_route(T, E, topk, _ptr(logits), _ptr(topk_ids), _ptr(topk_w), _ptr(rows), _ptr(offsets),
                              flags, _stream(stream)), "qlin_moe_route")


def qlin_moe_quantize_scatter(x, topk: int, rows, a_q, s_a, stream=None, *, flags: int = 0):
    T, H = x.shape
    _check(lib.qlin_moe_quantize_scatter(T, H, topk, _ptr(x), _ptr(rows), _ptr(a_q), _ptr(s_a), flags,
                                         _stream(stream)), "qlin_moe_quantize_scatter")


def qlin_moe_grouped_mm(fmt: int, E: int, a_q, s_a, offsets, w_q, s_w, c_out, stream=None, *,
                        variant: int = QLIN_VAR_AUTO, tile_n: int = 0, flags: int = 0):
    """Grouped scaled GEMM over experts: w_q [E * N, K], s_w [E * N], c_out [R, N]."""
    R, K = a_q.shape
    N = c_out.shape[1]
    _check(lib.qlin_moe_grouped_mm(fmt, variant, tile_n, E, R, N, K, _ptr(a_q), _ptr(s_a), _ptr(offsets), _ptr(w_q),
                                   _ptr(s_w), _ptr(c_out), flags, _stream(stream)), "qlin_moe_grouped_mm")


def qlin_moe_act_quantize(g, h_q, s_h, stream=None, *, flags: int = 0):
    R, I2 = g.shape
    _check(lib.qlin_moe_act_quantize(R, I2 // 2, _ptr(g), _ptr(h_q), _ptr(s_h), flags, _stream(stream)),
           "qlin_moe_act_quantize")


def qlin_moe_combine(y, topk_w, rows, out, stream=None, *, flags: int = 0):
    T, H = out.shape
    _check(lib.qlin_moe_combine(T, H, topk_w.shape[1], _ptr(y), _ptr(topk_w), _ptr(rows), _ptr(out), flags,
                                _stream(stream)), "qlin_moe_combine")


def qlin_moe_workspace_size(T: int, H: int, I: int, E: int, topk: int) -> int:
    out = _sz(0)
    _check(lib.qlin_moe_workspace_size(T, H, I, E, topk, ctypes.byref(out)), "qlin_moe_workspace_size")
    return out.value


def qlin_moe_forward(x, logits, topk: int, w1_q, s_w1, w2_q, s_w2, out, workspace, stream=None, *, flags: int = 0):
    """The whole FP8 MoE layer (x bf16 [T, H], logits [T, E], w1_q [E, 2I, H], w2_q [E, H, I])."""
    T, H = x.shape
    E = logits.shape[1]
    I = w2_q.shape[-1]
    _check(lib.qlin_moe_forward(T, H, I, E, topk, _ptr(x), _ptr(logits), _ptr(w1_q), _ptr(s_w1), _ptr(w2_q),
                                _ptr(s_w2), _ptr(out), flags, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)), "qlin_moe_forward")


def qlin_dispatch_table_load(path: str):
    _check(lib.qlin_dispatch_table_load(os.fsencode(path)), "qlin_dispatch_table_load")


def qlin_dispatch_table_clear():
    _check(lib.qlin_dispatch_table_clear(), "qlin_dispatch_table_clear")


def qlin_dispatch_query(fmt: int, M: int, N: int, K: int) -> dict:
    cfg = qlin_config()
    _check(lib.qlin_dispatch_query(fmt, M, N, K, ctypes.byref(cfg)), "qlin_dispatch_query")
    return cfg.as_dict()


def qlin_status_string(status: int) -> str:
    return status_string(status)


def qlin_sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return lib.qlin_sync_status(_stream(stream))


def qlin_selftest_wait_timeout(limit_us: int = 20000, stream=None):
    """Enqueue the failure-path self-test: a device wait that must give up
    after limit_us and record QLIN_ERR_DEVICE_TIMEOUT (read it back with
    qlin_sync_status)."""
    _check(lib.qlin_selftest_wait_timeout(limit_us, _stream(stream)), "qlin_selftest_wait_timeout")


def qlin_abi_version() -> int:
    return lib.qlin_abi_version()
