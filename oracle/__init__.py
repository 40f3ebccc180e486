"""CPU oracle for the quantized linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports, links or executes anything here, and this package
imports nothing from the product.

The arithmetic lives in ``qlin_oracle.c`` (plain C, one separately rounded
binary32 operation per step, exact integer sums); this module only marshals
numpy arrays to it.  bf16 tensors travel as their uint16 bit patterns.

Format codes: 0 = INT8 (W8A8), 1 = FP8 e4m3 per-token/per-channel,
2 = Block-FP8 (1x128 activation groups, 128x128 weight blocks), the three
formats named on the page "Helion in vLLM: A Unified Route to Tunable Linear
Kernels", section "What the integration changes".  ``gemm_bf16`` is the bf16
matmul of the page "[Kernel][Perf] Add Hopper (SM90) tuned config for
batch-invariant persistent matmul" (section "Summary").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

FMT_INT8 = 0
FMT_FP8 = 1
FMT_FP8_BLOCK = 2
FMT_MXFP8 = 4
FMT_NVFP4 = 5

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qlin_oracle.c")
_LIB = os.path.join(_HERE, "libqlin_oracle.so")

# Flags that keep every binary32 operation rounded exactly as written.
CFLAGS = ["-O2", "-std=c99", "-fno-fast-math", "-ffp-contract=off", "-fexcess-precision=standard",
          "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f32p = ctypes.POINTER(ctypes.c_float)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64 = ctypes.c_int64
        lib.qo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.qo_bf16_to_f32.restype = ctypes.c_float
        lib.qo_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.qo_f32_to_bf16.restype = ctypes.c_uint16
        lib.qo_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.qo_e4m3_decode.restype = ctypes.c_float
        lib.qo_e4m3_encode.argtypes = [ctypes.c_float]
        lib.qo_e4m3_encode.restype = ctypes.c_uint8
        lib.qo_e4m3_units.argtypes = [ctypes.c_uint8]
        lib.qo_e4m3_units.restype = ctypes.c_int64
        lib.qo_quantize_per_token.argtypes = [ctypes.c_int, u16p, i64, i64, i64, u8p, f32p]
        lib.qo_quantize_per_token.restype = None
        lib.qo_quantize_block.argtypes = [u16p, i64, i64, i64, i64, i64, u8p, f32p]
        lib.qo_quantize_block.restype = None
        lib.qo_scaled_mm.argtypes = [ctypes.c_int, i64, i64, i64, u8p, f32p, u8p, f32p, u16p,
                                     i64p, i64, i64p, i64, u16p, i32p]
        lib.qo_scaled_mm.restype = ctypes.c_int
        lib.qo_gemm_bf16.argtypes = [i64, i64, i64, u16p, u16p, u16p, i64p, i64, i64p, i64, u16p]
        lib.qo_gemm_bf16.restype = ctypes.c_int
        f32p_ = f32p
        lib.qo_moe_forward.argtypes = [i64, i64, i64, i64, i64, u16p, f32p_, u8p, f32p_, u8p, f32p_, i32p, f32p_,
                                       i32p, i32p, u16p, u8p, f32p_, u16p, u16p]
        lib.qo_moe_forward.restype = ctypes.c_int
        lib.qo_moe_act_quantize.argtypes = [i64, i64, u16p, u8p, f32p_]
        lib.qo_moe_act_quantize.restype = None
        lib.qo_moe_combine.argtypes = [i64, i64, i64, u16p, f32p_, i32p, u16p]
        lib.qo_moe_combine.restype = None
        lib.qo_e8m0_decode.argtypes = [ctypes.c_uint8]
        lib.qo_e8m0_decode.restype = ctypes.c_double
        lib.qo_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.qo_e2m1_decode.restype = ctypes.c_float
        lib.qo_e2m1_encode.argtypes = [ctypes.c_float]
        lib.qo_e2m1_encode.restype = ctypes.c_uint8
        lib.qo_quantize_mxfp8.argtypes = [u16p, i64, i64, i64, u8p, u8p]
        lib.qo_quantize_mxfp8.restype = None
        lib.qo_quantize_nvfp4.argtypes = [u16p, i64, i64, i64, ctypes.c_float, u8p, u8p]
        lib.qo_quantize_nvfp4.restype = None
        lib.qo_gemm_block_scaled.argtypes = [ctypes.c_int, i64, i64, i64, u8p, u8p, u8p, u8p, ctypes.c_float,
                                             ctypes.c_float, u16p, i64p, i64, i64p, i64, u16p]
        lib.qo_gemm_block_scaled.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _bits(x) -> np.ndarray:
    """bf16 input as a contiguous uint16 array (accepts torch bf16 or uint16 numpy)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # plumbing only: reinterpret bf16 storage as raw bits

    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------------------ scalars --
def bf16_to_f32(b: int) -> float:
    return _load().qo_bf16_to_f32(b)


def f32_to_bf16(f: float) -> int:
    return _load().qo_f32_to_bf16(f)


def e4m3_decode(code: int) -> float:
    return _load().qo_e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    return _load().qo_e4m3_encode(v)


def e4m3_units(code: int) -> int:
    return _load().qo_e4m3_units(code)


# --------------------------------------------------------------- quantisers --
def quantize_per_token(fmt: int, x) -> tuple[np.ndarray, np.ndarray]:
    """Per-token dynamic quantisation of a bf16 [rows, cols] matrix.

    Returns (q uint8 [rows, cols] -- int8 bits for INT8, e4m3 codes for FP8 --,
    s float32 [rows]).
    """
    assert fmt in (FMT_INT8, FMT_FP8)
    xb = _bits(x)
    rows, cols = xb.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows,), np.float32)
    _load().qo_quantize_per_token(fmt, _ptr(xb, ctypes.c_uint16), rows, cols, cols,
                                  _ptr(q, ctypes.c_uint8), _ptr(s, ctypes.c_float))
    return q, s


def quantize_block(x, block_rows: int, block_cols: int = 128) -> tuple[np.ndarray, np.ndarray]:
    """Block-FP8 quantisation; scales [ceil(rows/block_rows), cols/block_cols]."""
    xb = _bits(x)
    rows, cols = xb.shape
    assert cols % block_cols == 0
    q = np.empty((rows, cols), np.uint8)
    s = np.empty(((rows + block_rows - 1) // block_rows, cols // block_cols), np.float32)
    _load().qo_quantize_block(_ptr(xb, ctypes.c_uint16), rows, cols, cols, block_rows, block_cols,
                              _ptr(q, ctypes.c_uint8), _ptr(s, ctypes.c_float))
    return q, s


# -------------------------------------------------------------- scaled GEMM --
def scaled_mm(fmt: int, a_q: np.ndarray, s_a: np.ndarray, w_q: np.ndarray, s_w: np.ndarray,
              bias=None, m_idx=None, n_idx=None, want_acc: bool = False):
    """C = (A_q W_q^T) * s_a * s_w + bias as bf16 bits, optionally on a row/column sample.

    Returns uint16 C [len(m_idx), len(n_idx)] (or [M, N]); with want_acc (INT8)
    also the int32 accumulators.
    """
    a_q = np.ascontiguousarray(a_q, dtype=np.uint8)
    w_q = np.ascontiguousarray(w_q, dtype=np.uint8)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, K = a_q.shape
    N, K2 = w_q.shape
    assert K == K2 and K % 128 == 0
    if fmt == FMT_FP8_BLOCK:
        assert bias is None
        assert s_a.shape == (M, K // 128) and s_w.shape == ((N + 127) // 128, K // 128)
    else:
        assert s_a.shape == (M,) and s_w.shape == (N,)
    bb = None if bias is None else _bits(bias).reshape(-1)
    mi = None if m_idx is None else np.ascontiguousarray(m_idx, dtype=np.int64)
    ni = None if n_idx is None else np.ascontiguousarray(n_idx, dtype=np.int64)
    mc = M if mi is None else len(mi)
    nc = N if ni is None else len(ni)
    c = np.empty((mc, nc), np.uint16)
    acc = np.empty((mc, nc), np.int32) if want_acc else None
    rc = _load().qo_scaled_mm(fmt, M, N, K, _ptr(a_q, ctypes.c_uint8), _ptr(s_a, ctypes.c_float),
                              _ptr(w_q, ctypes.c_uint8), _ptr(s_w, ctypes.c_float),
                              _ptr(bb, ctypes.c_uint16), _ptr(mi, ctypes.c_int64), mc,
                              _ptr(ni, ctypes.c_int64), nc, _ptr(c, ctypes.c_uint16),
                              _ptr(acc, ctypes.c_int32))
    if rc == -1:
        raise OverflowError("INT8 accumulator left the int32 range")
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return (c, acc) if want_acc else c


def gemm_bf16(a, w, bias=None, m_idx=None, n_idx=None) -> np.ndarray:
    """C = bf16(fp32(A W^T) + bias) for bf16 A [M, K] and W [N, K] (torch bf16
    or uint16 bit arrays), optionally on a row / column sample; returns uint16
    bits [len(m_idx), len(n_idx)] (or [M, N])."""
    ab, wb = _bits(a), _bits(w)
    M, K = ab.shape
    N, K2 = wb.shape
    assert K == K2
    bb = None if bias is None else _bits(bias).reshape(-1)
    mi = None if m_idx is None else np.ascontiguousarray(m_idx, dtype=np.int64)
    ni = None if n_idx is None else np.ascontiguousarray(n_idx, dtype=np.int64)
    mc = M if mi is None else len(mi)
    nc = N if ni is None else len(ni)
    c = np.empty((mc, nc), np.uint16)
    rc = _load().qo_gemm_bf16(M, N, K, _ptr(ab, ctypes.c_uint16), _ptr(wb, ctypes.c_uint16),
                              _ptr(bb, ctypes.c_uint16), _ptr(mi, ctypes.c_int64), mc, _ptr(ni, ctypes.c_int64), nc,
                              _ptr(c, ctypes.c_uint16))
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return c


def moe_forward(x, logits: np.ndarray, w1_q: np.ndarray, s_w1: np.ndarray, w2_q: np.ndarray, s_w2: np.ndarray,
                topk: int) -> dict:
    """The FP8 MoE layer step by step (see qo_moe_forward): x bf16 [T, H],
    logits fp32 [T, E], W1_q [E, 2I, H] e4m3 codes with s_w1 [E, 2I], W2_q
    [E, H, I] with s_w2 [E, H].  Returns a dict of numpy arrays: topk_ids,
    topk_w, rows, offsets, g (bf16 bits [R, 2I]), h_q, s_h, y (bf16 bits
    [R, H]) and out (bf16 bits [T, H])."""
    xb = _bits(x)
    T, H = xb.shape
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    E = logits.shape[1]
    w1_q = np.ascontiguousarray(w1_q, dtype=np.uint8)
    w2_q = np.ascontiguousarray(w2_q, dtype=np.uint8)
    s_w1 = np.ascontiguousarray(s_w1, dtype=np.float32)
    s_w2 = np.ascontiguousarray(s_w2, dtype=np.float32)
    I = w2_q.shape[2]
    assert w1_q.shape == (E, 2 * I, H) and w2_q.shape == (E, H, I)
    assert s_w1.shape == (E, 2 * I) and s_w2.shape == (E, H)
    R = T * topk
    o = {"topk_ids": np.zeros((T, topk), np.int32), "topk_w": np.zeros((T, topk), np.float32),
         "rows": np.zeros((T, topk), np.int32), "offsets": np.zeros(E + 1, np.int32),
         "g": np.zeros((R, 2 * I), np.uint16), "h_q": np.zeros((R, I), np.uint8), "s_h": np.zeros(R, np.float32),
         "y": np.zeros((R, H), np.uint16), "out": np.zeros((T, H), np.uint16)}
    rc = _load().qo_moe_forward(T, H, I, E, topk, _ptr(xb, ctypes.c_uint16), _ptr(logits, ctypes.c_float),
                                _ptr(w1_q, ctypes.c_uint8), _ptr(s_w1, ctypes.c_float), _ptr(w2_q, ctypes.c_uint8),
                                _ptr(s_w2, ctypes.c_float), _ptr(o["topk_ids"], ctypes.c_int32),
                                _ptr(o["topk_w"], ctypes.c_float), _ptr(o["rows"], ctypes.c_int32),
                                _ptr(o["offsets"], ctypes.c_int32), _ptr(o["g"], ctypes.c_uint16),
                                _ptr(o["h_q"], ctypes.c_uint8), _ptr(o["s_h"], ctypes.c_float),
                                _ptr(o["y"], ctypes.c_uint16), _ptr(o["out"], ctypes.c_uint16))
    if rc != 0:
        raise RuntimeError(f"oracle moe_forward failed ({rc})")
    return o


def moe_act_quantize(g: np.ndarray):
    """The MoE activation step alone: g bf16 bits [R, 2I] -> (h_q [R, I], s_h [R])."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    R, I2 = g.shape
    hq = np.zeros((R, I2 // 2), np.uint8)
    sh = np.zeros(R, np.float32)
    _load().qo_moe_act_quantize(R, I2 // 2, _ptr(g, ctypes.c_uint16), _ptr(hq, ctypes.c_uint8), _ptr(sh, ctypes.c_float))
    return hq, sh


def moe_combine(y: np.ndarray, w: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """The MoE top-k reduction alone: y bf16 bits [R, H], w [T, k], rows [T, k] -> out bits [T, H]."""
    y = np.ascontiguousarray(y, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    T, k = w.shape
    H = y.shape[1]
    out = np.zeros((T, H), np.uint16)
    _load().qo_moe_combine(T, H, k, _ptr(y, ctypes.c_uint16), _ptr(w, ctypes.c_float), _ptr(rows, ctypes.c_int32),
                           _ptr(out, ctypes.c_uint16))
    return out


def bf16_bits_to_f32(c: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 values (exact)."""
    return (c.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------ block-scaled formats --
# MXFP8 (OCP Microscaling v1.0: E4M3 elements, 32-element blocks along K, E8M0
# scales) and NVFP4 (E2M1 elements, 16-element blocks, E4M3 block scales and a
# per-tensor fp32 decode scale g).  NVFP4 is listed among vLLM's formats on the
# page "Helion in vLLM: A Unified Route to Tunable Linear Kernels"
# (introduction); the readings are stated in qlin_oracle.c.
def e8m0_decode(code: int) -> float:
    return _load().qo_e8m0_decode(code)


def e2m1_decode(code: int) -> float:
    return _load().qo_e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    return _load().qo_e2m1_encode(v)


def quantize_mxfp8(x) -> tuple[np.ndarray, np.ndarray]:
    """MXFP8 codes uint8 [rows, cols] and E8M0 scale codes uint8 [rows, cols/32]."""
    xb = _bits(x)
    rows, cols = xb.shape
    assert cols % 32 == 0
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // 32), np.uint8)
    _load().qo_quantize_mxfp8(_ptr(xb, ctypes.c_uint16), rows, cols, cols, _ptr(q, ctypes.c_uint8),
                              _ptr(sf, ctypes.c_uint8))
    return q, sf


def quantize_nvfp4(x, g: float) -> tuple[np.ndarray, np.ndarray]:
    """NVFP4 packed codes uint8 [rows, cols/2] (element 2i in the low nibble) and
    E4M3 block-scale codes uint8 [rows, cols/16], for the per-tensor decode scale g."""
    xb = _bits(x)
    rows, cols = xb.shape
    assert cols % 16 == 0 and g > 0
    q = np.empty((rows, cols // 2), np.uint8)
    sf = np.empty((rows, cols // 16), np.uint8)
    _load().qo_quantize_nvfp4(_ptr(xb, ctypes.c_uint16), rows, cols, cols, float(np.float32(g)),
                              _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8))
    return q, sf


def gemm_block_scaled(fmt: int, a_q: np.ndarray, a_sf: np.ndarray, w_q: np.ndarray, w_sf: np.ndarray,
                      g_a: float = 1.0, g_w: float = 1.0, bias=None, m_idx=None, n_idx=None) -> np.ndarray:
    """Block-scaled GEMM (FMT_MXFP8 or FMT_NVFP4) as bf16 bits [len(m_idx), len(n_idx)]."""
    assert fmt in (FMT_MXFP8, FMT_NVFP4)
    a_q = np.ascontiguousarray(a_q, dtype=np.uint8)
    w_q = np.ascontiguousarray(w_q, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    w_sf = np.ascontiguousarray(w_sf, dtype=np.uint8)
    M, N = a_q.shape[0], w_q.shape[0]
    K = a_q.shape[1] * (2 if fmt == FMT_NVFP4 else 1)
    bs = 16 if fmt == FMT_NVFP4 else 32
    assert w_q.shape[1] == a_q.shape[1] and K % bs == 0
    assert a_sf.shape == (M, K // bs) and w_sf.shape == (N, K // bs)
    bb = None if bias is None else _bits(bias).reshape(-1)
    mi = None if m_idx is None else np.ascontiguousarray(m_idx, dtype=np.int64)
    ni = None if n_idx is None else np.ascontiguousarray(n_idx, dtype=np.int64)
    mc = M if mi is None else len(mi)
    nc = N if ni is None else len(ni)
    c = np.empty((mc, nc), np.uint16)
    rc = _load().qo_gemm_block_scaled(fmt, M, N, K, _ptr(a_q, ctypes.c_uint8), _ptr(a_sf, ctypes.c_uint8),
                                      _ptr(w_q, ctypes.c_uint8), _ptr(w_sf, ctypes.c_uint8),
                                      float(np.float32(g_a)), float(np.float32(g_w)), _ptr(bb, ctypes.c_uint16),
                                      _ptr(mi, ctypes.c_int64), mc, _ptr(ni, ctypes.c_int64), nc,
                                      _ptr(c, ctypes.c_uint16))
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return c
