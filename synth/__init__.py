"""Seeded synthetic inputs for the quantized linear layer workloads.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no quantisation, no GEMM) and is the only code shared by
the CPU oracle's tests and the CUDA path's tests and benchmark.

Every tensor is drawn in float32 on the CPU from a ``torch.Generator`` seeded
with ``seed + offset`` and then rounded to bfloat16 (round-to-nearest-even).
Per-tensor seed offsets: A = +0, W = +1, bias = +2, outlier-column pick = +3,
per-row magnitude = +4, mixed-stream draws = +5, batch-invariance filler rows
= +1000 + M.

Workloads (weights W are [N, K], nn.Linear layout; activations A are [M, K]):

* ``int8_smoke``   INT8 W8A8, N = K = 2048, M = 16; A ~ N(0,1) with 1 % of the
  columns (round(0.01 K), drawn without replacement) scaled x20 as outlier
  channels; W ~ N(0, 0.02); no bias.
* ``fp8_attn``     FP8 per-token/per-channel, N = 4096, K = 2048; A and W as
  above; bias ~ N(0, 0.1).
* ``fp8_block_down`` Block-FP8, N = 2048, K = 6144; A ~ N(0,1) with row m
  scaled by exp(U(ln 0.01, ln 100)) (per-token magnitude log-uniform in
  [0.01, 100]); W ~ N(0, 0.02); no bias.
* ``lm_head``      FP8 per-token/per-channel, N = 151936, K = 2048; A ~ N(0,1),
  W ~ N(0, 0.02); no bias, no outliers.
* ``fp8_vocab``    FP8 per-token/per-channel, N = 12288, K = 2048 (batch
  invariance shape); A and W as ``fp8_attn`` without bias.
* ``bf16_*``       bf16 matmul (no quantisation) on the five (N, K) shapes of
  the batch-invariant matmul sweep: vocab 12288 x 2048, down 2048 x 6144, attn
  4096 x 2048, lm_head 151936 x 2048, square 2048 x 2048; M sweep as above;
  A ~ N(0,1), W ~ N(0, 0.02), no bias.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

FMT_INT8 = 0
FMT_FP8 = 1
FMT_FP8_BLOCK = 2
FMT_BF16 = 3
FMT_MXFP8 = 4
FMT_NVFP4 = 5

M_SWEEP = (1, 4, 8, 16, 32, 64, 256, 512, 1024, 2048)
LM_HEAD_M = (1, 8, 64, 256, 1024, 2048)


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: int
    N: int
    K: int
    m_values: tuple
    outliers: bool        # 1 % of activation columns scaled x20
    bias: bool            # bf16 bias ~ N(0, 0.1)
    row_magnitude: bool   # per-row log-uniform magnitude in [0.01, 100]


WORKLOADS = {
    "int8_smoke": Workload("int8_smoke", FMT_INT8, 2048, 2048, (16,), True, False, False),
    "fp8_attn": Workload("fp8_attn", FMT_FP8, 4096, 2048, M_SWEEP, True, True, False),
    "fp8_block_down": Workload("fp8_block_down", FMT_FP8_BLOCK, 2048, 6144, M_SWEEP, False, False, True),
    "lm_head": Workload("lm_head", FMT_FP8, 151936, 2048, LM_HEAD_M, False, False, False),
    "fp8_vocab": Workload("fp8_vocab", FMT_FP8, 12288, 2048, M_SWEEP, True, False, False),
    "int8_square": Workload("int8_square", FMT_INT8, 2048, 2048, M_SWEEP, True, False, False),
    "bf16_vocab": Workload("bf16_vocab", FMT_BF16, 12288, 2048, M_SWEEP, False, False, False),
    "bf16_down": Workload("bf16_down", FMT_BF16, 2048, 6144, M_SWEEP, False, False, False),
    "bf16_attn": Workload("bf16_attn", FMT_BF16, 4096, 2048, M_SWEEP, False, False, False),
    "bf16_lm_head": Workload("bf16_lm_head", FMT_BF16, 151936, 2048, M_SWEEP, False, False, False),
    "bf16_square": Workload("bf16_square", FMT_BF16, 2048, 2048, M_SWEEP, False, False, False),
    # the block-scaled formats (NVFP4 is listed among vLLM's linear-layer formats)
    # on the attention-projection, MLP down-projection and lm_head shapes, with
    # the same activation recipes as the FP8 / Block-FP8 workloads of those shapes
    "mxfp8_attn": Workload("mxfp8_attn", FMT_MXFP8, 4096, 2048, M_SWEEP, True, True, False),
    "nvfp4_attn": Workload("nvfp4_attn", FMT_NVFP4, 4096, 2048, M_SWEEP, True, True, False),
    "mxfp8_down": Workload("mxfp8_down", FMT_MXFP8, 2048, 6144, M_SWEEP, False, False, True),
    "nvfp4_lm_head": Workload("nvfp4_lm_head", FMT_NVFP4, 151936, 2048, LM_HEAD_M, False, False, False),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def normal(shape, std: float, seed: int) -> torch.Tensor:
    """bf16 tensor of N(0, std^2) draws (fp32 draw, RNE to bf16)."""
    t = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def activations(w: Workload, M: int, seed: int = 0, seed_offset: int = 0) -> torch.Tensor:
    """Activation matrix A [M, K] (bf16) for a workload."""
    K = w.K
    a = torch.randn(M, K, generator=_gen(seed + seed_offset), dtype=torch.float32)
    if w.outliers:
        n_out = int(round(0.01 * K))
        cols = torch.randperm(K, generator=_gen(seed + 3))[:n_out]
        a[:, cols] *= 20.0
    if w.row_magnitude:
        u = torch.rand(M, generator=_gen(seed + 4 + seed_offset), dtype=torch.float64)
        lo, hi = math.log(0.01), math.log(100.0)
        mag = torch.exp(lo + (hi - lo) * u).to(torch.float32)
        a *= mag[:, None]
    return a.to(torch.bfloat16)


def weights(w: Workload, seed: int = 0) -> torch.Tensor:
    """Weight matrix W [N, K] (bf16), N(0, 0.02^2)."""
    return normal((w.N, w.K), 0.02, seed + 1)


def bias(w: Workload, seed: int = 0):
    """bf16 bias [N] ~ N(0, 0.1^2), or None."""
    if not w.bias:
        return None
    return normal((w.N,), 0.1, seed + 2)


def invariance_batch(w: Workload, M: int, fixed_rows: torch.Tensor, seed: int = 0) -> torch.Tensor:
    """Batch of M rows whose first min(M, 16) rows are ``fixed_rows``; the rest
    are fresh draws seeded per M."""
    a = activations(w, M, seed=seed, seed_offset=1000 + M)
    r = min(M, fixed_rows.shape[0])
    a[:r] = fixed_rows[:r]
    return a


def mixed_stream(n_calls: int = 1000, seed: int = 0):
    """Seeded list of (workload name, M): M ~ U{1..64} w.p. 0.8, else U{128..2048};
    the shape is uniform over the five (N, K, format) workloads."""
    g = _gen(seed + 5)
    names = ["fp8_attn", "fp8_block_down", "lm_head", "fp8_vocab", "int8_square"]
    out = []
    for _ in range(n_calls):
        name = names[int(torch.randint(len(names), (1,), generator=g))]
        if float(torch.rand(1, generator=g)) < 0.8:
            M = int(torch.randint(1, 65, (1,), generator=g))
        else:
            M = int(torch.randint(128, 2049, (1,), generator=g))
        out.append((name, M))
    return out


# FP8 MoE layer of the benchmark: the page's 192 experts with top-8 routing;
# hidden and expert intermediate sizes are not on the page (4096 and 1536 here)
MOE = {"E": 192, "topk": 8, "H": 4096, "I": 1536, "T": (1, 8, 64, 256, 1024)}


def moe_inputs(T: int, H: int, E: int, seed: int = 0):
    """x bf16 [T, H] ~ N(0,1) and router logits fp32 [T, E] ~ N(0, 4)."""
    x = torch.randn(T, H, generator=_gen(seed + 20), dtype=torch.float32).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=_gen(seed + 21), dtype=torch.float32) * 2.0
    return x, logits


def moe_weight_chunks(E: int, rows: int, cols: int, seed: int, device, chunk: int = 16):
    """Yield (e0, e1, W bf16 [(e1 - e0) * rows, cols] ~ N(0, 0.05^2)) drawn on
    `device` from a seeded generator, a few experts at a time (the full bf16
    weights of the benchmark's MoE would not need to exist at once)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    for e0 in range(0, E, chunk):
        e1 = min(E, e0 + chunk)
        w = torch.randn((e1 - e0) * rows, cols, generator=g, device=device, dtype=torch.float32) * 0.05
        yield e0, e1, w.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a CPU bf16 tensor's bit patterns."""
    import numpy as np

    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
