"""The quantized linear layer a user calls, composed from the C ABI.

``QuantizedLinear(fmt, weight, bias)`` quantises the bf16 weight once
(per output channel for INT8 / FP8, 128x128 blocks for Block-FP8) with the
library's own kernels, and its ``forward(x)`` runs the hot path through
``qlin_linear``: dynamic activation quantisation (per token, or per 1x128
group) followed by the scaled GEMM with the fused scale / bias / bf16
epilogue, launched as the quantiser's programmatic dependent (QLIN_PDL).  The
one-kernel mode (QLIN_FUSED) is opt-in through ``fused=True``.  Everything runs
in libqlin.so; this module only allocates tensors (through PyTorch's caching
allocator) and passes pointers.
"""
from __future__ import annotations

import torch

from . import qlin


class Workspace:
    """A zero-initialised device buffer for Split-K partials and tickets.

    The GEMM leaves the ticket words zeroed after every call, so the buffer is
    zero-filled only when it is (re)allocated.  Calls that may overlap in time
    (different streams) need separate workspaces.
    """

    def __init__(self, nbytes: int = 0, device="cuda"):
        self.device = torch.device(device)
        self.buf = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)

    def ensure(self, nbytes: int) -> torch.Tensor:
        if nbytes > self.buf.numel():
            self.buf = torch.zeros(int(nbytes), dtype=torch.uint8, device=self.device)
        return self.buf

    def reset_tickets(self):
        """Zero the 64 KiB ticket prefix again (needed after a device-side
        timeout, which can leave a tile's ticket half-counted)."""
        self.buf[: min(self.buf.numel(), TICKET_BYTES)].zero_()


TICKET_BYTES = 65536  # the Split-K ticket prefix of a workspace (include/qlin.h)


def check_device_status(stream=None, workspaces=()):
    """Synchronise and read the library's device status word.  On a device
    timeout, re-zero the ticket prefix of the given workspaces (so the next
    Split-K call counts its arrivals from zero) and raise QlinError."""
    st = qlin.qlin_sync_status(stream)
    if st == qlin.QLIN_ERR_DEVICE_TIMEOUT:
        for ws in workspaces:
            ws.reset_tickets()
        torch.cuda.synchronize()
    if st != qlin.QLIN_OK:
        raise qlin.QlinError(st, "device status")


def quantize_weight(fmt: int, weight: torch.Tensor, stream=None):
    """Quantise a bf16 weight [N, K] on the device; returns (w_q uint8 [N, K], s_w fp32)."""
    assert weight.dtype == torch.bfloat16 and weight.is_cuda and weight.dim() == 2
    N, K = weight.shape
    w_q = torch.empty(N, K, dtype=torch.uint8, device=weight.device)
    if fmt == qlin.QLIN_FMT_FP8_BLOCK:
        s_w = torch.empty((N + 127) // 128, K // 128, dtype=torch.float32, device=weight.device)
        qlin.qlin_quantize_block(weight, 128, w_q, s_w, stream)
    else:
        s_w = torch.empty(N, dtype=torch.float32, device=weight.device)
        qlin.qlin_quantize_per_token(fmt, weight, w_q, s_w, stream)
    return w_q, s_w


def quantize_activation(fmt: int, x: torch.Tensor, stream=None, flags: int = 0):
    """Dynamic activation quantisation; returns (a_q uint8 [M, K], s_a fp32)."""
    M, K = x.shape
    a_q = torch.empty(M, K, dtype=torch.uint8, device=x.device)
    if fmt == qlin.QLIN_FMT_FP8_BLOCK:
        s_a = torch.empty(M, K // 128, dtype=torch.float32, device=x.device)
        qlin.qlin_quantize_block(x, 1, a_q, s_a, stream, flags=flags)
    else:
        s_a = torch.empty(M, dtype=torch.float32, device=x.device)
        qlin.qlin_quantize_per_token(fmt, x, a_q, s_a, stream, flags=flags)
    return a_q, s_a


class QuantizedLinear:
    """y = x W^T + b with W8A8 INT8, FP8 per-token/per-channel or Block-FP8 arithmetic."""

    def __init__(self, fmt: int, weight: torch.Tensor, bias: torch.Tensor | None = None, workspace=None,
                 pdl: bool = True, fused: bool = False):
        self.fmt = fmt
        self.N, self.K = weight.shape
        self.w_q, self.s_w = quantize_weight(fmt, weight)
        # the weights are final once this returns, so later launches may read
        # them early (programmatic dependent launch)
        torch.cuda.current_stream(weight.device).synchronize()
        self.bias = bias
        self.flags = (qlin.QLIN_PDL if pdl else 0) | (qlin.QLIN_FUSED if fused else 0)
        self.workspace = workspace if workspace is not None else Workspace(device=weight.device)

    def forward(self, x: torch.Tensor, stream=None, variant: int = qlin.QLIN_VAR_AUTO, tile_n: int = 0,
                k_segments: int = 0, out: torch.Tensor | None = None) -> torch.Tensor:
        assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.shape[1] == self.K
        assert x.stride(1) == 1
        M = x.shape[0]
        a_q = torch.empty(M, self.K, dtype=torch.uint8, device=x.device)
        if self.fmt == qlin.QLIN_FMT_FP8_BLOCK:
            s_a = torch.empty(M, self.K // 128, dtype=torch.float32, device=x.device)
        else:
            s_a = torch.empty(M, dtype=torch.float32, device=x.device)
        c = out if out is not None else torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
        nbytes = qlin.qlin_scaled_mm_workspace_size(self.fmt, M, self.N, self.K, variant, tile_n, k_segments)
        ws = self.workspace.ensure(nbytes) if nbytes else None
        # quantisation + GEMM in one call (the quantiser, then the GEMM as its
        # programmatic dependent; one kernel where QLIN_FUSED applies)
        qlin.qlin_linear(self.fmt, x, a_q, s_a, self.w_q, self.s_w, self.bias, c, ws, stream, variant=variant,
                         tile_n=tile_n, k_segments=k_segments, flags=self.flags)
        return c

    __call__ = forward
