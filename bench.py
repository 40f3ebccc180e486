"""Benchmark of the quantized linear layer hot path on B200.

One step = one pass of the whole hot path over one batch per M of the
workload's M sweep: dynamic activation quantisation (per token, or per 1x128
group for Block-FP8) followed by the scaled GEMM with the variant the dispatch
table (or the built-in rule) picks for that (M, N, K, format).  Each GEMM of a
step reads a different copy of the quantised weight, rotating through enough
copies that the weights read between two uses of one copy exceed 2x the L2
(126 MB), and each step reads its own set of activation copies, so every
weight byte and every activation byte comes from HBM.

Prints one JSON line (rank 0):
  value       whole-job GEMM TFLOP/s over the device-timed steps of the
              headline workload (FP8 attention projection, M sweep), inputs
              resident, one CUDA graph per step
  e2e         the same steps through the same C ABI calls with the bf16
              activations copied in from pinned host memory and C copied back
              (eager launches; the copies run on two copy streams ordered by
              events, so they overlap each other and the kernels)
  roofline    the dominant kernel of the headline workload (largest share of
              device time) against the measured HBM / tensor peak
  per_m       per (M, N, K, format) of the headline workload: GEMM and
              quantiser time, TFLOP/s, HBM GB/s, roofline fraction
  workloads   the same per-M table, step time and dominant-kernel roofline for
              every workload of the metric (INT8 smoke, FP8 attention,
              Block-FP8 down projection, lm_head, FP8 12288 x 2048, INT8 2048^2),
              the bf16 matmul on its five shapes, the MXFP8 / NVFP4 workloads
              and the FP8 MoE layer
  tensor_peaks  dense FP8 (torch._scaled_mm) and INT8 (torch._int_mm) library
              GEMM throughput at 8192^3 measured on this GPU (burst, best of 10)
  cpu_baseline  the CPU oracle on a bounded sample (rank 0, N = 1 only), on one
              thread and on every host core

  --impl reference  times the CPU oracle as the reference arm instead.
  --fused           runs each layer through qlin_linear with QLIN_FUSED: one
                    kernel where the configuration is Swap-AB (the GEMM
                    quantises its own activation rows), else the same two
                    kernels; gpu_launches counts what is launched.

Multi-GPU: one process per GPU (torchrun); every rank runs the same
independent step on its own GPU (no data-path collective; weak scaling); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "scaled_mm TFLOPS & HBM GB/s vs roofline, per (M,N,K,format), 1×B200"
L2_BYTES = 126 * 1024 * 1024
FMT_NAME = {0: "int8", 1: "fp8", 2: "fp8_block", 3: "bf16", 4: "mxfp8", 5: "nvfp4"}
DTYPE = {0: "int8 (int32 accumulate)", 1: "fp8_e4m3 (fp32 accumulate)", 2: "fp8_e4m3 block-scaled (fp32 accumulate)",
         3: "bf16 (fp32 accumulate)", 4: "mxfp8 e4m3 / e8m0 (fp32 accumulate)",
         5: "nvfp4 e2m1 / e4m3 (fp32 accumulate)"}
BS_FMTS = (4, 5)  # block-scaled formats: scale factors applied inside the tensor core
HEADLINE = "fp8_attn"
# every workload of the metric: the headline plus the parity configurations
ALL_WORKLOADS = ("fp8_attn", "int8_smoke", "fp8_block_down", "lm_head", "fp8_vocab", "int8_square")
# the bf16 batch-invariant matmul on the five shapes of its sweep (no quantisation step)
BF16_WORKLOADS = ("bf16_vocab", "bf16_down", "bf16_attn", "bf16_lm_head", "bf16_square")
# the block-scaled formats MXFP8 / NVFP4 on the attention, down-projection and lm_head shapes
BS_WORKLOADS = ("mxfp8_attn", "nvfp4_attn", "mxfp8_down", "nvfp4_lm_head")


# ------------------------------------------------------------------ peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def measure_tensor_peaks(device, n=8192, reps=10):
    """Dense 8-bit library GEMM throughput on this GPU: torch._scaled_mm (e4m3,
    bf16 out) and torch._int_mm (int8, int32 out) at n^3, each call timed with
    CUDA events on the current stream, best of `reps` (burst)."""
    out = {"n": n, "reps": reps, "how": "best of 10 single calls, CUDA events, 2*n^3 flop"}
    a8 = torch.randn(n, n, device=device).to(torch.float8_e4m3fn)
    b8 = torch.randn(n, n, device=device).to(torch.float8_e4m3fn)
    one = torch.ones((), device=device, dtype=torch.float32)
    i8a = torch.randint(-127, 128, (n, n), device=device, dtype=torch.int8)
    i8b = torch.randint(-127, 128, (n, n), device=device, dtype=torch.int8)
    calls = {"fp8_tflops": lambda: torch._scaled_mm(a8, b8.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
             "int8_tops": lambda: torch._int_mm(i8a, i8b.t())}
    for key, fn in calls.items():
        try:
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            best = float("inf")
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                e1.synchronize()
                best = min(best, e0.elapsed_time(e1) / 1e3)
            out[key] = 2.0 * n ** 3 / best / 1e12
        except Exception as exc:  # a library without the kernel on this build: say so
            out[key] = None
            out[key + "_error"] = f"{type(exc).__name__}: {exc}"[:200]
    del a8, b8, i8a, i8b
    torch.cuda.synchronize()
    return out


def tensor_peak(peaks, fmt, tpk=None):
    """Dense tensor peak for a kernel timed in isolation (burst): bf16 the
    measured cuBLAS bf16 burst figure; 8-bit the measured library figure for
    the format when there is one, else the bf16 burst peak x 2 (the nominal
    8-bit / bf16 ratio)."""
    if fmt == 3:
        return peaks["bf16_tflops"], f"{peaks['source']} bf16_tflops (cuBLAS bf16 burst)"
    if fmt == 5:  # fp4 operands: twice the 8-bit rate (nominal 9 / 4.5 PFLOP/s dense)
        p8, src8 = tensor_peak(peaks, 1, tpk)
        return 2.0 * p8, src8 + " x 2 (nominal fp4 / fp8 ratio)"
    if tpk is not None:
        v = tpk.get("int8_tops" if fmt == 0 else "fp8_tflops")
        if v:
            return v, ("measured torch._int_mm int8" if fmt == 0 else "measured torch._scaled_mm e4m3") + " burst"
    return 2.0 * peaks["bf16_tflops"], f"{peaks['source']} bf16 burst x 2 (nominal 8-bit / bf16 ratio)"


def gemm_flops(M, N, K):
    return 2.0 * M * N * K


def gemm_bytes(M, N, K, fmt):
    """Algorithmic bytes per GEMM launch: the 8-bit operands A and W (as the
    roofline is defined on), plus scales, bias and the bf16 output separately."""
    elt = {3: 2.0, 5: 0.5}.get(fmt, 1.0)
    ab = int((M * K + N * K) * elt)
    if fmt in BS_FMTS:  # one scale byte per 32 (MXFP8) or 16 (NVFP4) elements
        scales = (M + N) * K // (32 if fmt == 4 else 16)
    else:
        scales = (M * (K // 128) + (N // 128) * (K // 128)) * 4 if fmt == 2 else (0 if fmt == 3 else (M + N) * 4)
    extra = scales + 2 * M * N
    return ab, extra


def quant_bytes(M, K, fmt):
    if fmt == 3:
        return 0  # bf16: no quantisation step
    if fmt == 4:
        return 2 * M * K + M * K + M * K // 32
    if fmt == 5:
        return 2 * M * K + M * K // 2 + M * K // 16
    return 2 * M * K + M * K + (M * (K // 128) if fmt == 2 else M) * 4


def measured_traffic(workload, fmt, M, N, K, cfg):
    """DRAM bytes (read + write) of one GEMM launch from the committed ncu
    record, or None when there is none for this launch or the kernel source
    has changed since it was taken."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    src = os.path.join(ROOT, "quantized_linear_layers_group_b200", "csrc", "gemm.cu")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if rec.get("gemm_source_sha256_16") != sha:
        return None
    from quantized_linear_layers_group_b200 import qlin

    for e in rec.get("entries", []):
        if (e["workload"], e["M"], e["N"], e["K"], e["format"]) == (workload, M, N, K, FMT_NAME[fmt]) and \
                e["variant"] == qlin.VARIANT_NAMES[cfg["variant"]] and e["tile_n"] == cfg["tile_n"]:
            return e["dram_read_bytes"] + e["dram_write_bytes"]
    return None


def kernel_of(fmt, cfg):
    """The compiled GEMM kernel a configuration runs, named as in the ncu
    launch list: qlin_gemm_kernel<format, swap_ab, tile_n, cluster, fused, pair>.
    Split-K shares the kernel of its orientation (the split is a run-time
    argument)."""
    from quantized_linear_layers_group_b200 import qlin

    v = cfg["variant"]
    swap = int(v in (qlin.QLIN_VAR_SWAPAB, qlin.QLIN_VAR_SWAPAB_SPLITK))
    pair = int(v == qlin.QLIN_VAR_PAIR)
    return f"qlin_gemm_kernel<{fmt}, {swap}, {cfg['tile_n']}, 0, 0, {pair}>"


def kernel_roofline(per_m, configs, fmt, N, K, hbm, tc_peak, total_dev_us):
    """Roofline of the dominant GEMM kernel: launches grouped by the kernel they
    run, the group with the largest share of the step's device time.  achieved
    = mean algorithmic bytes (or flops) per launch / mean launch duration; the
    bound is the larger of the group's summed HBM and tensor roofline times."""
    groups = {}
    for r in per_m:
        groups.setdefault(kernel_of(fmt, configs[r["M"]]), []).append(r)
    name, rows = max(groups.items(), key=lambda kv: sum(r["gemm_us"] for r in kv[1]))
    ms = [r["M"] for r in rows]
    t_mean = statistics.mean(r["gemm_us"] for r in rows) * 1e-6
    ab = [gemm_bytes(M, N, K, fmt)[0] for M in ms]
    fl = [gemm_flops(M, N, K) for M in ms]
    t_hbm = sum(b / (hbm * 1e9) for b in ab)
    t_tc = sum(f / (tc_peak * 1e12) for f in fl)
    out = {"kernel": name, "m_values": ms, "launches_per_step": len(ms),
           "share": sum(r["gemm_us"] for r in rows) / total_dev_us, "mean_launch_us": t_mean * 1e6}
    if t_hbm >= t_tc:
        a = statistics.mean(ab) / t_mean / 1e9
        out.update({"bound": "hbm", "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm})
    else:
        a = statistics.mean(fl) / t_mean / 1e12
        out.update({"bound": "tensor", "achieved": a, "peak": tc_peak, "unit": "TFLOP/s", "frac": a / tc_peak})
    return out


def measured_traffic_kernel(workload, fmt, N, K, configs, ms):
    """DRAM bytes of one launch of the dominant kernel, from the committed ncu
    record of one of its launches (the first M of the group that has one)."""
    for M in ms:
        t = measured_traffic(workload, fmt, M, N, K, configs[M])
        if t is not None:
            return t
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# --------------------------------------------------------------- the step
class HotPath:
    """Device buffers and the per-step launch sequence for one workload.

    Weights rotate per GEMM launch through `n_copies` copies, and each step
    (one CUDA graph) reads its own set of activation copies, so that the bytes
    read between two uses of one copy exceed 2x L2 for both."""

    def __init__(self, workload: synth.Workload, m_values, device, seed=0, fused=False):
        from quantized_linear_layers_group_b200 import linear, qlin

        self.qlin, self.linear = qlin, linear
        self.w = workload
        self.fmt = workload.fmt
        # fused: each M goes through qlin_linear with QLIN_FUSED (one kernel
        # where the configuration is Swap-AB, else the quantiser + the GEMM)
        self.fused = fused and self.fmt in (0, 1, 2)
        self.ms = list(m_values)
        self.device = device
        N, K = workload.N, workload.K
        w_cpu = synth.weights(workload, seed)
        b_cpu = synth.bias(workload, seed)
        w_dev = w_cpu.to(device)
        self.g_w = self.g_a = None
        if self.fmt == 3:  # bf16: the weight is used as it is
            w_q, s_w = w_dev, None
        elif self.fmt in BS_FMTS:  # offline: codes and tiled scale factors (NVFP4: decode scale amax / (6 * 448))
            if self.fmt == 5:
                self.g_w = (w_dev.float().abs().max() / 2688.0).reshape(1).contiguous()
            w_q = torch.empty(N, K // 2 if self.fmt == 5 else K, dtype=torch.uint8, device=device)
            s_w = torch.empty(qlin.block_scaled_sf_bytes(self.fmt, N, K), dtype=torch.uint8, device=device)
            qlin.qlin_quantize_block_scaled(self.fmt, w_dev, w_q, s_w, self.g_w)
            del w_dev
        else:
            w_q, s_w = linear.quantize_weight(self.fmt, w_dev)
            del w_dev
        self.bias = None if b_cpu is None else b_cpu.to(device)
        wbytes = N * K * {3: 2, 5: 0.5}.get(self.fmt, 1)
        # enough weight copies that the bytes read between two uses of a copy exceed 2x L2
        self.n_copies = max(2, math.ceil(2 * L2_BYTES / wbytes) + 1)
        self.w_copies = [(w_q if i == 0 else w_q.clone(), s_w if i == 0 or s_w is None else s_w.clone())
                         for i in range(self.n_copies)]
        # graphs per rotation of the weight copies; each graph = one step with its own activation set
        self.n_graphs = max(1, math.ceil(self.n_copies / len(self.ms)))
        step_bytes = len(self.ms) * wbytes + sum(2 * M * K for M in self.ms)
        self.n_act_sets = max(self.n_graphs, math.ceil(2 * L2_BYTES / step_bytes) + 1)
        a_cpu = {M: synth.activations(workload, M, seed=seed) for M in self.ms}
        self.a_sets = [{M: a_cpu[M].to(device) for M in self.ms} for _ in range(self.n_act_sets)]
        if self.fmt == 5:  # NVFP4 activations: a static decode scale, calibrated once on these inputs
            amax = max(float(a.float().abs().max()) for a in a_cpu.values())
            self.g_a = torch.tensor([amax / 2688.0], dtype=torch.float32, device=device)
        self.a_cpu = a_cpu
        self.a_host = None  # pinned copies, made by the first end-to-end step
        self.act = 0  # activation set of the step being issued
        self.a_q, self.s_a, self.c, self.c_host = {}, {}, {}, {}
        ws = 0
        for M in self.ms:
            if self.fmt in BS_FMTS:
                self.a_q[M] = torch.empty(M, K // 2 if self.fmt == 5 else K, dtype=torch.uint8, device=device)
                self.s_a[M] = torch.empty(qlin.block_scaled_sf_bytes(self.fmt, M, K), dtype=torch.uint8,
                                          device=device)
            else:
                self.a_q[M] = (torch.empty(M, K, dtype=torch.bfloat16, device=device) if self.fmt == 3 else
                               torch.empty(M, K, dtype=torch.uint8, device=device))
                self.s_a[M] = torch.empty(*((M, K // 128) if self.fmt == 2 else (M,)), dtype=torch.float32,
                                          device=device)
            self.c[M] = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            ws = max(ws, qlin.qlin_scaled_mm_workspace_size(self.fmt, M, N, K))
        self.workspace = torch.zeros(max(ws, 256), dtype=torch.uint8, device=device)
        self.calls = 0
        self.configs = {M: qlin.qlin_dispatch_query(self.fmt, M, N, K) for M in self.ms}
        # weights are final: launches may overlap the previous kernel's tail
        torch.cuda.synchronize(device)
        self.flags = qlin.QLIN_PDL

    def launch_quant(self, M, stream):
        q = self.qlin
        x = self.a_sets[self.act][M]
        if self.fmt == 3:
            return  # bf16: the GEMM reads the activations themselves
        if self.fmt in BS_FMTS:
            q.qlin_quantize_block_scaled(self.fmt, x, self.a_q[M], self.s_a[M], self.g_a, stream, flags=self.flags)
        elif self.fmt == 2:
            q.qlin_quantize_block(x, 1, self.a_q[M], self.s_a[M], stream, flags=self.flags)
        else:
            q.qlin_quantize_per_token(self.fmt, x, self.a_q[M], self.s_a[M], stream, flags=self.flags)

    def launch_gemm(self, M, stream):
        w_q, s_w = self.w_copies[self.calls % self.n_copies]
        self.calls += 1
        if self.fmt == 3:
            self.qlin.qlin_matmul_bf16(self.a_sets[self.act][M], w_q, self.bias, self.c[M], self.workspace, stream,
                                       flags=self.flags)
            return
        if self.fmt in BS_FMTS:
            self.qlin.qlin_block_scaled_mm(self.fmt, self.a_q[M], self.s_a[M], w_q, s_w, self.bias, self.c[M],
                                           self.g_a, self.g_w, self.workspace, stream, flags=self.flags)
            return
        self.qlin.qlin_scaled_mm(self.fmt, self.a_q[M], self.s_a[M], w_q, s_w, self.bias, self.c[M],
                                 self.workspace, stream, flags=self.flags)

    def layer_is_fused(self, M):
        """Whether qlin_linear runs M as one kernel: Swap-AB configurations
        whose unit of K blocks fits the resident activation operand (64 KiB)."""
        if not self.fused:
            return False
        cfg = self.configs[M]
        if cfg["variant"] not in (self.qlin.QLIN_VAR_SWAPAB, self.qlin.QLIN_VAR_SWAPAB_SPLITK):
            return False
        kblocks = self.w.K // 128
        per_unit = kblocks // cfg["k_segments"] if cfg["k_segments"] > 1 else kblocks
        return per_unit <= 65536 // (cfg["tile_n"] * 128)

    def kernels_per_step(self):
        return sum(1 if (self.fmt == 3 or self.layer_is_fused(M)) else 2 for M in self.ms)

    def launch_layer(self, M, stream):
        """Quantise + GEMM for one M: two PDL-chained kernels, or one call of
        qlin_linear with QLIN_FUSED."""
        if not self.fused:
            self.launch_quant(M, stream)
            self.launch_gemm(M, stream)
            return
        w_q, s_w = self.w_copies[self.calls % self.n_copies]
        self.calls += 1
        self.qlin.qlin_linear(self.fmt, self.a_sets[self.act][M], self.a_q[M], self.s_a[M], w_q, s_w, self.bias,
                              self.c[M], self.workspace, stream, flags=self.flags | self.qlin.QLIN_FUSED)

    def step(self, stream, act_set=None):
        """Issue one step: for each M, the quantiser then the GEMM (PDL)."""
        self.act = (self.act + 1) % self.n_act_sets if act_set is None else act_set
        for M in self.ms:
            self.launch_layer(M, stream)

    def capture_graphs(self, stream):
        """One CUDA graph per step of a rotation: graph g reads activation set
        g and the next len(ms) weight copies.  Exactly what the timed region
        replays."""
        graphs = []
        for g in range(self.n_graphs):
            cg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(cg, stream=stream):
                self.step(stream, act_set=g)
            graphs.append(cg)
        return graphs

    def step_e2e(self, stream):
        """The same step through the C ABI, with each M's activations copied in
        from pinned host memory and its C copied back.  The copies run on two
        copy streams, ordered against the kernels by events (copy-in ->
        quantise + GEMM -> copy-out), so transfers in both directions overlap
        each other and the kernels of other M.  Two activation sets alternate
        between steps.  Returns (h2d bytes, d2h bytes) of the step."""
        hb = db = 0
        if self.a_host is None:
            self.a_host = {M: self.a_cpu[M].pin_memory() for M in self.ms}
            self.c_host = {M: torch.empty(M, self.w.N, dtype=torch.bfloat16).pin_memory() for M in self.ms}
            self.s_in = torch.cuda.Stream(self.device)
            self.s_out = torch.cuda.Stream(self.device)
            self.e2e_step = 0
            self.ev_act_free = {}  # (set, M): the kernels that read that activation buffer are done
            self.ev_c_free = {}    # M: C[M] has been copied out
        slot = self.e2e_step % min(2, self.n_act_sets)
        if self.e2e_step == 0:  # the copy streams start after everything issued before
            start = torch.cuda.Event()
            start.record(stream)
            self.s_in.wait_event(start)
            self.s_out.wait_event(start)
        self.e2e_step += 1
        for M in self.ms:
            ev = self.ev_act_free.get((slot, M))
            if ev is not None:
                self.s_in.wait_event(ev)
            with torch.cuda.stream(self.s_in):
                self.a_sets[slot][M].copy_(self.a_host[M], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(self.s_in)
            hb += self.a_host[M].numel() * 2
            stream.wait_event(ev_in)
            if M in self.ev_c_free:
                stream.wait_event(self.ev_c_free[M])
            self.act = slot
            self.launch_layer(M, stream)
            ev_k = torch.cuda.Event()
            ev_k.record(stream)
            self.ev_act_free[(slot, M)] = ev_k
            self.s_out.wait_event(ev_k)
            with torch.cuda.stream(self.s_out):
                self.c_host[M].copy_(self.c[M], non_blocking=True)
            ev_out = torch.cuda.Event()
            ev_out.record(self.s_out)
            self.ev_c_free[M] = ev_out
            db += self.c[M].numel() * 2
        return hb, db

    def e2e_after(self, event):
        """Order the copy streams after `event` (the start of the timed region)."""
        self.s_in.wait_event(event)
        self.s_out.wait_event(event)

    def e2e_join(self, stream):
        """Make `stream` wait for the last copy-out issued (steps overlap: the next
        step's copy-in and kernels may start before this one's copies end)."""
        if self.ev_c_free:
            stream.wait_event(self.ev_c_free[self.ms[-1]])


class MoEPath:
    """The FP8 MoE layer (qlin_moe_forward: seven PDL-chained kernels) on the
    benchmark's MoE configuration, one token count at a time."""

    def __init__(self, device, seed=0):
        from quantized_linear_layers_group_b200 import qlin

        self.qlin = qlin
        c = synth.MOE
        self.E, self.k, self.H, self.I = c["E"], c["topk"], c["H"], c["I"]
        E, H, I = self.E, self.H, self.I
        self.w1 = torch.empty(E * 2 * I, H, dtype=torch.uint8, device=device)
        self.s1 = torch.empty(E * 2 * I, dtype=torch.float32, device=device)
        self.w2 = torch.empty(E * H, I, dtype=torch.uint8, device=device)
        self.s2 = torch.empty(E * H, dtype=torch.float32, device=device)
        for e0, e1, w in synth.moe_weight_chunks(E, 2 * I, H, seed + 30, device):
            qlin.qlin_quantize_per_token(1, w, self.w1[e0 * 2 * I:e1 * 2 * I], self.s1[e0 * 2 * I:e1 * 2 * I])
        for e0, e1, w in synth.moe_weight_chunks(E, H, I, seed + 31, device):
            qlin.qlin_quantize_per_token(1, w, self.w2[e0 * H:e1 * H], self.s2[e0 * H:e1 * H])
        torch.cuda.synchronize()
        self.device = device

    def time_t(self, T, stream, reps=8, replays=5):
        """Per-layer device time (us) of qlin_moe_forward at T tokens, from a
        CUDA graph of `reps` layers (median of `replays`), and the number of
        experts the routing activated."""
        q = self.qlin
        x, logits = synth.moe_inputs(T, self.H, self.E)
        x, logits = x.to(self.device), logits.to(self.device)
        out = torch.empty(T, self.H, dtype=torch.bfloat16, device=self.device)
        ws = torch.empty(q.qlin_moe_workspace_size(T, self.H, self.I, self.E, self.k), dtype=torch.uint8,
                         device=self.device)
        fwd = lambda: q.qlin_moe_forward(x, logits, self.k, self.w1, self.s1, self.w2, self.s2, out, ws, stream,
                                         flags=q.QLIN_PDL)
        for _ in range(3):
            fwd()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                fwd()
        g.replay()
        ts = []
        for _ in range(replays):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            g.replay()
            a1.record(stream)
            a1.synchronize()
            ts.append(a0.elapsed_time(a1) * 1e3 / reps)
        # experts the routing used (offsets live in the workspace after topk ids, weights, rows)
        R = T * self.k
        off0 = 3 * ((R * 4 + 255) // 256 * 256)
        offs = ws[off0:off0 + 4 * (self.E + 1)].view(torch.int32).cpu()
        active = int((offs[1:] - offs[:-1] > 0).sum())
        del g
        return statistics.median(ts), active

    def report(self, stream, peaks, tpk):
        tc_peak, tc_src = tensor_peak(peaks, 1, tpk)
        hbm = peaks["hbm_gbs"]
        per_t = []
        for T in synth.MOE["T"]:
            us, active = self.time_t(T, stream)
            R = T * self.k
            flops = 6.0 * R * self.H * self.I
            wbytes = active * 3 * self.H * self.I  # gate-up (2I x H) + down (H x I) of each active expert, FP8
            t_roof = max(wbytes / (hbm * 1e9), flops / (tc_peak * 1e12))
            per_t.append({"T": T, "rows": R, "active_experts": active, "layer_us": us,
                          "tflops": flops / (us * 1e-6) / 1e12, "weight_gbs": wbytes / (us * 1e-6) / 1e9,
                          "roofline_us": t_roof * 1e6, "frac_roofline": t_roof / (us * 1e-6),
                          "bound": "hbm" if wbytes / (hbm * 1e9) >= flops / (tc_peak * 1e12) else "tensor"})
        return {"E": self.E, "topk": self.k, "H": self.H, "I": self.I, "kernels_per_layer": 7,
                "peak_source": tc_src, "per_t": per_t}


def per_kernel_times(hp: HotPath, stream, reps=8, replays=5):
    """For each M: a graph of `reps` back-to-back launches of one kernel (the
    quantiser rotates activation sets, the GEMM weight copies), timed with
    events on the launching stream; per-launch time = graph time / reps,
    median of `replays` replays.  Returns ({M: quant us}, {M: gemm us})."""
    qt, gt = {}, {}
    for M in hp.ms:
        for kind in (("g",) if hp.fmt == 3 else ("q", "g")):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(reps):
                    if kind == "q":
                        hp.act = i % hp.n_act_sets
                        hp.launch_quant(M, stream)
                    else:
                        hp.launch_gemm(M, stream)
            for _ in range(2):
                g.replay()
            ts = []
            for _ in range(replays):
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                g.replay()
                a1.record(stream)
                a1.synchronize()
                ts.append(a0.elapsed_time(a1) * 1e3 / reps)
            (qt if kind == "q" else gt)[M] = statistics.median(ts)
            del g
        qt.setdefault(M, 0.0)
    torch.cuda.synchronize()
    return qt, gt


def workload_report(hp: HotPath, qt, gt, peaks, tpk):
    """Per-M table and dominant-kernel roofline of one workload."""
    from quantized_linear_layers_group_b200 import qlin

    w = hp.w
    N, K, fmt = w.N, w.K, w.fmt
    tc_peak, tc_src = tensor_peak(peaks, fmt, tpk)
    hbm = peaks["hbm_gbs"]
    per_m = []
    for M in hp.ms:
        tg, tq = gt[M] * 1e-6, qt[M] * 1e-6
        ab, extra = gemm_bytes(M, N, K, fmt)
        fl = gemm_flops(M, N, K)
        t_hbm, t_tc = ab / (hbm * 1e9), fl / (tc_peak * 1e12)
        t_roof = max(t_hbm, t_tc)
        cfg = hp.configs[M]
        per_m.append({"M": M, "N": N, "K": K, "format": FMT_NAME[fmt],
                      "variant": qlin.VARIANT_NAMES[cfg["variant"]], "tile_n": cfg["tile_n"],
                      "k_segments": cfg["k_segments"], "gemm_us": gt[M], "quant_us": qt[M],
                      "tflops": fl / tg / 1e12, "hbm_gbs": ab / tg / 1e9,
                      "hbm_gbs_all_bytes": (ab + extra) / tg / 1e9,
                      "roofline_us": t_roof * 1e6, "frac_roofline": t_roof / tg,
                      "bound": "hbm" if t_hbm >= t_tc else "tensor",
                      "quant_gbs": quant_bytes(M, K, fmt) / tq / 1e9 if tq > 0 else None,
                      "quant_frac_hbm": quant_bytes(M, K, fmt) / tq / 1e9 / hbm if tq > 0 else None})
    total = sum(gt[M] + qt[M] for M in hp.ms)
    roof = kernel_roofline(per_m, hp.configs, fmt, N, K, hbm, tc_peak, total)
    roof["traffic"] = measured_traffic_kernel(w.name, fmt, N, K, hp.configs, roof["m_values"])
    roof["peak_source"] = tc_src if roof["bound"] == "tensor" else f"{peaks['source']} hbm_gbs copy"
    return per_m, roof, tc_peak, tc_src


# ----------------------------------------------------------- distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def aggregate(per_rank_units: float, max_seconds: float, world: int) -> float:
    """Whole-job throughput: every rank processed per_rank_units; time is the max over ranks."""
    return per_rank_units * world / max_seconds


# -------------------------------------------------------------- CPU arm
_ORACLE_WEIGHTS = {}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_weight(workload: synth.Workload, seed=0):
    import oracle

    key = (workload.name, seed)
    if key not in _ORACLE_WEIGHTS:
        w = synth.weights(workload, seed)
        if workload.fmt == 2:
            _ORACLE_WEIGHTS[key] = oracle.quantize_block(w, 128, 128)
        else:
            _ORACLE_WEIGHTS[key] = oracle.quantize_per_token(workload.fmt, w)
    return _ORACLE_WEIGHTS[key]


def cpu_oracle_rows(workload: synth.Workload, rows_per_m, threads=1, seed=0):
    """The CPU oracle (as it stands) on a bounded sample: for each (M, r) in
    rows_per_m, the first r of M activation rows are quantised and their full C
    rows computed against the whole (offline-quantised) weight.  With
    threads > 1, row slices run concurrently on a thread pool (the oracle's C
    code runs without the interpreter lock).  Returns (seconds, GEMM flops)."""
    import oracle

    N, K = workload.N, workload.K
    wq, sw = _oracle_weight(workload, seed)
    b = synth.bias(workload, seed)
    inputs = [synth.activations(workload, M, seed=seed)[:r].contiguous() for M, r in rows_per_m]
    flops = sum(gemm_flops(r, N, K) for _, r in rows_per_m)

    def job(a):
        if workload.fmt == 2:
            aq, sa = oracle.quantize_block(a, 1, 128)
        else:
            aq, sa = oracle.quantize_per_token(workload.fmt, a)
        oracle.scaled_mm(workload.fmt, aq, sa, wq, sw, b)

    # split every sample into slices of a few rows so all threads stay busy
    slices = []
    for a in inputs:
        step = max(1, math.ceil(a.shape[0] / max(1, threads)))
        slices += [a[i:i + step].contiguous() for i in range(0, a.shape[0], step)]
    t0 = time.perf_counter()
    if threads <= 1:
        for s in slices:
            job(s)
    else:
        with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(job, slices))
    return time.perf_counter() - t0, flops


def reference_rows(workload: synth.Workload, cap: int):
    """The reference arm's per-step sample: every M of the sweep, at most `cap` rows of it."""
    return [(M, min(M, cap)) for M in workload.m_values]


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    rows = reference_rows(w, args.ref_rows)
    cores = host_cores()
    for _ in range(args.warmup):
        cpu_oracle_rows(w, rows, threads=cores)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, flops = cpu_oracle_rows(w, rows, threads=cores)
        times.append(dt)
    total = sum(times)
    value = flops * len(times) / total / 1e12
    desc = (f"{w.name}: every M of the sweep, its first min(M, {args.ref_rows}) rows quantised and their full "
            f"C rows computed (N={w.N}, K={w.K}), {cores} threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DTYPE[w.fmt],
            "data": "synthetic", "config": {"workload": w.name, "format": FMT_NAME[w.fmt], "N": w.N, "K": w.K,
                                            "m_values": list(w.m_values), "bias": w.bias,
                                            "parallelism": "single process"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main
def time_steps(hp: HotPath, stream, steps, warmup, world, local, use_graph=True):
    """The device-timed region: `steps` graph replays of whole steps (each
    graph reads its own activation set and rotates the weights), events on
    the launching stream around each replay, barrier + synchronise on both
    sides, clocks sampled meanwhile.  Returns (seconds, clocks)."""
    graphs = hp.capture_graphs(stream) if use_graph else []
    torch.cuda.synchronize()
    for i in range(warmup):
        if use_graph:
            graphs[i % len(graphs)].replay()
        else:
            hp.step(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        evs[i][0].record(stream)
        if use_graph:
            graphs[i % len(graphs)].replay()
        else:
            hp.step(stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    barrier(world)
    clk = clocks.stop()
    del graphs
    return max_over_ranks(sum(step_ms) / 1e3, world), clk


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--m", type=str, default=None, help="comma-separated M values (default: the workload's sweep)")
    ap.add_argument("--table", default=os.path.join(ROOT, "quantized_linear_layers_group_b200", "tables",
                                                    "b200.qlt"))
    ap.add_argument("--no-table", action="store_true")
    ap.add_argument("--fused", action="store_true",
                    help="quantise inside the GEMM where the configuration is Swap-AB (qlin_linear, QLIN_FUSED)")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="replay each device-timed step as a CUDA graph (default)")
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="measure the headline workload only")
    ap.add_argument("--no-peaks", action="store_true", help="skip the 8-bit library peak measurement")
    ap.add_argument("--ref-rows", type=int, default=64, help="rows per M in a reference-arm step")
    ap.add_argument("--baseline-rows", type=int, default=1024, help="rows per M of the all-core cpu_baseline sample")
    args = ap.parse_args(argv)
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"

    rank, world, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, rank, world)
        barrier(world)
        return

    from quantized_linear_layers_group_b200 import qlin

    if not args.no_table and os.path.exists(args.table):
        qlin.qlin_dispatch_table_load(args.table)
    workload = synth.WORKLOADS[args.workload]
    ms = [int(x) for x in args.m.split(",")] if args.m else list(workload.m_values)
    device = torch.device("cuda", local)
    stream = torch.cuda.Stream(device)
    peaks = load_peaks()

    with torch.cuda.stream(stream):
        hp = HotPath(workload, ms, device, fused=args.fused)
        for _ in range(args.warmup):
            hp.step(stream)
        torch.cuda.synchronize()
        st = qlin.qlin_sync_status(stream)
        if st != 0:
            raise RuntimeError(f"device status after warm-up: {qlin.qlin_status_string(st)}")

        # ---------------------------------------------- device-timed steps
        elapsed_s, clk = time_steps(hp, stream, args.steps, args.warmup, world, local, args.graph)

        # ------------------------------------------------- end-to-end steps
        for _ in range(2):
            hp.step_e2e(stream)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        hp.e2e_after(e0)
        hb = db = 0
        for _ in range(args.steps):
            hb, db = hp.step_e2e(stream)
        hp.e2e_join(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)

        # ------------------------------------------- per-kernel launch times
        tpk = None if args.no_peaks else measure_tensor_peaks(device)
        qt, gt = per_kernel_times(hp, stream)
        per_m, roof, tc_peak, tc_src = workload_report(hp, qt, gt, peaks, tpk)
        kernels_per_step = hp.kernels_per_step()
        st = qlin.qlin_sync_status(stream)
        if st != 0:
            raise RuntimeError(f"device status: {qlin.qlin_status_string(st)}")
        del hp
        torch.cuda.empty_cache()

        # ------------------------------ every workload of the metric, per M
        workloads = {}
        if not args.no_workloads and world == 1:
            for name in ALL_WORKLOADS + BF16_WORKLOADS + BS_WORKLOADS:
                w = synth.WORKLOADS[name]
                wh = HotPath(w, list(w.m_values), device)
                for _ in range(3):
                    wh.step(stream)
                w_s, _ = time_steps(wh, stream, 5, 3, 1, local, args.graph)
                wq, wg = per_kernel_times(wh, stream)
                w_per_m, w_roof, _, _ = workload_report(wh, wq, wg, peaks, tpk)
                fl = sum(gemm_flops(M, w.N, w.K) for M in w.m_values)
                workloads[name] = {"format": FMT_NAME[w.fmt], "N": w.N, "K": w.K, "m_values": list(w.m_values),
                                   "step_us": w_s / 5 * 1e6, "step_tflops": fl * 5 / w_s / 1e12,
                                   "roofline": w_roof, "per_m": w_per_m}
                st = qlin.qlin_sync_status(stream)
                if st != 0:
                    raise RuntimeError(f"device status ({name}): {qlin.qlin_status_string(st)}")
                del wh
                torch.cuda.empty_cache()
            mp = MoEPath(device)
            workloads["moe_fp8"] = mp.report(stream, peaks, tpk)
            del mp
            torch.cuda.empty_cache()

    N, K, fmt = workload.N, workload.K, workload.fmt
    flops_step = sum(gemm_flops(M, N, K) for M in ms)
    value = aggregate(flops_step * args.steps, elapsed_s, world) / 1e12
    e2e_value = aggregate(flops_step * args.steps, e2e_s, world) / 1e12
    # for context: the single longest launch of the step
    big = max(per_m, key=lambda r: r["gemm_us"])
    largest = {"kernel": f"qlin_gemm_kernel M={big['M']} N={N} K={K} {FMT_NAME[fmt]}", "M": big["M"],
               "us": big["gemm_us"], "bound": big["bound"]}
    if big["bound"] == "hbm":
        largest.update({"achieved": big["hbm_gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": big["hbm_gbs"] / peaks["hbm_gbs"]})
    else:
        largest.update({"achieved": big["tflops"], "peak": tc_peak, "unit": "TFLOP/s",
                        "frac": big["tflops"] / tc_peak})

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * elapsed_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE[fmt], "data": "synthetic",
            "config": {"workload": workload.name, "format": FMT_NAME[fmt], "N": N, "K": K, "m_values": ms,
                       "bias": workload.bias,
                       "l2": ("inputs larger than L2: weights rotate per GEMM and activations per step, "
                              "> 2x L2 between two uses of one copy"),
                       "parallelism": "replicas" if world > 1 else "single GPU", "cuda_graph": args.graph,
                       "fused": bool(args.fused),
                       "e2e": ("each M's activations copied in from pinned host memory and C copied back, on "
                               "two copy streams ordered by events, overlapping the kernels; eager launches"),
                       "pdl": True,
                       "table": (not args.no_table and os.path.exists(args.table))},
            "roofline": roof,
            "roofline_largest_launch": largest,
            "tensor_peak_used": {"value": tc_peak, "source": tc_src},
            "tensor_peaks": tpk,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db},
            "gpu_launches": kernels_per_step * args.steps,
            "clocks": clk,
            "per_m": per_m}
    if workloads:
        line["workloads"] = workloads
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = reference_rows(workload, args.baseline_rows)
        cores = host_cores()
        dt1, fl1 = cpu_oracle_rows(workload, [(M, min(r, 64)) for M, r in rows], threads=1)
        dtn, fln = cpu_oracle_rows(workload, rows, threads=cores)
        line["cpu_baseline"] = {
            "value": fln / dtn / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": (f"{workload.name}: every M of the sweep, its first min(M, {args.baseline_rows}) rows "
                       f"quantised and their full C rows computed (N={N}, K={K}), {cores} threads"),
            "seconds": dtn,
            "one_thread": {"value": fl1 / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1, "seconds": dt1,
                           "sample": "the same, first min(M, 64) rows, 1 thread"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
