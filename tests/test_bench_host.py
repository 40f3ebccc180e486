"""Host-side pieces of bench.py: the multi-process harness (max over ranks,
whole-job aggregation) on two gloo ranks, and the JSON of the reference arm
(the CPU oracle) on a tiny sample."""
import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    t = bench.max_over_ranks(1.0 + rank, world)        # rank 1 is the slow one
    bench.barrier(world)
    v = bench.aggregate(100.0, t, world)               # 100 units per rank
    out.put((rank, t, v))
    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.0, 2.0]              # both ranks see the max time
    assert [r[2] for r in res] == [100.0, 100.0]          # 200 units / 2 s


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--ref-rows", "2", "--workload", "int8_smoke"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_dominant_kernel_groups_launches_like_the_launch_list():
    # launches of one compiled kernel (here the Swap-AB tile-16 kernel serving
    # M <= 64) are grouped before ranking by share of the step, as ncu's
    # launch list groups them; the roofline uses the group's mean launch
    import bench
    from quantized_linear_layers_group_b200 import qlin

    ms = [1, 4, 8, 16, 32, 64, 256, 512, 1024, 2048]
    cfg = {M: {"variant": qlin.QLIN_VAR_SWAPAB if M <= 64 else (qlin.QLIN_VAR_PAIR if M > 1024 else
                                                                 qlin.QLIN_VAR_PLAIN),
               "tile_n": 16 if M <= 64 else (128 if M <= 512 else 256), "k_segments": 1} for M in ms}
    us = {1: 7.0, 4: 7.0, 8: 7.0, 16: 7.0, 32: 7.0, 64: 8.0, 256: 9.0, 512: 10.0, 1024: 12.0, 2048: 18.0}
    per_m = [{"M": M, "gemm_us": us[M]} for M in ms]
    total = sum(us.values()) + 20.0
    r = bench.kernel_roofline(per_m, cfg, 1, 4096, 2048, 6550.4, 2751.2, total)
    assert r["kernel"] == "qlin_gemm_kernel<1, 1, 16, 0, 0, 0>"
    assert r["m_values"] == [1, 4, 8, 16, 32, 64] and r["launches_per_step"] == 6
    assert abs(r["share"] - 43.0 / total) < 1e-12
    ab = sum(M * 2048 + 4096 * 2048 for M in r["m_values"]) / 6
    assert r["bound"] == "hbm" and abs(r["achieved"] - ab / (43.0 / 6 * 1e-6) / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6550.4) < 1e-12
    # pair and plain 256 tiles are different kernels; one-CTA tiles of 128 and 256 too
    assert bench.kernel_of(1, cfg[2048]) == "qlin_gemm_kernel<1, 0, 256, 0, 0, 1>"
    assert bench.kernel_of(1, cfg[1024]) == "qlin_gemm_kernel<1, 0, 256, 0, 0, 0>"
    assert bench.kernel_of(1, {"variant": qlin.QLIN_VAR_SWAPAB_SPLITK, "tile_n": 16}) == \
        bench.kernel_of(1, cfg[16])


def test_fused_layers_and_kernel_count_follow_the_configurations():
    # With --fused, a layer is one kernel when its configuration is Swap-AB
    # and a unit's K blocks fit the resident 64 KiB activation operand
    # (K/128/S <= 65536 / (tile_n * 128)); every other layer is the quantiser
    # plus the GEMM.  gpu_launches is built from this count.
    import bench
    import synth
    from quantized_linear_layers_group_b200 import qlin

    hp = bench.HotPath.__new__(bench.HotPath)
    hp.qlin = qlin
    hp.w = synth.WORKLOADS["fp8_attn"]          # K = 2048: 16 K blocks
    hp.fmt = hp.w.fmt
    hp.ms = [1, 64, 256, 2048]
    hp.configs = {
        1: {"variant": qlin.QLIN_VAR_SWAPAB, "tile_n": 16, "k_segments": 1},          # 16 <= 32: fused
        64: {"variant": qlin.QLIN_VAR_SWAPAB, "tile_n": 64, "k_segments": 1},         # 16 > 8: two kernels
        256: {"variant": qlin.QLIN_VAR_SWAPAB_SPLITK, "tile_n": 64, "k_segments": 2},  # 8 <= 8: fused
        2048: {"variant": qlin.QLIN_VAR_PLAIN, "tile_n": 256, "k_segments": 1},       # plain: two kernels
    }
    hp.fused = True
    assert [hp.layer_is_fused(M) for M in hp.ms] == [True, False, True, False]
    assert hp.kernels_per_step() == 1 + 2 + 1 + 2
    hp.fused = False
    assert not any(hp.layer_is_fused(M) for M in hp.ms)
    assert hp.kernels_per_step() == 2 * len(hp.ms)
