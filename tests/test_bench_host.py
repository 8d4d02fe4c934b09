"""Host-side logic of bench.py, on CPU: the rank helpers over a real
world-size-2 gloo group, the work and byte counts, and the reference arm's
rank rule."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from bidirectional_mamba_denoiser_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slowest = bench.max_over_ranks(10.0 + rank, world, device="cpu")
        rate = bench.whole_job_rate(1000.0, world, slowest)
        bench.barrier(world)
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, slowest, rate in got:
        assert slowest == 11.0  # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 1000.0 / 11.0 * 1e-6)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(2e6, 1, 0.5) == pytest.approx(4.0)


def test_layer_and_block_bytes():
    # x, z, dt_f, dt_b, out: 5 x 2 B per element; B/C of both directions: 4 x 16 x 2 B per token
    assert bench.layer_bytes(8, 2048, 4096, 16, 2) == 8 * 2048 * (4096 * 10 + 128)
    w = W.BLOCK_CACHED
    state = 16 * 4096 * 16 * 4 + 16 * 3 * 4096 * 2
    assert bench.block_bytes(w) == bench.layer_bytes(16, 32, 4096, 16, 2) + state + state // 128


def test_workload_mapping():
    a = bench.parse_args([])
    # the default is the metric's own configuration: batch 1, d_inner 4096, L 65536
    assert bench.workload_of(a) is W.LONG_SEQ[65536] and a.steps >= 3 and a.warmup >= 3
    assert bench.workload_of(bench.parse_args(["--workload", "layer"])) is W.LAYER_1P3B
    assert bench.workload_of(bench.parse_args(["--workload", "long", "--L", "4096"])).L == 4096
    assert bench.workload_of(bench.parse_args(["--workload", "block"])) is W.BLOCK_CACHED
    sw = bench.workload_of(bench.parse_args(["--workload", "sweep", "--L", "32768"]))
    assert sw.extra["layers"] == 48 and sw.extra["steps"] == 128


def test_reference_arm_runs_on_rank0_only():
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args, rank=1, world=2) is None


def test_roofline_fields():
    ops = 42 * 8 * 2048 * 4096  # the default workload's MUFU operations per launch
    r = bench.roofline(ops, 1.0, {"sm_mhz": 1965.0}, "x", "y")
    assert r["bound"] == "alu" and r["traffic"] is None
    assert r["peak"] == pytest.approx(148 * 16 * 1965e6 / 1e9, rel=1e-4)
    assert r["achieved"] == pytest.approx(ops / 1e-3 / 1e9, rel=1e-4)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=1e-4)
    assert bench.roofline(ops, 1.0, None, "long_b1_L65536_D4096_bf16", "layer_tma_kernel")["traffic"] > 0


def test_every_workload_resolves_and_names_its_sizes():
    for wl in ("layer", "long", "block", "sweep", "decode", "decode_mamba2", "mamba2", "mamba2_long", "sharded",
               "proj"):
        w = bench.workload_of(bench.parse_args(["--workload", wl]))
        assert w.batch >= 1 and w.L >= 1 and w.d_inner >= 1
        assert f"b{w.batch}" in w.name or "b8" in w.name or "b16" in w.name
    assert bench.workload_of(bench.parse_args(["--workload", "sharded"])).L == 262144
    assert bench.workload_of(bench.parse_args(["--workload", "proj"])).extra["d_model"] == 2048


def test_tensor_roofline_and_flop_counts():
    # dual form: 4 products per chunk, head and direction
    Q, N, P = 128, 128, 32
    per_chunk = 2.0 * (Q * Q * N + Q * P * N + N * P * Q + Q * P * Q)
    assert bench.mamba2_ssd_flops(8, 2048, 120, P, N) == per_chunk * 16 * 120 * 8 * 2
    r = bench.roofline_tensor(1.0e12, 1.0, "w", "k")  # 1 TFLOP in 1 ms = 1000 TFLOP/s
    assert r["achieved"] == 1000.0 and abs(r["frac"] - 1000.0 / r["peak"]) < 1e-4 and r["bound"] == "tensor"


def test_sweep_pool_exceeds_twice_l2():
    for L in (2048, 8192, 32768, 131072):
        per_set = bench.layer_input_bytes(1, L, 4096, 16, 2)
        r = bench.pool_size(per_set)
        assert r >= 2 and r * per_set > 2 * bench.L2_BYTES
    assert bench.pool_size(bench.layer_input_bytes(1, 2048, 4096, 16, 2)) == 5


def test_hbm_roofline_fields():
    r = bench.roofline_hbm(1.0e9, 1.0, "w", "k")  # 1 GB in 1 ms = 1000 GB/s
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["achieved"] == 1000.0
    assert abs(r["frac"] - 1000.0 / r["peak"]) < 1e-4
    # the Mamba-2 call at batch 8, L 2048: 528 MB of algorithmic traffic
    assert bench.mamba2_bytes(8, 2048, 120, 32, 128) == 8 * 2048 * (2 * 4096 + 3840 + 240 + 3840) * 2


def test_cpu_model_is_named():
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()
