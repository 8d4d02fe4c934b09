#!/usr/bin/env python
"""Throughput of the bidirectional Mamba mixer layer on B200.

Default workload: one layer call at batch 8, L = 2048, d_inner = 4096,
d_state = 16, bf16 I/O with fp32 state (the 1.3B-model layer shape), on
synthetic seeded inputs.  A step is one bimamba_layer_fwd call (one kernel
launch: conv, softplus, both scan directions, D skip, sum and gate).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload layer|long] [--L L]

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs its
own replica of the workload on its own GPU -- the layer has no exchange step
across batch rows or channels -- and value is the total over ranks divided
by the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from bidirectional_mamba_denoiser_b200 import workloads as W  # noqa: E402

METRIC = "bi-Mamba layer Mtokens/s"
UNIT = "Mtokens/s"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["layer", "long"], default="layer")
    ap.add_argument("--L", type=int, default=65536, help="sequence length of --workload long")
    ap.add_argument("--lanes", type=int, default=0, help="lanes per channel (0 = library's choice)")
    ap.add_argument("--chunk", type=int, default=0, help="TMA chunk length selector: 0 auto, 1 = 16, 2 = 32")
    ap.add_argument("--family", type=int, default=0, help="kernel family: 0 auto, 1 chunked, 2 per-token fused")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    return ap.parse_args()


def workload_of(args) -> W.Workload:
    return W.LAYER_1P3B if args.workload == "layer" else W.LONG_SEQ.get(args.L) or \
        W.Workload(f"long_b1_L{args.L}_D4096_bf16", 1, args.L, 4096, 16, "bf16", 2)


def algorithmic_bytes(w: W.Workload) -> int:
    """Bytes the layer must move once: x, z, dt_f, dt_b read and out written
    per (token, channel); B_f, C_f, B_b, C_b read per token."""
    e = 2 if w.dtype == "bf16" else 4
    return w.batch * w.L * (w.d_inner * 5 * e + 4 * w.d_state * e)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------- distributed

def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], device="cuda", dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.idx)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.2)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r[2] > 150.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in loaded),
                "power_w_max": max(r[2] for r in loaded), "samples": len(loaded), "reasons": reasons}


# ---------------------------------------------------------------- cpu baseline (the oracle)

def oracle_sample_rate(w: W.Workload, inputs, params, budget_s: float):
    """The fp64 oracle, timed on a channel sample of the same inputs;
    returns (Mtokens/s scaled to the whole layer, channels, seconds, threads)."""
    import oracle
    from tests import parity_util as U
    threads = oracle.max_threads()
    nch = max(threads, 8)
    for _ in range(3):
        chans = U.sample_channels(w.d_inner, min(nch, w.d_inner), seed=99)
        si, sp = U.channel_subset(inputs, params, chans)
        t0 = time.perf_counter()
        oracle.layer_fwd(si, sp)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * budget_s or len(chans) >= w.d_inner:
            break
        nch = int(min(w.d_inner, max(nch + 1, nch * budget_s / max(dt, 1e-3))))
        nch = max(threads, (nch // threads) * threads)
    layer_s = dt * w.d_inner / len(chans)
    return w.tokens / layer_s / 1e6, len(chans), dt, threads


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, local):
    from bidirectional_mamba_denoiser_b200 import bimamba as bm
    w = workload_of(args)
    dev = torch.device("cuda", local)
    flags = (((args.lanes << bm.BIMAMBA_LANES_SHIFT) if args.lanes else 0) | (args.chunk << bm.BIMAMBA_CHUNK_SHIFT)
             | (args.family << bm.BIMAMBA_FAMILY_SHIFT))
    sets = [W.make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed + 1000 * i + rank, device=dev)
            for i in range(2)]
    out = torch.empty(w.batch, w.L, w.d_inner, device=dev, dtype=W.torch_dtype(w.dtype))
    ws = torch.empty(bm.bimamba_workspace_bytes(w.batch, w.L, w.d_inner, w.d_state), device=dev,
                     dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        inp, par = sets[i & 1]
        bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par, out=out, flags=flags,
                             workspace=ws, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(local)
    sampler.start()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)
    ms_per_step = ms_max / args.steps
    value = world * w.tokens * args.steps / (ms_max / 1e3) / 1e6

    # roofline of the (only) kernel: algorithmic bytes per launch / launch time
    peak, peak_src = load_peaks()
    achieved = algorithmic_bytes(w) / (ms / args.steps / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": None, "peak_source": peak_src,
            "kernel": "layer_kernel", "algorithmic_bytes_per_launch": algorithmic_bytes(w)}

    # end to end: host (pinned) inputs -> device, the C-ABI call, result -> host
    e2e = None
    if not args.no_e2e:
        inp, par = sets[0]
        host = {k: v.to("cpu").pin_memory() for k, v in inp.items()}
        dbuf = {k: torch.empty_like(v) for k, v in inp.items()}
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = hout.numel() * hout.element_size()
        k2 = max(3, min(args.steps, 20))

        def e2e_step():
            for k in host:
                dbuf[k].copy_(host[k], non_blocking=True)
            bm.bimamba_layer_fwd(dbuf["x"], dbuf["z"], dbuf["dt"], dbuf["B"], dbuf["C"], par, out=out,
                                 flags=flags, workspace=ws, stream=stream)
            hout.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        barrier(world)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(k2):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        ms2 = max_over_ranks(a0.elapsed_time(a1), world)
        e2e = {"value": round(world * w.tokens * k2 / (ms2 / 1e3) / 1e6, 4), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k2}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp, par = sets[0]
        v, nch, secs, thr = oracle_sample_rate(w, inp, par, args.cpu_budget)
        cpu = {"value": round(v, 6), "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": f"{nch} of {w.d_inner} channels x {w.batch} batch rows x L={w.L} "
                         f"({secs:.1f} s), scaled by {w.d_inner}/{nch}"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seq_len": w.L, "d_inner": w.d_inner,
                       "d_state": w.d_state, "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (two rotating input sets)"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps, "clocks": clocks,
            "hbm_gbs_algorithmic": round(achieved, 1),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------- reference arm (the oracle)

def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    from tests import parity_util as U
    w = workload_of(args)
    inp, par = W.make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed,
                           device="cuda" if torch.cuda.is_available() else "cpu")
    threads = oracle.max_threads()
    per_step = min(30.0, 150.0 / max(1, args.steps + args.warmup))
    # size one step's channel sample to about per_step seconds
    nch = max(1, threads)
    chans = U.sample_channels(w.d_inner, nch, seed=7)
    si, sp = U.channel_subset(inp, par, chans)
    t0 = time.perf_counter()
    oracle.layer_fwd(si, sp)
    t1 = time.perf_counter() - t0
    nch = int(max(1, min(w.d_inner, nch * per_step / max(t1, 1e-3))))
    chans = U.sample_channels(w.d_inner, nch, seed=7)
    si, sp = U.channel_subset(inp, par, chans)
    for _ in range(args.warmup):
        oracle.layer_fwd(si, sp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.layer_fwd(si, sp)
    secs = time.perf_counter() - t0
    layer_s = secs / args.steps * w.d_inner / len(chans)
    value = w.tokens / layer_s / 1e6
    sample = f"{len(chans)} of {w.d_inner} channels x {w.batch} batch rows x L={w.L} per step, scaled by " \
             f"{w.d_inner}/{len(chans)}"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(layer_s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.L, "d_inner": w.d_inner,
                   "d_state": w.d_state, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank, world, local = dist_init(args)
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
