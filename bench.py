#!/usr/bin/env python
"""Throughput of the bidirectional Mamba mixer layer on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload layer|long|block|sweep] [--L L]

Workloads (synthetic seeded inputs, bf16 I/O, fp32 state, d_state 16):
  long   (default) one layer call at batch 1, d_inner 4096, L = --L (default
         65536): the layer throughput against sequence length; a step is one
         bimamba_layer_fwd (one kernel launch: conv, softplus, both scan
         directions, D skip, sum and gate).  The line also carries the same
         measurement at L = 4096, 16384, 65536 and 131072 ("l_sweep")
  layer  the same at batch 8, L 2048 -- the 1.3B layer shape
  block  block-cached decoding at batch 16, d_inner 4096: the forward state of
         a 65536-token prefix is built once, then a step is one
         bimamba_block_step over a 32-token block (commit every 128th step);
         steps are replayed from a CUDA graph
  sweep  a denoiser-shaped stack: one step is 48 layer calls at batch 1,
         L = --L (default 8192), each layer with its own inputs; the line adds
         the mixer time of a full 128-step generation

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs its own
replica on its own GPU -- the layer has no exchange step across batch rows or
channels -- and value is the total over ranks divided by the slowest rank's
device time (scaling "weak").
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

from bidirectional_mamba_denoiser_b200 import workloads as W  # noqa: E402

METRIC = "bi-Mamba layer Mtokens/s"
UNIT = "Mtokens/s"

SMS = 148
MUFU_PER_SM_CLK = 16          # special-function-unit lanes per SM per clock (B200)
MUFU_PER_ELEM_LAYER = 42      # 32 state exps + 2x(SiLU 2 + softplus 2) + gate SiLU 2
MUFU_PER_ELEM_FWD = 20        # one direction: 16 state exps + SiLU 2 + softplus 2

# DRAM bytes (read + write) per launch from the ncu capture summarised in
# profiles/ -- the workload and kernel they were taken on; anything else null.
# The chunked kernel's figure was taken at L 16384 and scaled by the token
# count (its traffic is linear in L); the block step's at a 4096-token prefix
# (a step reads the same bytes whatever the prefix length).
NCU_TRAFFIC = {

    ("layer_1p3b_b8_L2048_D4096_bf16", "fused_layer_kernel"): 1307.9e6,
    ("mamba2_1p3b_b8_L2048_H120x32_N128_bf16", "m2_prep + m2_ssd dual-form kernel (both directions)"): 1026.2e6,
    ("long_b1_L16384_D4096_bf16", "layer_tma_kernel"): 1457.4e6,
    ("long_b1_L65536_D4096_bf16", "layer_tma_kernel"): 4 * 1457.4e6,
    ("block_cached_b16_P65536_G32_D4096_bf16", "async_block_kernel"): 22.2e6,
    ("block_cached_b16_P4096_G32_D4096_bf16", "async_block_kernel"): 22.2e6,
    ("proj_1p3b_b8_L2048_dmodel2048_D4096_bf16", "gemm_bf16_persistent_kernel (input projection)"): 733.4e6,
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["layer", "long", "block", "sweep", "decode", "decode_mamba2", "mamba2",
                                           "mamba2_long", "sharded", "proj"], default="long")
    ap.add_argument("--L", type=int, default=0, help="sequence length of --workload long/sweep; prefix length of --workload block/decode/decode_mamba2")
    ap.add_argument("--lanes", type=int, default=0, help="lanes per channel / group size (0 = library's choice)")
    ap.add_argument("--chunk", type=int, default=0, help="chunk length selector: 0 auto, 1 = 16, 2 = 32")
    ap.add_argument("--family", type=int, default=0,
                    help="kernel family: 0 auto, 1 chunked, 2 per-token fused, 3 chunked parallel scan")
    ap.add_argument("--flags", type=lambda v: int(v, 0), default=0, help="further flag bits (tuning knobs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-l-sweep", action="store_true", help="long: skip the per-L lines")
    ap.add_argument("--segments", type=int, default=0,
                    help="long: scan the sequence as this many segments side by side, with carries (two passes)")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    return ap.parse_args(argv)


def workload_of(args) -> W.Workload:
    if args.workload == "layer":
        return W.LAYER_1P3B
    if args.workload in ("decode", "decode_mamba2"):
        w = W.BLOCK_DECODE if args.workload == "decode" else W.BLOCK_DECODE_M2
        if args.L:  # a shorter prompt (same block steps)
            return W.Workload(w.name.replace(f"_P{w.extra['prefix']}_", f"_P{args.L}_"), w.batch, w.L, w.d_inner,
                              w.d_state, w.dtype, w.seed, extra={**w.extra, "prefix": args.L})
        return w
    if args.workload == "mamba2":
        return W.MAMBA2_1P3B
    if args.workload == "sharded":
        return W.SHARDED_SEQ
    if args.workload == "proj":
        return W.PROJ_1P3B
    if args.workload == "mamba2_long":
        L = args.L or 16384
        return W.MAMBA2_LONG.get(L) or W.Workload(f"mamba2_b1_L{L}_H120x32_N128_bf16", 1, L, 3840, 128, "bf16",
                                                  6, extra={"nheads": 120, "headdim": 32})
    if args.workload == "block":
        if args.L:  # a shorter cached prefix (same block steps)
            w = W.BLOCK_CACHED
            return W.Workload(f"block_cached_b{w.batch}_P{args.L}_G{w.L}_D{w.d_inner}_{w.dtype}", w.batch, w.L,
                              w.d_inner, w.d_state, w.dtype, w.seed, extra={**w.extra, "prefix": args.L})
        return W.BLOCK_CACHED
    if args.workload == "sweep":
        L = args.L or 8192
        return W.DENOISER_SWEEP.get(L) or W.Workload(f"denoiser_48x128_b1_L{L}_D4096_bf16", 1, L, 4096, 16,
                                                     "bf16", 3, extra={"layers": 48, "steps": 128})
    L = args.L or 65536
    return W.LONG_SEQ.get(L) or W.Workload(f"long_b1_L{L}_D4096_bf16", 1, L, 4096, 16, "bf16", 2)


def layer_bytes(batch: int, L: int, D: int, N: int, esz: int) -> int:
    """Bytes one layer call must move: x, z, dt_f, dt_b read and out written
    per (token, channel); B_f, C_f, B_b, C_b read per token."""
    return batch * L * (D * 5 * esz + 4 * N * esz)


def block_bytes(w: W.Workload, esz: int = 2) -> int:
    """One block step: the block's inputs and output, the cached state (fp32)
    and conv tail read; the commit's writes are amortised over the steps of a
    block."""
    b, G, D, N = w.batch, w.extra["block"], w.d_inner, w.d_state
    state = b * D * N * 4 + b * 3 * D * esz
    return layer_bytes(b, G, D, N, esz) + state + state // w.extra["steps_per_block"]


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


L2_BYTES = 126 * 1024 * 1024


def pool_size(input_bytes_per_set: int) -> int:
    """Distinct input sets a step cycles through so that the sets' total
    exceeds twice the L2 (each call's inputs then come from HBM)."""
    return max(2, -(-2 * L2_BYTES // max(1, input_bytes_per_set)) + 1)


# ---------------------------------------------------------------- ranks

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


def max_over_ranks(v: float, world: int, device="cuda") -> float:
    """The largest of every rank's v (timing is the slowest rank's)."""
    if world == 1:
        return v
    t = torch.tensor([v], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float, scale: float = 1e-6) -> float:
    """Units all ranks processed over the slowest rank's time (weak scaling)."""
    return world * units_per_rank / seconds_max * scale


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
                parts = [q.strip() for q in line.split(",")]
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


def timed(step, steps: int, warmup: int, world: int, dev, stream):
    """Device time of `steps` calls of step(i) after `warmup` untimed ones:
    CUDA events on the launch stream, barrier + synchronize on both sides.
    Returns (ms on this rank, clocks)."""
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(warmup + i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop()
    return e0.elapsed_time(e1), clocks


def e2e_pipelined(call, host: dict, out_shape, out_dtype, steps: int, world: int, dev, stream):
    """End to end with host buffers: every step copies its inputs from pinned
    host memory to the device, runs `call(inputs, out, stream)` and copies its
    output back to pinned host memory.  Consecutive steps overlap the way a
    caller streaming many calls would run them: copies in, compute and copies
    out on three streams, two buffer sets, ordered by events.  Device time
    from the first copy in to the last copy out, max over ranks (ms)."""
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dbuf = [{k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in host.items()} for _ in range(2)]
    obuf = [torch.empty(out_shape, dtype=out_dtype, device=dev) for _ in range(2)]
    hout = [torch.empty(out_shape, dtype=out_dtype).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(h2d):
                if i >= 2:
                    h2d.wait_event(ev_done[j])  # step i-2 no longer reads this input set
                for k in host:
                    dbuf[j][k].copy_(host[k], non_blocking=True)
                ev_in[j].record(h2d)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])  # step i-2's output has left this buffer
            call(dbuf[j], obuf[j], stream)
            ev_done[j].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_done[j])
                hout[j].copy_(obuf[j], non_blocking=True)
                ev_out[j].record(d2h)

    run(2)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    run(steps)
    e1.record(d2h)
    torch.cuda.synchronize(dev)
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world)


def roofline(mufu_ops: float, launch_ms: float, clocks, workload: str, kernel: str):
    """The binding roof of this path is the special-function unit (one exp
    per state update): achieved MUFU operations per second against the unit
    count x clock."""
    mhz = (clocks or {}).get("sm_mhz") or 1965.0
    peak = SMS * MUFU_PER_SM_CLK * mhz * 1e6 / 1e9
    achieved = mufu_ops / (launch_ms / 1e3) / 1e9
    return {"bound": "alu", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "Gop/s (MUFU)",
            "frac": round(achieved / peak, 4), "traffic": NCU_TRAFFIC.get((workload, kernel)),
            "peak_source": f"148 SMs x 16 MUFU lanes/clk x {mhz:.0f} MHz", "kernel": kernel}


def roofline_hbm(bytes_per_call: float, call_ms: float, workload: str, kernel: str):
    """HBM roof: algorithmic bytes per call over its time, against the
    measured copy bandwidth."""
    peak, src = load_peaks()
    achieved = bytes_per_call / (call_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": NCU_TRAFFIC.get((workload, kernel)),
            "peak_source": f"{src} HBM copy bandwidth", "kernel": kernel}


def hbm_fraction(bytes_per_launch: float, launch_ms: float):
    peak, src = load_peaks()
    achieved = bytes_per_launch / (launch_ms / 1e3) / 1e9
    return {"achieved_gbs": round(achieved, 1), "peak_gbs": peak, "frac": round(achieved / peak, 4),
            "peak_source": src, "algorithmic_bytes_per_launch": int(bytes_per_launch)}


# ---------------------------------------------------------------- cpu baseline (the oracle)

def oracle_sample_rate(w: W.Workload, inputs, params, budget_s: float):
    """The fp64 oracle on a channel sample of the same inputs, scaled to the
    whole layer: (Mtokens/s, channels, seconds, threads)."""
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
    return w.batch * w.L / layer_s / 1e6, len(chans), dt, threads


# ---------------------------------------------------------------- our arm

def flags_of(args, bm):
    return (((args.lanes << bm.BIMAMBA_LANES_SHIFT) if args.lanes else 0) | (args.chunk << bm.BIMAMBA_CHUNK_SHIFT)
            | (args.family << bm.BIMAMBA_FAMILY_SHIFT) | args.flags)


def layer_launches(batch: int, d_inner: int, args, carry: bool = False) -> int:
    """The library's kernel launches per layer call: two (B/C widening, then
    the layer) for the per-token family at one lane per channel and for the
    chunked family at 8 lanes per channel with 32-token chunks, one otherwise."""
    fam = args.family or (2 if 2 * batch * d_inner >= SMS * 8 * 32 else 1)
    if fam == 2:
        return 2 if (carry or args.lanes in (0, 1)) else 1
    if fam != 1 or (args.flags & 0x2000):  # BIMAMBA_CHUNKED_WIDE
        return 1
    lanes = args.lanes or (4 if 2 * batch * d_inner * 4 >= SMS * 1024 else 8)
    chunk = 32 if lanes >= 8 else 16
    if args.chunk and not carry:
        chunk = 16 if args.chunk == 1 else 32
    return 2 if (lanes == 8 and chunk == 32) else 1


def kernel_name(w: W.Workload, args) -> str:
    if args.workload in ("block", "decode"):
        return "async_block_kernel"
    fam = args.family or (2 if 2 * w.batch * w.d_inner >= SMS * 8 * 32 else 1)
    return {2: "fused_layer_kernel", 3: "layer_pscan_kernel"}.get(fam, "layer_tma_kernel")


def layer_input_bytes(batch: int, L: int, D: int, N: int, esz: int) -> int:
    """Bytes of one layer call's inputs: x, z, dt_f, dt_b and B_f, C_f, B_b, C_b."""
    return batch * L * (D * 4 * esz + 4 * N * esz)


def l_sweep(args, bm, rank, world, dev, stream, flags, lengths=(4096, 16384, 65536, 131072)):
    """The layer at batch 1, d_inner 4096 over sequence lengths: per L, two
    rotating input sets (each far larger than L2), CUDA-event time per call,
    Mtokens/s, algorithmic HBM fraction and MUFU fraction."""
    rows = []
    for L in lengths:
        w = W.LONG_SEQ.get(L) or W.Workload(f"long_b1_L{L}_D4096_bf16", 1, L, 4096, 16, "bf16", 2)
        sets = [W.make_case(w.batch, L, w.d_inner, w.d_state, w.dtype, w.seed + 1000 * i + rank, device=dev)
                for i in range(2)]
        out = torch.empty(w.batch, L, w.d_inner, device=dev, dtype=W.torch_dtype(w.dtype))
        ws = torch.empty(bm.bimamba_workspace_bytes(w.batch, L, w.d_inner, w.d_state), device=dev,
                         dtype=torch.uint8)

        def step(i):
            inp, par = sets[i % 2]
            bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par, out=out, flags=flags,
                                 workspace=ws, stream=stream)

        steps = max(5, min(args.steps, 50 * 65536 // L))
        ms, clocks = timed(step, steps, max(3, args.warmup), world, dev, stream)
        call_ms = max_over_ranks(ms, world) / steps
        elems = w.batch * L * w.d_inner
        rows.append({"L": L, "ms_per_call": round(call_ms, 4),
                     "Mtokens_s": round(whole_job_rate(w.batch * L, world, call_ms / 1e3), 4),
                     "hbm_frac": hbm_fraction(layer_bytes(w.batch, L, w.d_inner, w.d_state, 2), call_ms)["frac"],
                     "mufu_frac": roofline(MUFU_PER_ELEM_LAYER * elems, call_ms, clocks, w.name,
                                           kernel_name(w, args))["frac"],
                     "steps": steps, "sm_mhz": (clocks or {}).get("sm_mhz")})
        del sets, out, ws
        torch.cuda.empty_cache()
    return rows


def run_chunked(args, w, bm, rank, world, dev, stream):
    """long --segments k: the batch-1 layer scanned as k segments side by side
    (sharded.ChunkedLayer: a pass from zero, the carry composition, a second
    pass), for comparison with the single-pass kernels.  The segment views
    and their conv halos are set up before the timed region."""
    from bidirectional_mamba_denoiser_b200 import sharded as SH
    ops = SH.CudaOps(flags_of(args, bm))
    plans = []
    for i in range(2):
        inp, par = W.make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed + 1000 * i + rank, device=dev)
        plans.append(SH.ChunkedLayer(inp, par, args.segments, ops))
        del inp
    torch.cuda.empty_cache()

    def step(i):
        plans[i % 2].run()

    ms, clocks = timed(step, args.steps, args.warmup, world, dev, stream)
    ms_max = max_over_ranks(ms, world)
    call_ms = ms / args.steps
    elems = w.batch * w.L * w.d_inner
    return {
        "value": whole_job_rate(w.batch * w.L * args.steps, world, ms_max / 1e3),
        "ms_per_step": ms_max / args.steps,
        "gpu_launches": args.steps * (2 * layer_launches(args.segments, w.d_inner, args, carry=True) + args.segments),
        "roofline": roofline(MUFU_PER_ELEM_LAYER * elems, call_ms, clocks, w.name, "fused_layer_kernel x 2 passes"),
        "hbm": hbm_fraction(layer_bytes(w.batch, w.L, w.d_inner, w.d_state, 2), call_ms),
        "clocks": clocks,
        "schedule": f"{args.segments} segments of {w.L // args.segments} tokens as batch rows: pass from zero, "
                    f"carry composition, pass from the carries (MUFU fraction counts one pass's work)",
    }


def run_layer_like(args, w, bm, rank, world, dev, stream):
    """layer / long / sweep: steps of bimamba_layer_fwd.  The sweep cycles its
    48 layer calls through a pool of input sets (each set with its own
    parameters) whose total exceeds twice the L2; the kernel's cost does not
    depend on the values, so this stands in for fresh inputs per layer and
    step."""
    flags = flags_of(args, bm)
    if args.workload == "sweep":
        nsets = pool_size(layer_input_bytes(w.batch, w.L, w.d_inner, w.d_state, 2))
        calls = w.extra["layers"]
    else:
        nsets, calls = 2, 1
    sets = [W.make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed + 1000 * i + rank, device=dev)
            for i in range(nsets)]
    out = torch.empty(w.batch, w.L, w.d_inner, device=dev, dtype=W.torch_dtype(w.dtype))
    ws = torch.empty(bm.bimamba_workspace_bytes(w.batch, w.L, w.d_inner, w.d_state), device=dev,
                     dtype=torch.uint8)

    def step(i):
        for c in range(calls):
            inp, par = sets[(i * calls + c) % nsets]
            bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par, out=out, flags=flags,
                                 workspace=ws, stream=stream)

    ms, clocks = timed(step, args.steps, args.warmup, world, dev, stream)
    ms_max = max_over_ranks(ms, world)
    call_ms = ms / args.steps / calls
    elems = w.batch * w.L * w.d_inner
    res = {
        "value": whole_job_rate(w.batch * w.L * calls * args.steps, world, ms_max / 1e3),
        "ms_per_step": ms_max / args.steps,
        "gpu_launches": args.steps * calls * layer_launches(w.batch, w.d_inner, args),
        "roofline": roofline(MUFU_PER_ELEM_LAYER * elems, call_ms, clocks, w.name, kernel_name(w, args)),
        "hbm": hbm_fraction(layer_bytes(w.batch, w.L, w.d_inner, w.d_state, 2), call_ms),
        "clocks": clocks,
    }
    if args.workload == "sweep":
        res["sequence_mixer_s"] = round(call_ms * w.extra["layers"] * w.extra["steps"] / 1e3, 4)
        res["sequence_note"] = f"{w.extra['layers']} layers x {w.extra['steps']} steps x {call_ms:.4f} ms per call"
        res["input_pool"] = (f"{nsets} input sets of {layer_input_bytes(w.batch, w.L, w.d_inner, w.d_state, 2)} "
                             f"bytes, cycled by the 48 layer calls (total > 2 x L2)")

    if not args.no_e2e:
        inp, par = sets[0]
        host = {k: v.to("cpu").pin_memory() for k, v in inp.items()}
        k2 = max(3, min(args.steps, 20))

        def call(d, o, st):
            bm.bimamba_layer_fwd(d["x"], d["z"], d["dt"], d["B"], d["C"], par, out=o, flags=flags, workspace=ws,
                                 stream=st)

        ms2 = e2e_pipelined(call, host, out.shape, out.dtype, k2, world, dev, stream)
        res["e2e"] = {"value": round(whole_job_rate(w.batch * w.L * k2, world, ms2 / 1e3), 4),
                      "unit": UNIT, "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host.values()),
                      "d2h_bytes_per_step": out.numel() * out.element_size(), "steps": k2,
                      "schedule": "copy in, compute, copy out of consecutive steps overlapped on three streams"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp, par = sets[0]
        v, nch, secs, thr = oracle_sample_rate(w, inp, par, args.cpu_budget)
        res["cpu_baseline"] = {"value": round(v, 6), "unit": UNIT, "cores": thr, "cpu_model": cpu_model(),
                               "kind": "oracle",
                               "sample": f"{nch} of {w.d_inner} channels x {w.batch} batch rows x L={w.L} "
                                         f"({secs:.1f} s), scaled by {w.d_inner}/{nch}"}
    if args.workload == "long" and not args.no_l_sweep:
        del sets
        torch.cuda.empty_cache()
        res["l_sweep"] = l_sweep(args, bm, rank, world, dev, stream, flags)
    return res


def run_block(args, w, bm, rank, world, dev, stream):
    """block: a prefix state, then block steps replayed from a CUDA graph."""
    P, G, spb = w.extra["prefix"], w.extra["block"], w.extra["steps_per_block"]
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + rank)
    par = W.make_params(w.d_inner, w.d_state, g, dev)
    pre = W.make_inputs(w.batch, P, w.d_inner, w.d_state, w.dtype, g, dev)
    h = torch.empty(w.batch, w.d_inner, w.d_state, device=dev, dtype=torch.float32)
    tail = torch.empty(w.batch, 3, w.d_inner, device=dev, dtype=W.torch_dtype(w.dtype))
    # one untimed call first: the first launch of a kernel also loads its module
    bm.bimamba_prefix_state(pre["x"], pre["dt"], pre["B"], par, h_out=h, conv_x_out=tail, stream=stream)
    torch.cuda.synchronize(dev)
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    bm.bimamba_prefix_state(pre["x"], pre["dt"], pre["B"], par, h_out=h, conv_x_out=tail, stream=stream)
    p1.record(stream)
    torch.cuda.synchronize(dev)
    prefix_ms = p0.elapsed_time(p1)
    del pre
    torch.cuda.empty_cache()
    pool = [W.make_inputs(w.batch, G, w.d_inner, w.d_state, w.dtype, g, dev) for _ in range(8)]
    out = torch.empty(w.batch, G, w.d_inner, device=dev, dtype=W.torch_dtype(w.dtype))

    def one(i):
        blk = pool[i % len(pool)]
        commit = (i % spb) == spb - 1
        bm.bimamba_block_step((h, tail), blk["x"], blk["z"], blk["dt"], blk["B"], blk["C"], par, out=out,
                              new_state=(h, tail) if commit else None, stream=stream)

    # one block's steps captured once (the decoding loop's shape) and replayed
    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(spb):
            one(i)
    reps = max(1, args.steps // spb)

    def step(_):
        graph.replay()

    ms, clocks = timed(step, reps, max(1, args.warmup // spb), world, dev, stream)
    ms_max = max_over_ranks(ms, world)
    nsteps = reps * spb
    step_ms = ms / nsteps
    elems = w.batch * G * w.d_inner
    del graph
    return {
        "value": whole_job_rate(w.batch * G * nsteps, world, ms_max / 1e3),
        "ms_per_step": ms_max / nsteps, "gpu_launches": nsteps,
        "roofline": roofline(MUFU_PER_ELEM_LAYER * elems, step_ms, clocks, w.name, kernel_name(w, args)),
        "hbm": hbm_fraction(block_bytes(w), step_ms), "clocks": clocks,
        "prefix_state_ms": round(prefix_ms, 3),
        "prefix_mufu_frac": roofline(MUFU_PER_ELEM_FWD * w.batch * P * w.d_inner, prefix_ms, clocks, w.name,
                                     "prefix")["frac"],
        "steps_timed": nsteps, "graph": f"{spb} block steps per CUDA graph replay",
    }


# ---------------------------------------------------------------- Mamba-2 mixer

FP32_FMA_PER_SM_CLK = 128     # FP32 lanes per SM per clock (B200), one FMA each


def mamba2_bytes(batch: int, L: int, H: int, P: int, N: int, esz: int = 2) -> int:
    """Bytes one Mamba-2 mixer call must move: xBC of both directions, z, dt of
    both directions read and out written."""
    CH = H * P + 2 * N
    return batch * L * (2 * CH + H * P + 2 * H + H * P) * esz


def roofline_fma(flops: float, call_ms: float, clocks, workload: str, kernel: str):
    """Binding roof of the Mamba-2 scan on CUDA cores: FP32 FMA throughput,
    148 SMs x 128 lanes x 2 flops x the SM clock."""
    mhz = (clocks or {}).get("sm_mhz") or 1965.0
    peak = SMS * FP32_FMA_PER_SM_CLK * 2 * mhz * 1e6 / 1e12
    achieved = flops / (call_ms / 1e3) / 1e12
    return {"bound": "alu", "achieved": round(achieved, 2), "peak": round(peak, 2), "unit": "TFLOP/s (FP32 FMA)",
            "frac": round(achieved / peak, 4), "traffic": NCU_TRAFFIC.get((workload, kernel)),
            "peak_source": f"148 SMs x {FP32_FMA_PER_SM_CLK} FP32 lanes x 2 x {mhz:.0f} MHz", "kernel": kernel}


def roofline_tensor(flops: float, call_ms: float, workload: str, kernel: str):
    """Tensor-core roof of the chunked dual form: executed MMA flops per call
    against the measured dense bf16 rate (fp16 operands run at the same rate)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured bf16 dense (burst), fp16 at the same rate"
    except Exception:
        peak, src = 1590.0, "fallback bf16 dense (burst), fp16 at the same rate"
    achieved = flops / (call_ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": NCU_TRAFFIC.get((workload, kernel)), "peak_source": src,
            "kernel": kernel}


def mamba2_ssd_flops(batch: int, L: int, H: int, P: int, N: int, Q: int = 128) -> float:
    """MMA flops of one dual-form call: per chunk of Q steps, head and
    direction G = C B^T (Q x Q x N), C S^T (Q x P x N), B^T W (N x P x Q) and
    M (delta x) (Q x P x Q), at 2 flops per multiply-add."""
    nc = (L + Q - 1) // Q
    per_chunk = 2.0 * (Q * Q * N + Q * P * N + N * P * Q + Q * P * Q)
    return per_chunk * nc * H * batch * 2


def mamba2_oracle_rate(w: W.Workload, inputs, params, budget_s: float):
    """The fp64 oracle on a sample of heads, scaled to all heads:
    (Mtokens/s, heads, seconds, threads)."""
    import oracle
    from tests import parity_util as U
    H = w.extra["nheads"]
    threads = oracle.max_threads()
    k = 1
    while True:
        heads = sorted({int(h) for h in np.linspace(0, H - 1, k)})
        si, sp, _ = U.head_subset(inputs, params, heads)
        t0 = time.perf_counter()
        oracle.mamba2_layer_fwd(si, sp)
        dt = time.perf_counter() - t0
        if dt >= 0.3 * budget_s or len(heads) >= H:
            break
        k = int(min(H, max(k + 1, k * 0.6 * budget_s / max(dt, 1e-3))))
    layer_s = dt * H / len(heads)
    return w.batch * w.L / layer_s / 1e6, len(heads), dt, threads


def run_mamba2(args, w, bm, rank, world, dev, stream):
    """mamba2 / mamba2_long: steps of bimamba2_layer_fwd (two launches each on
    the tensor-core path, three on the CUDA-core one)."""
    H, P, N = w.extra["nheads"], w.extra["headdim"], w.d_state
    flags = flags_of(args, bm)
    sets = [W.make_mamba2_case(w.batch, w.L, H, P, N, w.dtype, w.seed + 1000 * i + rank, device=dev)
            for i in range(2)]
    out = torch.empty(w.batch, w.L, H * P, device=dev, dtype=W.torch_dtype(w.dtype))
    ws = torch.empty(bm.bimamba2_workspace_bytes(w.batch, w.L, H, P, N), device=dev, dtype=torch.uint8)

    def step(i):
        inp, par = sets[i % 2]
        bm.bimamba2_layer_fwd(inp["xbc"], inp["z"], inp["dt"], par, out=out, workspace=ws, stream=stream,
                              flags=flags)

    ms, clocks = timed(step, args.steps, args.warmup, world, dev, stream)
    ms_max = max_over_ranks(ms, world)
    call_ms = ms / args.steps
    tokens = w.batch * w.L
    flops = 4.0 * P * N * H * 2 * tokens  # the recurrence: two FMAs per state per token and direction
    tensor_path = w.dtype == "bf16" and not (flags & bm.BIMAMBA_NO_TMA)
    res = {
        "value": whole_job_rate(tokens * args.steps, world, ms_max / 1e3),
        "ms_per_step": ms_max / args.steps,
        "gpu_launches": (2 if tensor_path else 3) * args.steps,
        "hbm": hbm_fraction(mamba2_bytes(w.batch, w.L, H, P, N), call_ms),
        "clocks": clocks,
        "recurrence_flops_per_token": int(flops / tokens),
    }
    if tensor_path:
        # By the method's own work the call is bound by HBM: its algorithmic
        # bytes take longer at the measured copy bandwidth than its recurrence
        # flops at the tensor peak.  The dual form's executed MMA flops (a
        # dense equivalent that also multiplies the masked zeros) are reported
        # beside it.
        res["roofline"] = roofline_hbm(mamba2_bytes(w.batch, w.L, H, P, N), call_ms, w.name,
                                       "m2_prep + m2_ssd dual-form kernel (both directions)")
        res["tensor_executed"] = roofline_tensor(mamba2_ssd_flops(w.batch, w.L, H, P, N), call_ms, w.name,
                                                 "m2_ssd dual-form kernel executed MMA")
        res["fp32_equivalent"] = roofline_fma(flops, call_ms, clocks, w.name, "recurrence-equivalent")
    else:
        res["roofline"] = roofline_fma(flops, call_ms, clocks, w.name, "m2_prep_kernel + 2 x m2_scan_kernel")
    if not args.no_e2e:
        inp, par = sets[0]
        host = {k: v.to("cpu").pin_memory() for k, v in inp.items()}
        k2 = max(3, min(args.steps, 20))

        def call(d, o, st):
            bm.bimamba2_layer_fwd(d["xbc"], d["z"], d["dt"], par, out=o, workspace=ws, stream=st, flags=flags)

        ms2 = e2e_pipelined(call, host, out.shape, out.dtype, k2, world, dev, stream)
        res["e2e"] = {"value": round(whole_job_rate(tokens * k2, world, ms2 / 1e3), 4),
                      "unit": UNIT, "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host.values()),
                      "d2h_bytes_per_step": out.numel() * out.element_size(), "steps": k2,
                      "schedule": "copy in, compute, copy out of consecutive steps overlapped on three streams"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp, par = sets[0]
        v, nh, secs, thr = mamba2_oracle_rate(w, inp, par, args.cpu_budget)
        res["cpu_baseline"] = {"value": round(v, 6), "unit": UNIT, "cores": thr, "cpu_model": cpu_model(),
                               "kind": "oracle",
                               "sample": f"{nh} of {H} heads x {w.batch} batch rows x L={w.L} ({secs:.1f} s), "
                                         f"scaled by {H}/{nh}"}
    return res


def run_decode(args, w, bm, rank, world, dev, stream):
    """decode: block-cached decoding through a stack of layers, one cached
    state per layer; each block (steps x layers block steps, commits on the
    last step) replays as one CUDA graph."""
    from bidirectional_mamba_denoiser_b200 import decode
    layers, P, G, K = w.extra["layers"], w.extra["prefix"], w.extra["block"], w.extra["steps_per_block"]
    mixer = w.extra.get("mixer", "mamba1")
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + rank)
    if mixer == "mamba1":
        params = [W.make_params(w.d_inner, w.d_state, g, dev) for _ in range(layers)]
        dec = decode.BlockDecoder(params, w.batch, w.d_inner, W.torch_dtype(w.dtype), dev)
        pre = W.make_inputs(w.batch, P, w.d_inner, w.d_state, w.dtype, g, dev)
        pws = None
    else:
        H, Pd = w.extra["nheads"], w.extra["headdim"]
        params = [W.make_mamba2_params(H, Pd, w.d_state, g, dev) for _ in range(layers)]
        dec = decode.BlockDecoder(params, w.batch, w.d_inner, W.torch_dtype(w.dtype), dev, d_state=w.d_state,
                                  mixer="mamba2", nheads=H, block_len=G)
        pre = W.make_mamba2_inputs(w.batch, P, H, Pd, w.d_state, w.dtype, g, dev)
        pws = torch.empty(bm.bimamba2_workspace_bytes(w.batch, P, H, Pd, w.d_state), device=dev, dtype=torch.uint8)
    torch.cuda.synchronize(dev)
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    dec.prefill(lambda layer: pre, P, stream=stream, workspace=pws)  # one prompt, each layer its own parameters
    p1.record(stream)
    torch.cuda.synchronize(dev)
    prefill_ms = p0.elapsed_time(p1)
    del pre, pws
    torch.cuda.empty_cache()
    if mixer == "mamba1":
        pool = [W.make_inputs(w.batch, G, w.d_inner, w.d_state, w.dtype, g, dev) for _ in range(8)]
    else:
        pool = [W.make_mamba2_inputs(w.batch, G, H, Pd, w.d_state, w.dtype, g, dev) for _ in range(8)]
    out = torch.empty(layers, w.batch, G, w.d_inner, device=dev, dtype=W.torch_dtype(w.dtype))

    def inputs(s, layer):
        return pool[(s * layers + layer) % len(pool)]

    dec.block(K, inputs, out, stream=stream)  # one eager block (module loads, first launches)
    torch.cuda.synchronize(dev)
    graph = dec.capture_block(K, inputs, out, stream)
    reps = max(1, args.steps // K)

    def step(_):
        graph.replay()

    ms, clocks = timed(step, reps, max(1, args.warmup // K), world, dev, stream)
    ms_max = max_over_ranks(ms, world)
    calls = reps * K * layers
    call_ms = ms / calls
    elems = w.batch * G * w.d_inner
    del graph
    if mixer == "mamba1":
        launches = calls
        roof = roofline(MUFU_PER_ELEM_LAYER * elems, call_ms, clocks, w.name, kernel_name(w, args))
        hbm = hbm_fraction(block_bytes(w), call_ms)
    else:
        # bf16 blocks of at most 32 steps over a multiple of 4 heads: conv features, the block's
        # Gram matrix, its closed form on the tensor cores and the combination; else the conv
        # features, both directions' step-by-step scans and the combination.  A commit adds the
        # conv tail.
        tensor = w.dtype == "bf16" and G <= 32 and H % 4 == 0
        launches = reps * ((4 if tensor else 3) * K * layers + layers)
        roof = roofline_fma(4.0 * Pd * w.d_state * H * 2 * w.batch * G, call_ms, clocks, w.name,
                            "m2_prep + m2_block_gram + m2_block_mma + m2_combine (block step; the "
                            "recurrence's FP32-equivalent work)" if tensor else
                            "m2_prep + 2 x m2_scan_kernel (block step)")
        state = w.batch * H * Pd * w.d_state * 4 + w.batch * 3 * (w.d_inner + 2 * w.d_state) * 2
        hbm = hbm_fraction(mamba2_bytes(w.batch, G, H, Pd, w.d_state) + state + state // K, call_ms)
    return {
        "value": whole_job_rate(w.batch * G * calls, world, ms_max / 1e3),
        "ms_per_step": ms_max / (reps * K), "gpu_launches": launches,
        "roofline": roof, "hbm": hbm, "clocks": clocks,
        "generated_tokens_per_s": round(w.batch * G * reps * world / (ms_max / 1e3), 1),
        "prefill_ms": round(prefill_ms, 3), "layers": layers, "steps_per_block": K,
        "graph": f"one block = {K} steps x {layers} layers = {K * layers} block steps per CUDA graph replay",
    }


def run_sharded(args, w, bm, rank, world, dev, stream):
    """One sequence of w.L tokens cut into `world` contiguous segments, one
    per rank: per step each rank runs the sequence-sharded layer on its
    segment (halo and aggregate all-gathers over NCCL, two carry passes and
    the carry composition in the CUDA library).  Strong scaling.  Rank 0
    also times, on its own GPU, one rank's share at 2, 4 and 8 segments (the
    collectives replaced by stacking), for the projection to more GPUs."""
    from bidirectional_mamba_denoiser_b200 import sharded as SH
    flags = flags_of(args, bm)
    ops = SH.CudaOps(flags)
    Ls = w.L // world
    seg, par = W.make_case(w.batch, Ls, w.d_inner, w.d_state, w.dtype, w.seed + rank, device=dev)

    def step(i):
        if world > 1:
            SH.sharded_layer_fwd(seg, par, ops=ops)
        else:
            SH.emulate_sharded(seg, par, [Ls], ops=ops)

    ms, clocks = timed(step, args.steps, args.warmup, world, dev, stream)
    ms_max = max_over_ranks(ms, world)
    step_ms = ms / args.steps
    elems = w.batch * Ls * w.d_inner
    res = {
        "value": whole_job_rate(w.batch * Ls * args.steps, world, ms_max / 1e3),
        "ms_per_step": ms_max / args.steps, "scaling": "strong",
        "gpu_launches": (2 * layer_launches(w.batch, w.d_inner, args, carry=True) + 1) * args.steps,
        "roofline": roofline(MUFU_PER_ELEM_LAYER * elems, step_ms / 2, clocks, w.name, kernel_name(w, args)),
        "clocks": clocks,
        "method": "two layer passes per segment (from zero for the aggregates, then from the composed carries)",
    }
    del seg
    torch.cuda.empty_cache()
    if rank == 0:
        proj = {}
        for R in (2, 4, 8):
            n = w.L // R
            one, p1 = W.make_case(w.batch, n, w.d_inner, w.d_state, w.dtype, w.seed + 100 + R, device=dev)
            h_all = torch.zeros(R, 2, w.batch, w.d_inner, w.d_state, device=dev)
            ds_all = torch.zeros(R, 2, w.batch, w.d_inner, device=dev)
            edges = torch.stack([SH.halo_edges(one)] * R)
            mid = R // 2  # a middle segment: both halos and both carries are real

            halo = SH.neighbour_halos(edges, mid)

            def share(i):
                SH.pass_from_zero(one, halo, p1, ops)
                SH.pass_with_carries(one, halo, p1, h_all, ds_all, mid, ops)

            k = max(3, args.steps // 4)
            ms_r, _ = timed(share, k, 2, 1, dev, stream)
            proj[str(R)] = {"per_rank_ms": round(ms_r / k, 3),
                            "projected_value": round(w.batch * w.L / (ms_r / k) / 1e3, 3)}
            del one
            torch.cuda.empty_cache()
        res["emulated_ranks"] = proj
        res["emulated_note"] = ("one rank's segment of L/R tokens timed on this GPU; projected_value = L / that "
                                "time, before the three all-gathers (a few hundred KB in all)")
    return res


def run_proj(args, w, bm, rank, world, dev, stream):
    """The layer's neighbours at the 1.3B shape: AdaLN of the hidden states,
    the input projection into the layer's inputs, and the output projection
    of a layer output, per step.  Two input sets alternate (each above L2).
    Each op is also timed alone, for its own roofline."""
    dm, D = w.extra["d_model"], w.d_inner
    M = w.batch * w.L
    cases = [W.make_proj_case(w.batch, w.L, dm, D, w.d_state, w.seed + 10 * i + rank, device=dev) for i in range(2)]
    a = torch.empty(w.batch, w.L, dm, device=dev, dtype=torch.bfloat16)
    ins = bm.bimamba_in_proj(a, cases[0]["w_in"], D)
    o = torch.empty(w.batch, w.L, dm, device=dev, dtype=torch.bfloat16)

    def op_adaln(i):
        c = cases[i & 1]
        bm.bimamba_adaln(c["h"], c["gamma"], c["beta"], out=a, stream=stream)

    def op_in(i):
        bm.bimamba_in_proj(a, cases[i & 1]["w_in"], D, out=ins, stream=stream)

    def op_out(i):
        c = cases[i & 1]
        bm.bimamba_out_proj(c["y"], c["w_out"], out=o, stream=stream)

    def step(i):
        op_adaln(i)
        op_in(i)
        op_out(i)

    ms, clocks = timed(step, args.steps, args.warmup, world, dev, stream)
    ms_max = max_over_ranks(ms, world)
    per = {}
    for name, fn in (("adaln", op_adaln), ("in_proj", op_in), ("out_proj", op_out)):
        t, _ = timed(fn, args.steps, args.warmup, 1, dev, stream)
        per[name] = t / args.steps
    f_in = 2.0 * M * dm * (4 * D + 4 * w.d_state)
    f_out = 2.0 * M * D * dm
    roof = roofline_tensor(f_in, per["in_proj"], w.name, "gemm_bf16_persistent_kernel (input projection)")
    adaln_bytes = M * dm * 2 * 2
    return {
        "value": whole_job_rate(M * args.steps, world, ms_max / 1e3),
        "ms_per_step": ms_max / args.steps, "gpu_launches": 3 * args.steps, "roofline": roof, "clocks": clocks,
        "kernels_ms": {k: round(v, 4) for k, v in per.items()},
        "out_proj_roofline": roofline_tensor(f_out, per["out_proj"], w.name, "gemm_bf16_persistent_kernel (output projection)"),
        "adaln_hbm": hbm_fraction(adaln_bytes, per["adaln"]),
        "note": "value = tokens through AdaLN + input projection + output projection per second",
    }


def run_ours(args, rank, world, local):
    from bidirectional_mamba_denoiser_b200 import bimamba as bm
    w = workload_of(args)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    if args.workload in ("block", "decode", "decode_mamba2"):
        side = torch.cuda.Stream(dev)  # graphs cannot be captured on the legacy default stream
        with torch.cuda.stream(side):
            res = (run_block if args.workload == "block" else run_decode)(args, w, bm, rank, world, dev, side)
    elif args.workload in ("mamba2", "mamba2_long"):
        res = run_mamba2(args, w, bm, rank, world, dev, stream)
    elif args.workload == "sharded":
        res = run_sharded(args, w, bm, rank, world, dev, stream)
    elif args.workload == "proj":
        res = run_proj(args, w, bm, rank, world, dev, stream)
    elif args.workload == "long" and args.segments > 1:
        res = run_chunked(args, w, bm, rank, world, dev, stream)
    else:
        res = run_layer_like(args, w, bm, rank, world, dev, stream)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(res.pop("value"), 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(res.pop("ms_per_step"), 5),
            "higher_is_better": True, "scaling": res.pop("scaling", "weak"), "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seq_len": w.L, "d_inner": w.d_inner,
                       "d_state": w.d_state,
                       "parallelism": f"sequence{world}" if args.workload == "sharded" else f"replicas{world}",
                       "l2": "inputs larger than L2 (rotating input sets)"
                       if args.workload not in ("block", "decode", "decode_mamba2")
                       else "block inputs rotate over 8 sets (state stays L2-resident, as in decoding)"},
            "roofline": res.pop("roofline"), "cpu_baseline": res.pop("cpu_baseline", None),
            "e2e": res.pop("e2e", None), "gpu_launches": res.pop("gpu_launches"), "clocks": res.pop("clocks"),
        }
        line.update(res)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------- reference arm (the oracle)

def run_reference(args, rank, world):
    """The fp64 CPU oracle, timed on the host cores on a channel sample of the
    same workload (rank 0 only; other ranks exit without work)."""
    if rank != 0:
        return None
    import oracle
    from tests import parity_util as U
    w = workload_of(args)
    if args.workload == "block":
        w = W.Workload(w.name, w.batch, w.extra["block"], w.d_inner, w.d_state, w.dtype, w.seed)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if args.workload in ("mamba2", "mamba2_long"):
        return run_reference_mamba2(args, w, world, dev)
    if args.workload == "proj":
        return run_reference_proj(args, w, world)
    inp, par = W.make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed, device=dev)
    threads = oracle.max_threads()
    per_step = min(30.0, 150.0 / max(1, args.steps + args.warmup))
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
    value = w.batch * w.L / layer_s / 1e6
    sample = (f"{len(chans)} of {w.d_inner} channels x {w.batch} batch rows x L={w.L} per step, scaled by "
              f"{w.d_inner}/{len(chans)}")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(layer_s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.L, "d_inner": w.d_inner,
                   "d_state": w.d_state, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "cpu_model": cpu_model(),
                         "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


def run_reference_proj(args, w, world):
    """The reference arm for the neighbours: the fp64 oracle (AdaLN and both
    projections, numpy) on a sample of token rows, scaled to all rows."""
    import oracle
    dm, D = w.extra["d_model"], w.d_inner
    M = w.batch * w.L
    c = W.make_proj_case(1, 256, dm, D, w.d_state, seed=w.seed)
    per_step = min(30.0, 150.0 / max(1, args.steps + args.warmup))

    def one(rows):
        h, y = c["h"][:, :rows], c["y"][:, :rows]
        a = oracle.adaln(h, c["gamma"], c["beta"])
        oracle.in_proj(a, c["w_in"], D)
        oracle.out_proj(y, c["w_out"])

    t0 = time.perf_counter()
    one(16)
    t1 = time.perf_counter() - t0
    rows = int(max(16, min(256, 16 * per_step / max(t1, 1e-3))))
    for _ in range(args.warmup):
        one(rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one(rows)
    secs = (time.perf_counter() - t0) / args.steps * M / rows
    value = M / secs / 1e6
    threads = oracle.max_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.L, "d_inner": D, "d_state": w.d_state,
                   "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "cpu_model": cpu_model(),
                         "kind": "oracle",
                         "sample": f"{rows} of {M} token rows per step (numpy fp64), scaled by {M}/{rows}"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


def run_reference_mamba2(args, w, world, dev):
    """The reference arm for the Mamba-2 workloads: the fp64 oracle on a sample
    of heads per step, scaled to all heads."""
    import oracle
    from tests import parity_util as U
    H, P, N = w.extra["nheads"], w.extra["headdim"], w.d_state
    inp, par = W.make_mamba2_case(w.batch, w.L, H, P, N, w.dtype, w.seed, device=dev)
    threads = oracle.max_threads()
    per_step = min(30.0, 150.0 / max(1, args.steps + args.warmup))
    si, sp, _ = U.head_subset(inp, par, [0])
    t0 = time.perf_counter()
    oracle.mamba2_layer_fwd(si, sp)
    t1 = time.perf_counter() - t0
    k = int(max(1, min(H, per_step / max(t1, 1e-3))))
    heads = sorted({int(h) for h in np.linspace(0, H - 1, k)})
    si, sp, _ = U.head_subset(inp, par, heads)
    for _ in range(args.warmup):
        oracle.mamba2_layer_fwd(si, sp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.mamba2_layer_fwd(si, sp)
    secs = time.perf_counter() - t0
    layer_s = secs / args.steps * H / len(heads)
    value = w.batch * w.L / layer_s / 1e6
    sample = f"{len(heads)} of {H} heads x {w.batch} batch rows x L={w.L} per step, scaled by {H}/{len(heads)}"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(layer_s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.L, "d_inner": w.d_inner,
                   "d_state": w.d_state, "nheads": H, "headdim": P, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "cpu_model": cpu_model(),
                         "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


def main():
    args = parse_args()
    rank, world, local = dist_init(args)
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
