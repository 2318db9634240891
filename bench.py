#!/usr/bin/env python
"""Benchmark of the fused MoE layer forward (moe_fused_forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config qwen36|nemotron|large_e|tiny] [--T 4096] [--routing router|zipf]
                    [--workload layer|router_topk] [--path auto|small|large]
                    [--schedule auto|static|dynamic] [--no-sweep | --sweep-all] [--no-cpu]

A step is one complete layer forward (router logits, top-k, permutation, FC1 + activation,
FC2 + weighted combine, shared expert, finalize) over T tokens of synthetic input drawn
by the seeded generator.  Rank 0 prints one JSON line.  With N > 1 (torchrun, one
process per GPU) every rank runs an independent replica on its own batch (the layer
has no cross-token exchange), the timed region is bracketed by barriers and
synchronisation, and the time is the maximum over ranks.

``--impl reference`` times the CPU oracle (single-threaded FP64 C) on a bounded token
sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_35_b200 import inputs as gen  # noqa: E402

L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2: written between timed steps
METRIC = "fused MoE layer \u00b5s & tokens/s vs T=1..8192, % HBM/tensor roofline, 1\u00d7B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, local, world


def dist_init(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def barrier(world: int, device=None):
    if world > 1:
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled during the timed region by a
    polling thread: NVML every 2 ms on the GPU matched by PCI bus id, else one-shot
    nvidia-smi queries back to back."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    NVML_BITS = (0x8, 0x40, 0x20, 0x4)  # the same reasons as NVML clock-event bits

    def __init__(self, gpu_index: int):
        import threading
        self.idx = gpu_index
        self.rows = []
        self.raw = []
        self.source = "nvidia-smi"
        self._nvml = self._nvml_handle(gpu_index)
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()

    @staticmethod
    def _nvml_handle(gpu_index):
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(gpu_index)
        except Exception:  # no NVML binding: fall back to nvidia-smi
            return None
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:
            pass
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return None

    def _query_nvml(self):
        nv, h = self._nvml
        try:
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
            getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            bits = getr(h)
        except Exception:
            return False
        act = ["Active" if bits & b else "Not Active" for b in self.NVML_BITS]
        self.rows.append([str(sm), str(mx), f"{pw:.1f}", hex(bits)] + act)
        return True

    def _query(self):
        try:
            r = subprocess.run(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
        except (OSError, subprocess.SubprocessError):
            return
        for line in r.stdout.strip().splitlines():
            self.raw.append(line)
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 8:
                self.rows.append(f)

    def _loop(self):
        while not self._stop.is_set():
            if self._nvml is not None and self._query_nvml():
                self.source = "nvml"
                time.sleep(0.002)
            else:
                self._query()

    def stop(self):
        self._stop.set()
        self._t.join(timeout=15)
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "raw": self.raw[:2]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [v for v in (num(r[0]) for r in self.rows) if v is not None]
        mx = [v for v in (num(r[1]) for r in self.rows) if v is not None]
        reasons = sorted({n for r in self.rows for n, v in zip(self.REASONS, r[4:8]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows), "source": self.source}


# ---------------------------------------------------------------- algorithmic accounting
def accounting(shape, T: int, U: int, router: bool, Is: int):
    """Algorithmic bytes / flops of the layer and of each kernel.  U = distinct routed
    experts touched by the call.  Weights of untouched experts are not counted; h, acc,
    permutation indices are implementation traffic, except where a kernel's own
    operand is h (FC2 reads it, FC1 writes it)."""
    H, I, E, K = shape.H, shape.I, shape.E, shape.K
    rows1 = 2 * I if shape.act == "swiglu" else I
    rows1s = 2 * Is if shape.act == "swiglu" else Is
    h_bytes = (T * K * I + T * Is) * 2
    k = {}
    k["prep"] = {"bytes": E * H * 2 if router and T > 64 else 0, "flops": 0}
    k["router"] = {"bytes": E * H * 2 + T * H * 2 + T * E * 4, "flops": 2 * T * E * H}
    k["topk"] = {"bytes": T * E * 4 + T * K * 8, "flops": 0}
    k["route"] = {"bytes": T * E * 4 + T * K * 8, "flops": 0}
    # exact re-evaluation of ~K candidate logits per token: an x row and a router row each
    k["refine"] = {"bytes": T * K * H * 2 * 2, "flops": 2 * T * K * H}
    k["select"] = {"bytes": T * K * 12 + T * K * 8, "flops": 0}
    k["permute"] = {"bytes": T * K * 4 * 2, "flops": 0}
    k["fc1"] = {"bytes": U * rows1 * H * 2 + rows1s * H * 2 + T * H * 2 + h_bytes,
                "flops": 2 * T * K * rows1 * H + 2 * T * rows1s * H}
    k["fc2"] = {"bytes": U * H * I * 2 + H * Is * 2 + h_bytes + T * H * 2,
                "flops": 2 * T * K * H * I + 2 * T * H * Is}
    k["finalize"] = {"bytes": T * H * (4 + 2 + (2 if Is else 0)), "flops": 0}
    layer_bytes = U * (rows1 + I) * H * 2 + (E * H * 2 if router else 0) + 2 * T * H * 2 + \
        (rows1s + Is) * H * 2 + 4 * E
    layer_flops = 2 * T * K * (rows1 + I) * H + (2 * T * E * H if router else 0) + 2 * T * (rows1s + Is) * H
    return {"layer": {"bytes": layer_bytes, "flops": layer_flops}, "kernels": k}


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu
# capture of the default workload (seed 0, one GPU), keyed by (config, T, routing, kernel).
# The capture and its command are summarised in profiles/; an entry is removed whenever
# its kernel changes, so that a stale count is never reported.
NCU_TRAFFIC = {
    ("qwen36", 4096, "router", "fc1"): 1.174206e9 + 66.226432e6,
    ("qwen36", 4096, "router", "fc2"): 0.626002e9 + 12.780800e6,
}


def roofline_of(acc: dict, dur_s: float, peaks: dict):
    t_hbm = acc["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = acc["flops"] / (peaks["bf16_tflops"] * 1e12)
    if t_tc > t_hbm:
        ach = acc["flops"] / dur_s / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"]}
    ach = acc["bytes"] / dur_s / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}


# ---------------------------------------------------------------- our arm
class Bench:
    def __init__(self, shape, T, device, seed, routing, path="auto", schedule="auto", tiles=(0, 0)):
        import mixture_experts_layer_35_b200.moe as moe
        self.moe = moe
        self.shape, self.T, self.device = shape, T, device
        self.d = gen.make_layer(shape, T, seed=seed, device=str(device), routing=routing)
        self.logits = self.d["router_logits"]
        w = {k: self.d[k] for k in ("router_w", "bias", "w13", "w2", "ws13", "ws2") if self.d.get(k) is not None}
        self.layer = moe.MoELayer(shape, w, path=path, schedule=schedule, tiles=tiles)
        self.desc = self.layer.desc(T, self.logits)
        self.ws = self.layer.workspace(self.desc, device)
        self.out = torch.empty((T, shape.H), dtype=torch.bfloat16, device=device)
        self.path = moe.select_path(self.desc)
        self.launches = moe.launches(self.desc)
        self.Is = shape.I_shared if w.get("ws13") is not None else 0
        self.flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        # One complete layer forward per CUDA-graph replay (the launch sequence is
        # captured once; replays carry no host launch overhead).
        self.stream = torch.cuda.Stream(device)
        # The inputs were generated, and the workspace allocated, in the default stream's
        # order: the side stream may only start once that work is done (the workspace can
        # reuse a block that a pending generator kernel still writes).
        torch.cuda.synchronize(device)
        self.step_eager(stream=self.stream)  # tensor-map and attribute set-up outside capture
        torch.cuda.synchronize(device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            self.step_eager(stream=self.stream)
        torch.cuda.synchronize(device)

    def flush(self):
        self.flush_buf.fill_(1)

    def step_eager(self, x=None, out=None, stream=None):
        self.moe.fused_forward_raw(self.desc, self.d["x"] if x is None else x, self.out if out is None else out,
                                   self.ws, stream=stream)

    def step(self):
        self.graph.replay()

    def distinct_experts(self):
        _, _, ids, _ = self.layer.forward(self.d["x"], router_logits=self.logits, return_routing=True,
                                          stream=self.stream)
        torch.cuda.synchronize(self.device)
        return int(torch.unique(ids).numel())

    def timed(self, steps: int, warmup: int, world: int = 1, clocks=None):
        for _ in range(warmup):
            self.flush()
            self.step()
        torch.cuda.synchronize(self.device)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        barrier(world, self.device)
        torch.cuda.synchronize(self.device)
        sampler = ClockSampler(self.device.index) if clocks else None
        for a, b in evs:
            self.flush()
            a.record()
            self.step()
            b.record()
        torch.cuda.synchronize(self.device)
        clk = sampler.stop() if sampler else None
        barrier(world, self.device)
        per = [a.elapsed_time(b) for a, b in evs]
        self.last_step_s = statistics.median(per) / 1e3 + 2e-5
        return per, clk

    def telemetry(self):
        """Phase trace of one eager forward behind an L2 flush (moe_layer_desc.trace):
        per tensor-core kernel, launch skew, input wait, load span, tail."""
        trace = self.moe.trace_buffer(self.device)
        desc = self.layer.desc(self.T, self.logits, trace=trace)
        self.flush()
        self.moe.fused_forward_raw(desc, self.d["x"], self.out, self.ws, stream=self.stream)
        torch.cuda.synchronize(self.device)
        return self.moe.trace_summary(trace, torch.cuda.get_device_properties(self.device).multi_processor_count)

    def clock_soak(self, seconds: float):
        """Clocks while the same step (L2 flush + graph replay) repeats back to back for
        about ``seconds``: a longer window than a short timed region gives the sampler."""
        n = max(1, int(seconds / max(self.last_step_s, 1e-5)))
        sampler = ClockSampler(self.device.index)
        for _ in range(n):
            self.flush()
            self.step()
        torch.cuda.synchronize(self.device)
        out = sampler.stop()
        out["steps"] = n
        return out

    def per_kernel(self, steps: int):
        """Average duration of each kernel of the step, from events recorded between the
        launches (moe_fused_forward_timed).  Each call is enqueued right behind the L2
        flush, so the host enqueues the kernels while the GPU is still busy and no
        launch gap enters the intervals; the events do stop consecutive kernels from
        overlapping, so the sum exceeds the graph-replay step slightly."""
        n = self.launches
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        for e in evs:  # torch creates the CUDA event on its first record
            e.record()
        self.kernel_timing = "events between launches enqueued behind the L2 flush"
        tot = np.zeros(n)
        for _ in range(steps):
            self.flush()
            self.moe.fused_forward_timed(self.desc, self.d["x"], self.out, self.ws, evs)
            torch.cuda.synchronize(self.device)
            tot += np.array([evs[i].elapsed_time(evs[i + 1]) for i in range(n)])
        return tot / steps

    def e2e(self, steps: int, warmup: int):
        """End to end through the public forward call, every step copying its input x from
        pinned host memory and reading its output back to pinned host memory.

        Returns (pipelined ms per step, serial ms per step, H2D bytes, D2H bytes).  The
        pipelined loop is how a serving loop runs the layer: the input copy, the forward
        and the read-back each have a stream, with two device buffers for x and for out,
        so step i's forward overlaps step i+1's input copy and step i-1's read-back.  It
        writes no L2 flush between steps: each step streams its 1.6+ GB of weights,
        far more than L2.  The serial loop runs copy, forward, read-back one after
        another, behind an L2 flush each step."""
        T, H = self.T, self.shape.H
        dev = self.device
        x_host = self.d["x"].to("cpu").pin_memory()
        out_host = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(self.d["x"]) for _ in range(2)]
        out_dev = [torch.empty_like(self.out) for _ in range(2)]
        s_in, s_fwd, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_fwd = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        torch.cuda.synchronize(dev)

        def pipelined_step(i):
            b = i % 2
            if i >= 2:  # buffer pair b was last used by step i - 2
                s_in.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(s_in)
            s_fwd.wait_event(ev_in[b])
            if i >= 2:
                s_fwd.wait_event(ev_out[b])
            self.moe.fused_forward_raw(self.desc, x_dev[b], out_dev[b], self.ws, stream=s_fwd)
            ev_fwd[b].record(s_fwd)
            s_out.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out_dev[b], non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(warmup):
            pipelined_step(i)
        torch.cuda.synchronize(dev)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(s_in)
        for i in range(steps):
            pipelined_step(i)
        end.record(s_out)
        torch.cuda.synchronize(dev)
        pipelined = start.elapsed_time(end) / steps

        serial = []
        for _ in range(steps):
            self.flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            x_dev[0].copy_(x_host, non_blocking=True)
            self.step_eager(x=x_dev[0])
            out_host[0].copy_(self.out, non_blocking=True)
            b.record()
            torch.cuda.synchronize(dev)
            serial.append(a.elapsed_time(b))
        return pipelined, float(np.mean(serial)), T * H * 2, T * H * 2


def cpu_oracle_rate(shape, d, budget_s: float, max_tokens: int):
    """Tokens/s of the single-threaded CPU oracle on a bounded sample of the workload."""
    import oracle
    h = gen.to_numpy_inputs(d)
    T = h["x"].shape[0]
    rows = np.random.default_rng(0).permutation(T)[:max_tokens].astype(np.int32)
    done, t0 = 0, time.perf_counter()
    while done < len(rows) and time.perf_counter() - t0 < budget_s:
        oracle.forward(shape, h, rows[done:done + 1])
        done += 1
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def cpu_oracle_rate_all_cores(shape, d, tokens_per_core: int):
    """Tokens/s of the same single-threaded oracle sharded by token ranges over every host
    core as separate processes (oracle.parallel).  The workers are started, and have
    mapped the inputs, before the timed span."""
    from oracle import parallel as opar
    h = gen.to_numpy_inputs(d)
    T = h["x"].shape[0]
    cores = opar.host_cores()
    n = min(T, cores * tokens_per_core)
    rows = np.random.default_rng(1).permutation(T)[:n].astype(np.int32)
    with opar.ShardedOracle(shape, h, cores) as pool:
        pool.forward(rows[:cores])  # workers started and inputs mapped before the timed span
        t0 = time.perf_counter()
        pool.forward(rows)
        dt = time.perf_counter() - t0
    return n / dt, n, dt, cores


def host_cpu_info():
    """Core count and CPU model of the host (lscpu), for the CPU-baseline lines."""
    from oracle import parallel as opar
    model = None
    try:
        r = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10)
        for line in r.stdout.splitlines():
            if line.startswith("Model name:"):
                model = line.split(":", 1)[1].strip()
                break
    except (OSError, subprocess.SubprocessError):
        pass
    return {"nproc": opar.host_cores(), "cpu_count": os.cpu_count(), "model": model}


def run_ours(args, rank, local, world):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    shape = gen.SHORT[args.config]
    peaks, peaks_src = load_peaks()
    b = Bench(shape, args.T, device, seed=args.seed + rank, routing=args.routing, path=args.path,
              schedule=args.schedule, tiles=(args.fc1_tile, args.fc2_tile))
    per, clk = b.timed(args.steps, args.warmup, world, clocks=True)
    local_ms = float(sum(per))
    total_ms = max_over_ranks(local_ms, world, device)
    ms_step = total_ms / args.steps
    value = world * args.T * args.steps / (total_ms / 1e3)

    U = b.distinct_experts()
    router = b.logits is None
    acc = accounting(shape, args.T, U, router, b.Is)
    kt = b.per_kernel(max(3, min(args.steps, 10)))
    names = b.moe.kernel_plan(b.desc)
    dom = int(np.argmax(kt))
    dom_name = names[dom]
    roof = roofline_of(acc["kernels"][dom_name], kt[dom] / 1e3, peaks)
    roof["kernel"] = f"{dom_name} ({b.path} path)"
    roof["timing"] = b.kernel_timing
    roof["traffic"] = (NCU_TRAFFIC.get((args.config, args.T, args.routing, dom_name))
                       if args.seed == 0 and b.path == "large" else None)
    roof["peak_source"] = f"of {peaks_src}"
    layer_roof = roofline_of(acc["layer"], ms_step / 1e3, peaks)
    e2e_pipe, e2e_serial, bi, bo = b.e2e(args.steps, args.warmup)
    e2e_pipe = max_over_ranks(e2e_pipe, world, device)
    e2e_serial = max_over_ranks(e2e_serial, world, device)
    e2e_value = world * args.T / (e2e_pipe / 1e3)

    telem = b.telemetry() if b.path == "large" else None
    clk_soak = b.clock_soak(args.soak_s) if args.soak_s > 0 else None
    dev_err = b.moe.get_error(b.ws)
    line = {
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded generator, random-init weights of the layer's shape)",
        "config": {"workload": f"{shape.name} T={args.T} routing={args.routing}", "tokens_per_step": args.T,
                   "timing": "one CUDA-graph replay of moe_fused_forward per step",
                   "path": b.path, "schedule": args.schedule, "token_tiles": list(b.moe.token_tiles(b.desc)),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write), steps timed with CUDA events",
                   "distinct_experts": U},
        "roofline": roof,
        "layer_roofline": layer_roof,
        "kernel_ms": {n: round(float(v), 5) for n, v in zip(names, kt)},
        "telemetry": telem,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                "timing": "public forward call per step, pinned H2D of x and D2H of out inside each step; "
                          "copy-in, forward and read-back on three streams with double buffers, steps "
                          "pipelined, no L2 flush (each step streams more weight bytes than L2 holds)",
                "serial_value": world * args.T / (e2e_serial / 1e3),
                "serial_timing": "copy-in, forward, read-back one after another, L2 flushed before each step"},
        "gpu_launches": b.launches * args.steps,
        "device_error": dev_err,
        "clocks": clk,
        "clocks_soak": clk_soak,
        "us_per_step_p10_p50_p90": [float(np.percentile(per, q)) * 1e3 for q in (10, 50, 90)],
    }
    del b
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_sweep:
        line["sweep"] = sweep(args, device, peaks)
    if rank == 0 and world == 1 and not args.no_cpu:
        dcpu = gen.make_layer(shape, args.T, seed=args.seed, device=str(device), routing=args.routing)
        rate1, n1, dt1 = cpu_oracle_rate(shape, dcpu, args.cpu_budget / 3, 400)
        per_core = max(1, int(rate1 * args.cpu_budget * 2 / 3))
        rate, n, dt, cores = cpu_oracle_rate_all_cores(shape, dcpu, per_core)
        info = host_cpu_info()
        line["cpu_baseline"] = {
            "value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} random tokens of the same workload in {dt:.1f} s: the single-threaded FP64 C oracle "
                      f"sharded by token ranges over {cores} processes",
            "host": info,
            "single_core": {"value": rate1, "unit": "tokens/s", "cores": 1,
                            "sample": f"{n1} tokens in {dt1:.1f} s on one core"}}
        del dcpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier(world, device)
    if world > 1:
        torch.distributed.destroy_process_group()


def sweep(args, device, peaks):
    """Per-T latency curve of the layer (median of short timed runs, L2 flushed)."""
    rows = []
    plan = [("qwen36", t) for t in gen.T_SWEEP]
    if args.sweep_all:
        plan += [("nemotron", t) for t in gen.T_SWEEP] + [("large_e", t) for t in gen.LARGE_E_T]
    cache = {}
    for cfg, T in plan:
        shape = gen.SHORT[cfg]
        print(f"sweep: {cfg} T={T}", file=sys.stderr, flush=True)
        try:
            b = Bench(shape, T, device, seed=1, routing="router", path=args.path, schedule=args.schedule)
            per, _ = b.timed(args.sweep_steps, 5)
            med = statistics.median(per)
            U = b.distinct_experts()
            acc = accounting(shape, T, U, True, b.Is)["layer"]
            rf = roofline_of(acc, med / 1e3, peaks)
            rows.append({"config": cfg, "T": T, "path": b.path, "us": med * 1e3,
                         "us_p10_p90": [float(np.percentile(per, 10)) * 1e3, float(np.percentile(per, 90)) * 1e3],
                         "steps": len(per), "tokens_per_s": T / (med / 1e3),
                         "distinct_experts": U, "bound": rf["bound"], "frac_of_roofline": rf["frac"],
                         "achieved": rf["achieved"], "unit": rf["unit"],
                         "device_error": b.moe.get_error(b.ws)})
            del b
        except Exception as e:  # report, keep sweeping
            rows.append({"config": cfg, "T": T, "error": str(e)[:200]})
        cache.clear()
        torch.cuda.empty_cache()
    return rows


# ---------------------------------------------------------------- router top-k alone
ROUTER_E, ROUTER_K = 256, 10


def run_router_topk(args, rank, local, world):
    """The router-top-k-only workload: moe_router_topk on BF16 logits [M, 256] (M = --T),
    sigmoid scores, an FP32 selection bias ~ N(0, 0.5), top-10, renormalised, with ~10 %
    of rows holding a designed exact tie.  One step is one call over all M rows."""
    import mixture_experts_layer_35_b200.moe as moe
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    peaks, peaks_src = load_peaks()
    M, E, K = args.T, ROUTER_E, ROUTER_K
    case = gen.make_router_case(M, E, K, seed=args.seed + rank, bias_mode="random")
    lg = case["logits"].to(device)
    bias = case["bias"].to(device)
    outs = tuple(torch.empty((M, K), dtype=dt, device=device) for dt in (torch.float32, torch.int32, torch.int32))
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.Stream(device)
    call = lambda x=lg: moe.router_topk(x, K, "sigmoid", bias, True, stream=stream, out=outs)  # noqa: E731
    torch.cuda.synchronize(device)  # inputs and outputs were made in the default stream's order
    call()
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call()
    torch.cuda.synchronize(device)
    for _ in range(args.warmup):
        flush_buf.fill_(1)
        graph.replay()
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize(device)
    sampler = ClockSampler(device.index)
    for a, b in evs:
        flush_buf.fill_(1)
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize(device)
    clk = sampler.stop()
    barrier(world, device)
    per = [a.elapsed_time(b) for a, b in evs]
    total_ms = max_over_ranks(float(sum(per)), world, device)
    ms_step = total_ms / args.steps
    value = world * M * args.steps / (total_ms / 1e3)
    acc = {"bytes": M * E * 2 + E * 4 + M * K * 12, "flops": 0}
    roof = roofline_of(acc, ms_step / 1e3, peaks)
    roof.update({"kernel": "topk_kernel", "timing": "CUDA-graph replay, one launch per step", "traffic": None,
                 "peak_source": f"of {peaks_src}"})
    # end to end: pinned host logits in, weights and ids out, through the public call
    lg_host = case["logits"].pin_memory()
    w_host = torch.empty((M, K), dtype=torch.float32).pin_memory()
    id_host = torch.empty((M, K), dtype=torch.int32).pin_memory()
    lg_dev = torch.empty_like(lg)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush_buf.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        lg_dev.copy_(lg_host, non_blocking=True)
        moe.router_topk(lg_dev, K, "sigmoid", bias, True, out=outs)
        w_host.copy_(outs[0], non_blocking=True)
        id_host.copy_(outs[1], non_blocking=True)
        b.record()
        torch.cuda.synchronize(device)
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_total = max_over_ranks(float(sum(e2e_ms)), world, device)
    line = {
        "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded generator, designed ties)",
        "config": {"workload": f"router-top-k-only BF16 logits [{M},{E}] top-{K} sigmoid+bias renorm",
                   "rows_per_step": M, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)"},
        "roofline": roof,
        "e2e": {"value": world * M * args.steps / (e2e_total / 1e3), "unit": "rows/s",
                "h2d_bytes_per_step": M * E * 2, "d2h_bytes_per_step": M * K * 8},
        "gpu_launches": args.steps, "clocks": clk,
        "us_per_step_p10_p50_p90": [float(np.percentile(per, q)) * 1e3 for q in (10, 50, 90)],
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        import oracle
        hl = gen.bf16_bits(case["logits"])
        hb = case["bias"].numpy()
        t0, n = time.perf_counter(), 0
        while n < M and time.perf_counter() - t0 < args.cpu_budget:
            oracle.topk(hl[n:n + 64], K, "sigmoid", hb, True, logits_bf16=True)
            n += min(64, M - n)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n / dt, "unit": "rows/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} rows of the same logits in {dt:.2f} s (single-threaded C)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier(world, device)
    if world > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------- reference arm (CPU oracle)
def run_reference(args, rank, local, world):
    if rank != 0:
        return
    shape = gen.SHORT[args.config]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    d = gen.make_layer(shape, args.T, seed=args.seed, device=dev, routing=args.routing)
    import oracle
    h = gen.to_numpy_inputs(d)
    del d
    from oracle import parallel as opar
    cores = opar.host_cores() if args.ref_cores == 0 else args.ref_cores
    sample = max(1, args.ref_tokens) * cores
    rng = np.random.default_rng(0)
    times = []
    # The worker processes and their memory-mapped copy of the inputs are set up once,
    # outside the timed steps (as loading the weights is for the GPU arm).
    pool = opar.ShardedOracle(shape, h, cores) if cores > 1 else None
    try:
        for i in range(args.warmup + args.steps):
            rows = rng.choice(args.T, min(sample, args.T), replace=False).astype(np.int32)
            t0 = time.perf_counter()
            if pool is None:
                oracle.forward(shape, h, rows)
            else:
                pool.forward(rows)
            dt = time.perf_counter() - t0
            if i >= args.warmup:
                times.append(dt)
    finally:
        if pool is not None:
            pool.close()
    tot = sum(times)
    sample = min(sample, args.T)
    value = sample * args.steps / tot
    line = {"impl": "reference", "metric": METRIC,
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded generator)",
            "config": {"workload": f"{shape.name} T={args.T} routing={args.routing}",
                       "sample": f"{sample} tokens per step"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{sample} random tokens of the workload per step, the single-threaded "
                                       f"FP64 C oracle sharded by token ranges over {cores} processes",
                             "host": host_cpu_info()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=["layer", "router_topk"], default="layer",
                   help="layer: moe_fused_forward on --config; router_topk: moe_router_topk alone, M = --T rows")
    p.add_argument("--config", choices=sorted(gen.SHORT), default="qwen36")
    p.add_argument("--T", type=int, default=4096)
    p.add_argument("--routing", choices=["router", "zipf"], default="router")
    p.add_argument("--path", choices=["auto", "small", "large"], default="auto",
                   help="force an execution path (selector studies); auto = the library's choice")
    p.add_argument("--schedule", choices=["auto", "static", "dynamic"], default="auto",
                   help="tile schedule of the grouped GEMMs (auto = the library's choice)")
    p.add_argument("--fc1-tile", type=int, default=0, help="FC1 token rows per tile (0 = the library's choice)")
    p.add_argument("--fc2-tile", type=int, default=0, help="FC2 token rows per tile (0 = the library's choice)")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--sweep-all", action="store_true")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline (profiling runs)")
    p.add_argument("--cpu-budget", type=float, default=15.0)
    p.add_argument("--ref-tokens", type=int, default=4, help="reference arm: tokens per core per step")
    p.add_argument("--ref-cores", type=int, default=0, help="reference arm: processes (0 = every host core)")
    p.add_argument("--sweep-steps", type=int, default=30)
    p.add_argument("--soak-s", type=float, default=1.0,
                   help="seconds of repeated steps after the timed region, for a longer clock record")
    args = p.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    rank, local, world = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, local, world)
    elif args.workload == "router_topk":
        run_router_topk(args, rank, local, world)
    else:
        run_ours(args, rank, local, world)


if __name__ == "__main__":
    main()
