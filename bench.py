#!/usr/bin/env python
"""Throughput of the 3LC codec on B200, one JSON line on stdout (rank 0).

A step is one pass of the whole hot path over one synthetic gradient:
tlc_compress (error feedback, magnitude, ternary quantization with sparsity
multiplication, quartic packing, zero-run encoding), tlc_decompress (dense
fp32 output) and tlc_decompress_accumulate (the stream added into a dense
fp32 aggregation buffer).  The workload is the flat 2^28-value fp32 tensor,
Laplace(0, 1e-4) with 90% exact zeros in geometric runs (mean 64), s = 1.9,
with the error buffer carried from step to step and a fresh gradient every
step (a few seeded gradients resident on the device, taken in turn).  Inputs
(2 GiB of x + err) exceed the 126 MB L2, so every step streams from HBM.

value = 4n bytes of fp32 input per step and GPU / device time per step.
Under torchrun each rank compresses its own tensor (replicas, weak scaling);
the step time is the maximum over ranks.  `--impl reference` times the CPU
oracle on a bounded sample of the same workload instead.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("compress & decompress GB/s of fp32 input on 1 B200; % of HBM roofline; "
          "bits/value")
S_PARAM = 1.9


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--log2n", type=int, default=28, help="tensor size 2^k (default 28)")
    p.add_argument("--e2e-steps", type=int, default=8)
    p.add_argument("--dense", action="store_true",
                   help="config 3 shape with uniform values and s = 1: a dense stream "
                        "(the decoder's weak case), an extra line, not the headline")
    p.add_argument("--grads", type=int, default=4,
                   help="seeded gradients kept on the device and taken in turn, one per step")
    p.add_argument("--cpu-baseline-log2n", type=int, default=26)
    p.add_argument("--cpu-baseline-seconds", type=float, default=10.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sweep", action="store_true",
                   help="--impl reference: also time the oracle per direction over the "
                        "config-3 sweep 2^20..2^24 and configs 1 and 5")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--graph", action="store_true",
                   help="configs 2, 4, 5: replay each step from a CUDA graph of its calls")
    p.add_argument("--per-tensor", action="store_true",
                   help="configs 2/4: one C-ABI call per tensor instead of a plan")
    p.add_argument("--exchange", choices=["allgather", "sharded"], default=None,
                   help="time the data-parallel exchange step (NCCL, every rank) on the "
                        "headline workload instead of the single-GPU codec step")
    p.add_argument("--config", type=int, default=3, choices=[1, 2, 3, 4, 5],
                   help="workload: 3 (default, the headline) or another of the five "
                        "parity configs, measured the same way (extra lines)")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def gradient(args, n, step):
    """The gradient of one step: the workload's seeded tensor, or with
    --dense uniform values in [-1, 1) (with s = 1 a large share of the values
    quantize to +-1, so nearly every group is a literal byte of the stream)."""
    import numpy as np

    import synth
    if args.dense:
        return (synth.uniforms(synth.key_for(step, 5), n) * 2 - 1).astype(np.float32)
    return synth.flat_tensor(args.config, n=n, step=step)


def workload_config(n, log2n, dense=False):
    if dense:
        return {
            "workload": (f"flat fp32 tensor of 2^{log2n} values, uniform in [-1, 1), s=1.0 "
                         "(a dense stream, about one byte per five values); step = compress "
                         "+ decompress + decompress-accumulate (K=1), error buffer carried, a "
                         "fresh gradient each step"),
            "n": n, "s": 1.0, "input_bytes_per_step": 4 * n,
            "l2": "inputs (x + err = 8n bytes) larger than the 126 MB L2; no flush"
            if n >= 1 << 24 else "inputs partly L2-resident"}
    return {
        "workload": (f"flat fp32 tensor of 2^{log2n} values, Laplace(0,1e-4) with 90% exact "
                     f"zeros in geometric runs (mean 64), s={S_PARAM}; step = compress + "
                     "decompress + decompress-accumulate (K=1), error buffer carried, a "
                     "fresh gradient each step (seeded gradients resident on the device, "
                     "taken in turn)"),
        "n": n,
        "s": S_PARAM,
        "input_bytes_per_step": 4 * n,
        "l2": "inputs (x + err = 8n bytes) larger than the 126 MB L2; no flush",
    }


# ----------------------------------------------------------- clock sampler --

class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML (read-only queries)
    every `period` seconds on a background thread; only samples between
    mark("start") and mark("end") are summarised."""

    NAMES = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
             ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
             ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
             ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, bus_id=None, period=0.01):
        import threading

        import pynvml
        pynvml.nvmlInit()
        self.nv = pynvml
        self.h = (pynvml.nvmlDeviceGetHandleByPciBusId(bus_id) if bus_id
                  else pynvml.nvmlDeviceGetHandleByIndex(0))
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        self.samples = []
        self.period = period
        self.halt = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv, h = self.nv, self.h
        while not self.halt.is_set():
            try:
                self.samples.append((time.time(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                pass
            self.halt.wait(self.period)

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        self.halt.set()
        self.thread.join(5)
        t0, t1 = getattr(self, "start", None), getattr(self, "end", None)
        rows = [r for r in self.samples if t0 is None or t1 is None or t0 <= r[0] <= t1]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"],
                    "samples": 0, "source": "nvml"}
        reasons = sorted({name for _, _, bits in rows for name, attr in self.NAMES
                          if bits & getattr(self.nv, attr)})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": self.max_mhz,
                "sm_min_mhz": min(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "source": "nvml"}


def ClockSampler(bus_id=None):
    """NVML sampler when pynvml works, else nvidia-smi -lms."""
    try:
        return NvmlClockSampler(bus_id)
    except Exception:
        return SmiClockSampler(bus_id)


class SmiClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id=None):
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "50"]
        if bus_id:
            cmd += ["-i", bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def mark(self, which):
        """Record the host time at which the timed region starts / ends."""
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.split(",") for r in self.tmp.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.tmp.name)
        t0, t1 = getattr(self, "start", None), getattr(self, "end", None)
        if t0 is not None and t1 is not None:
            import datetime as _dt
            kept = []
            for r in rows:
                try:
                    ts = _dt.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    continue
                if t0 - 0.03 <= ts <= t1 + 0.03:
                    kept.append(r)
            rows = kept or rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ ours ----

def run_ours(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    import gradient_traffic_compression_b200 as tlc
    import synth
    from gradient_traffic_compression_b200.exchange import max_over_ranks

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    global S_PARAM
    if args.config == 1:
        S_PARAM = synth.CONFIGS[1]["s"]
        args.log2n = 20
        args.no_e2e = True
        args.no_cpu_baseline = True
    if args.dense:
        S_PARAM = 1.0
        args.no_cpu_baseline = True
    n = 1 << args.log2n
    # A fresh gradient every step: a few seeded gradients of the workload,
    # resident on the device, taken in turn (each rank its own), while the
    # error buffer carries over from step to step.
    xs = []
    for k in range(args.grads):
        xs.append(torch.from_numpy(gradient(args, n, 1000 * rank + k)).to(dev))
    err = torch.zeros(n, dtype=torch.float32, device=dev)
    cap = tlc.tlc_compress_bound(n)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    out_len = torch.zeros(1, dtype=torch.int64, device=dev)
    y = torch.empty(n, dtype=torch.float32, device=dev)
    acc = torch.zeros(n, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    turn = [0]

    def step():
        x = xs[turn[0] % len(xs)]
        turn[0] += 1
        tlc.tlc_compress(x, S_PARAM, err, out, out_len, status, stream)
        tlc.tlc_decompress(out, n, y, in_len=out_len, in_cap=cap, dev_status=status,
                           stream=stream)
        tlc.tlc_decompress_accumulate([out], n, acc, in_lens=out_len, in_caps=[cap],
                                      dev_status=status, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")

    bus = None
    try:
        pr = torch.cuda.get_device_properties(dev)
        bus = "%08X:%02X:%02X.0" % (int(pr.pci_domain_id), int(pr.pci_bus_id),
                                    int(pr.pci_device_id))
    except Exception:
        bus = None

    # The dominant kernel kind, from a pass with every kind timed (part of
    # the warm-up, untimed).
    tlc.tlc_kernel_timing_kinds(None)
    tlc.tlc_kernel_timing(True)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    tlc.tlc_kernel_timing(False)
    pre = tlc.tlc_kernel_timing_read()
    dom = max((k for k in pre if pre[k][0]), key=lambda k: pre[k][1])

    # --graph: CUDA graphs of the calls, so that small tensors are timed on
    # the GPU rather than at the host's launch rate.  Per resident gradient:
    # one graph of `reps` whole steps (the timed region) and one graph of
    # `reps` calls of each leg (the breakdown pass); reps shrinks as the
    # tensor grows, to 1 from 2^26 values on.
    graphs, leg_graphs = [], []
    graph_launches = None
    reps = max(1, min(32, 1 << max(0, 26 - args.log2n))) if args.graph else 1
    if args.graph:
        tlc.tlc_kernel_timing_kinds([])
        tlc.tlc_kernel_timing(True)
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(stream)
        calls = [
            lambda k: tlc.tlc_compress(xs[k], S_PARAM, err, out, out_len, status, cs),
            lambda k: tlc.tlc_decompress(out, n, y, in_len=out_len, in_cap=cap,
                                         dev_status=status, stream=cs),
            lambda k: tlc.tlc_decompress_accumulate([out], n, acc, in_lens=out_len,
                                                    in_caps=[cap], dev_status=status, stream=cs),
        ]
        for k in range(len(xs)):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cs):
                for _ in range(reps):
                    for call in calls:
                        call(k)
            graphs.append(gr)
        tlc.tlc_kernel_timing(False)
        per_graph = tlc.tlc_kernel_timing_read()
        graph_launches = sum(v[0] for v in per_graph.values()) / len(graphs) / reps
        for k in range(len(xs)):
            trio = []
            for call in calls:
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=cs):
                    for _ in range(reps):
                        call(k)
                trio.append(gr)
            leg_graphs.append(trio)
        for gr in graphs:
            gr.replay()
        for trio in leg_graphs:
            for gr in trio:
                gr.replay()
        torch.cuda.synchronize()
        args.steps = max(reps, args.steps // reps * reps)

    # Timed region: K steps between two events, with an event pair around
    # each launch of the dominant kernel only (each pair costs a few
    # microseconds of device time).  Every launch is counted.
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(bus)
    time.sleep(0.2)
    tlc.tlc_kernel_timing_kinds([dom])
    tlc.tlc_kernel_timing(True)
    sampler.mark("start")
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    if graphs:
        for i in range(args.steps // reps):
            graphs[i % len(graphs)].replay()
    else:
        for i in range(args.steps):
            step()
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark("end")
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    tlc.tlc_kernel_timing(False)
    kern = tlc.tlc_kernel_timing_read()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")
    total_ms = t_start.elapsed_time(t_end)
    if graphs:
        # replays do not pass through the library: the dominant kernel's
        # launch time comes from the timed pre-pass, launches from the capture
        dom_ms = pre[dom][1] / max(pre[dom][0], 1)
        kern = {k: (int(graph_launches * args.steps) if k == dom else 0, 0.0) for k in kern}
        kern[dom] = (int(graph_launches * args.steps), 0.0)
    else:
        dom_ms = kern[dom][1] / max(kern[dom][0], 1)
    total_ms, dom_ms = max_over_ranks([total_ms, dom_ms], device=dev)

    # Breakdown pass after the timed region (not part of `value`): every
    # kind timed, and events between the three calls of each step.
    steps2 = max(1, min(args.steps, 100))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps2)]
    tlc.tlc_kernel_timing_kinds(None)
    tlc.tlc_kernel_timing(True)
    for k in range(steps2):
        e = ev[k]
        e[0].record(stream)
        if graphs:
            # each leg replayed from its graph of `reps` calls, events between
            for i, gr in enumerate(leg_graphs[k % len(leg_graphs)]):
                gr.replay()
                e[i + 1].record(stream)
            continue
        tlc.tlc_compress(xs[k % len(xs)], S_PARAM, err, out, out_len, status, stream)
        e[1].record(stream)
        tlc.tlc_decompress(out, n, y, in_len=out_len, in_cap=cap, dev_status=status,
                           stream=stream)
        e[2].record(stream)
        tlc.tlc_decompress_accumulate([out], n, acc, in_lens=out_len, in_caps=[cap],
                                      dev_status=status, stream=stream)
        e[3].record(stream)
    torch.cuda.synchronize()
    tlc.tlc_kernel_timing(False)
    kern2 = tlc.tlc_kernel_timing_read()
    legs = [sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps2)) / steps2 / reps
            for i in range(3)]
    legs = max_over_ranks(legs, device=dev)

    L = int(out_len.item())
    nnz = int(torch.count_nonzero(y).item())
    ms_step = total_ms / args.steps
    in_bytes = 4 * n
    value = world * in_bytes / (ms_step * 1e-3) / 1e9
    peak, peak_kind = load_peaks()

    # bytes each kernel must move: read x and err (8n); read x, err and
    # write err and the stream (12n + L); read the stream and write y
    # (L + 4n); read the stream and read-modify-write acc at non-zeros.
    # On the deferred-placement path (large n) k_quant_zre stages the
    # encoded bytes and k_zre_place writes the stream (L).
    # Large streams get a counting pass over the stream (L) before each
    # decode kernel.
    deferred = pre.get("k_zre_place", (0, 0.0))[0] > 0
    algo = {
        "k_absmax": 8 * n,
        "k_quant_zre": 12 * n + (0 if deferred else L),
        "k_zre_place": L,
        "k_decode_count": L,
        "k_decode_write": L + 4 * n,
        "k_decode_accumulate": L + 8 * nnz,
    }
    kernels = {}
    for name, (launches, ms) in kern2.items():
        if launches == 0:
            continue
        per = ms / launches
        gbs = algo[name] / (per * 1e-3) / 1e9
        kernels[name] = {"launches": launches, "avg_ms": round(per, 5),
                         "algo_bytes_per_launch": algo[name], "achieved_gbs": round(gbs, 1),
                         "frac": round(gbs / peak, 4)}
    dom_gbs = algo[dom] / (dom_ms * 1e-3) / 1e9
    c_ms, d_ms, a_ms = legs
    compress_bytes = algo["k_absmax"] + algo["k_quant_zre"] + (L if deferred else 0)
    decompress_bytes = algo["k_decode_write"]
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": (workload_config(n, args.log2n, args.dense) if args.config == 3 else
                   {"workload": synth.CONFIGS[args.config]["name"], "n": n, "s": S_PARAM,
                    "l2": "L2-resident (x + err = 8 MiB)"}) | {"parallelism": f"replicas x{world}"}
                  | ({"calls": f"CUDA graphs of {reps} whole steps, replayed"}
                     if graphs else {}),
        "clocks": clocks,
        "gpu_launches": int(sum(v[0] for v in kern.values())),
        "roofline": {
            "bound": "hbm",
            "kernel": dom,
            "achieved": round(dom_gbs, 1),
            "peak": peak,
            "peak_source": f"{peak_kind} hbm_gbs",
            "unit": "GB/s",
            "frac": round(dom_gbs / peak, 4),
            "traffic": traffic_for(dom, n),
            "timing": (f"CUDA events around every {dom} launch in the timed region"
                       if not graphs else
                       f"CUDA events around each {dom} launch of a pre-pass (the timed "
                       "region replays CUDA graphs)"),
        },
        "legs": {
            "compress_gbs": round(in_bytes / (c_ms * 1e-3) / 1e9, 1),
            "compress_ms": round(c_ms, 5),
            "compress_hbm_frac": round(compress_bytes / (c_ms * 1e-3) / 1e9 / peak, 4),
            "decompress_gbs": round(in_bytes / (d_ms * 1e-3) / 1e9, 1),
            "decompress_ms": round(d_ms, 5),
            "decompress_hbm_frac": round(decompress_bytes / (d_ms * 1e-3) / 1e9 / peak, 4),
            "accumulate_gbs": round(in_bytes / (a_ms * 1e-3) / 1e9, 1),
            "accumulate_ms": round(a_ms, 5),
            "stream_bytes": L,
            "bits_per_value": round(8 * L / n, 5),
            "nonzero_values": nnz,
        },
        "kernels": kernels,
        "breakdown": (f"legs and kernels: a separate pass of {steps2} steps after the timed "
                      "region, with events between the calls and around every kernel"
                      if not graphs else
                      f"legs: a separate pass of {steps2} replays after the timed region, "
                      f"each leg from its own CUDA graph of {reps} calls, events between the "
                      "replays (per-kernel times are not taken inside graphs)"),
    }

    if not args.no_e2e:
        del xs
        torch.cuda.empty_cache()
        xs_h = [gradient(args, n, 1000 * rank + k) for k in range(2)]
        result["e2e"] = run_e2e(args, tlc, torch, dev, xs_h, n, cap, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args)
    return result


def run_e2e(args, tlc, torch, dev, xs_h, n, cap, world):
    """The step through the public API with host buffers.  Every step copies
    its gradient x in from pinned host memory (two seeded gradients, taken in
    turn), compresses it (the error
    buffer stays on the device: it is the codec's state, like a model's
    weights), decompresses and accumulates, and copies the stream buffer
    (its capacity and the length word) and the decoded y out to pinned host
    memory.  Two buffer sets and three streams (copy-in, compute, copy-out)
    let step i's copy-out overlap step i+1's copy-in; a step's compute waits
    for its own copy-in, and a buffer is refilled only after its last
    reader is done."""
    import torch.distributed as dist

    from gradient_traffic_compression_b200.exchange import max_over_ranks
    xh = [torch.from_numpy(a).pin_memory() for a in xs_h]
    yh = [torch.empty(n, dtype=torch.float32).pin_memory() for _ in range(2)]
    sh = [torch.empty(cap, dtype=torch.uint8).pin_memory() for _ in range(2)]
    lh = [torch.empty(1, dtype=torch.int64).pin_memory() for _ in range(2)]
    xd = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(2)]
    yd = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(2)]
    od = [torch.empty(cap, dtype=torch.uint8, device=dev) for _ in range(2)]
    ld = [torch.zeros(1, dtype=torch.int64, device=dev) for _ in range(2)]
    err = torch.zeros(n, dtype=torch.float32, device=dev)
    acc = torch.zeros(n, dtype=torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    s_c = torch.cuda.current_stream(dev)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b = i % 2
        s_in.wait_event(ev_c[b])            # step i-2 no longer reads xd[b]
        with torch.cuda.stream(s_in):
            xd[b].copy_(xh[i % len(xh)], non_blocking=True)
        ev_in[b].record(s_in)
        s_c.wait_event(ev_in[b])
        s_c.wait_event(ev_out[b])           # step i-2's outputs are out
        tlc.tlc_compress(xd[b], S_PARAM, err, od[b], ld[b], st, s_c)
        tlc.tlc_decompress(od[b], n, yd[b], in_len=ld[b], in_cap=cap, dev_status=st, stream=s_c)
        tlc.tlc_decompress_accumulate([od[b]], n, acc, in_lens=ld[b], in_caps=[cap],
                                      dev_status=st, stream=s_c)
        ev_c[b].record(s_c)
        s_out.wait_event(ev_c[b])
        with torch.cuda.stream(s_out):
            sh[b].copy_(od[b], non_blocking=True)
            lh[b].copy_(ld[b], non_blocking=True)
            yh[b].copy_(yd[b], non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_c)
    s_in.wait_stream(s_c)
    s_out.wait_stream(s_c)
    for i in range(args.e2e_steps):
        step(i)
    s_c.wait_stream(s_in)
    s_c.wait_stream(s_out)
    t1.record(s_c)
    torch.cuda.synchronize()
    ms = max_over_ranks([t0.elapsed_time(t1) / args.e2e_steps], device=dev)[0]
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the e2e run")
    L = int(lh[(args.e2e_steps - 1) % 2].item())
    if L < 4 or L > cap:
        raise RuntimeError(f"e2e stream length {L} out of range")
    return {"value": round(world * 4 * n / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 3), "steps": args.e2e_steps,
            "h2d_bytes_per_step": 4 * n, "d2h_bytes_per_step": cap + 8 + 4 * n,
            "path": "pinned host x -> device; tlc_compress (error buffer resident); "
                    "tlc_decompress; tlc_decompress_accumulate; stream buffer, length and "
                    "y -> pinned host; copy-in, compute and copy-out on three streams, "
                    "two buffer sets"}


# ------------------------------------------- tensor sets and K streams ----

def run_config_set(args, rank, world, local):
    """Configs 2 and 4 (per-layer tensors, one plan call per leg or one call
    per tensor, error buffers carried) and 5 (K = 8 workers' streams summed),
    with a fresh gradient set every step (--grads seeded steps of the
    workload, taken in turn).  Same legs and timing as the headline; extra
    lines, not the headline workload."""
    import torch
    import torch.distributed as dist

    import gradient_traffic_compression_b200 as tlc
    import synth
    from gradient_traffic_compression_b200.exchange import max_over_ranks

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = synth.CONFIGS[args.config]
    s = cfg["s"]
    # A fresh gradient set every step: the workload's steps 0 .. P-1 (each
    # rank its own), resident on the device and taken in turn, while the
    # error buffers carry over from step to step.
    P = max(1, args.grads)
    sets = []
    for k in range(P):
        st_k = 1000 * rank + k
        if args.config == 5:
            xs_h = [synth.flat_tensor(5, step=st_k, worker=w) for w in range(cfg["k"])]
        else:
            xs_h = synth.tensor_set(args.config, st_k)
        sets.append([torch.from_numpy(a).to(dev) for a in xs_h])
        ns = [a.size for a in xs_h]
        del xs_h
    cur = [0]   # the gradient set of the current step
    total = sum(ns)
    errs = [torch.zeros(n, dtype=torch.float32, device=dev) for n in ns]
    caps = [tlc.tlc_compress_bound(n) for n in ns]
    outs = [torch.empty(c, dtype=torch.uint8, device=dev) for c in caps]
    lens = torch.zeros(len(ns), dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    strm = [torch.cuda.current_stream()]   # the stream the legs run on
    stream = strm[0]
    if args.config == 5:
        acc = torch.zeros(ns[0], dtype=torch.float32, device=dev)
        ys, accs = None, None
    else:
        ys = [torch.empty(n, dtype=torch.float32, device=dev) for n in ns]
        accs = [torch.zeros(n, dtype=torch.float32, device=dev) for n in ns]

    use_plan = args.config in (2, 4) and not args.per_tensor
    if use_plan:
        # a plan binds its tensors: one per gradient set, all sharing the
        # error buffers, the outputs and the arena
        plans = [tlc.Plan(xs, errs, ys) for xs in sets]
        arena = torch.empty(plans[0].arena_bytes, dtype=torch.uint8, device=dev)
        acc_plan = tlc.Plan(ys=accs)

    def leg_compress():
        if use_plan:
            plans[cur[0]].compress(s, arena, lens, status, strm[0])
            return
        xs = sets[cur[0]]
        for i in range(len(ns)):
            tlc.tlc_compress(xs[i], s, errs[i], outs[i], lens[i:i + 1], status, strm[0])

    def leg_decompress():
        if use_plan:
            plans[0].decompress(arena, lens, accumulate=False, dev_status=status,
                                stream=strm[0])
        elif args.config != 5:
            for i in range(len(ns)):
                tlc.tlc_decompress(outs[i], ns[i], ys[i], in_len=lens[i:i + 1], in_cap=caps[i],
                                   dev_status=status, stream=strm[0])

    def leg_accumulate():
        if use_plan:
            acc_plan.decompress(arena, lens, accumulate=True, dev_status=status, stream=strm[0])
        elif args.config == 5:
            tlc.tlc_decompress_accumulate(outs, ns[0], acc, in_lens=lens, in_caps=caps,
                                          dev_status=status, stream=strm[0])
        else:
            for i in range(len(ns)):
                tlc.tlc_decompress_accumulate([outs[i]], ns[i], accs[i], in_lens=lens[i:i + 1],
                                              in_caps=[caps[i]], dev_status=status,
                                              stream=strm[0])

    leg_fns = [leg_compress, leg_decompress, leg_accumulate]

    def legs():
        for fn in leg_fns:
            fn()
            yield
        cur[0] = (cur[0] + 1) % P

    for _ in range(max(3, args.warmup)):
        for _ in legs():
            pass
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 50))
    graph = None
    # --graph: `reps` whole steps captured as one CUDA graph (several for a
    # small tensor set, so that the GPU, not the host's launch rate, sets the
    # time), replayed in the timed region; launches counted while captured
    reps = (16 if total < (1 << 24) else 1) if args.graph else 1
    if args.graph:
        reps = -(-reps // P) * P   # whole turns of the gradient sets per replay
    leg_graphs = []
    if args.graph:
        tlc.tlc_kernel_timing_kinds([])
        tlc.tlc_kernel_timing(True)
        graph = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(stream)
        strm[0] = cs
        with torch.cuda.graph(graph, stream=cs):
            for _ in range(reps):
                for _ in legs():
                    pass
        tlc.tlc_kernel_timing(False)
        per_step = {k: (v[0] // reps, v[1]) for k, v in tlc.tlc_kernel_timing_read().items()}
        # one graph of `reps` calls per leg, for the breakdown pass
        for fn in leg_fns:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cs):
                for r in range(reps):
                    cur[0] = r % P
                    fn()
            leg_graphs.append(gr)
        cur[0] = 0
        strm[0] = stream
        graph.replay()
        torch.cuda.synchronize()
        steps = max(reps, steps // reps * reps)
    # timed region: whole steps between two events; launches counted, no
    # per-kernel events
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    tlc.tlc_kernel_timing_kinds([])
    tlc.tlc_kernel_timing(True)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps // reps):
        if graph is not None:
            graph.replay()
        else:
            for _ in legs():
                pass
    t1.record(stream)
    torch.cuda.synchronize()
    tlc.tlc_kernel_timing(False)
    launches = tlc.tlc_kernel_timing_read()
    if graph is not None:
        launches = {k: (v[0] * steps, 0.0) for k, v in per_step.items()}
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    step_ms = max_over_ranks([t0.elapsed_time(t1) / steps], device=dev)[0]
    # breakdown pass: events between the legs and around every kernel
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    tlc.tlc_kernel_timing_kinds(None)
    tlc.tlc_kernel_timing(True)
    for k in range(steps):
        ev[k][0].record(stream)
        if leg_graphs:
            for j, gr in enumerate(leg_graphs):
                gr.replay()
                ev[k][j + 1].record(stream)
            continue
        for j, _ in enumerate(legs()):
            ev[k][j + 1].record(stream)
    torch.cuda.synchronize()
    tlc.tlc_kernel_timing(False)
    kern = tlc.tlc_kernel_timing_read()
    legs_ms = [sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps)) / steps / reps
               for i in range(3)]
    L = int(lens.sum().item())
    in_bytes = 4 * total
    peak, _ = load_peaks()
    res = {
        "metric": METRIC, "value": round(world * in_bytes / (step_ms * 1e-3) / 1e9, 2),
        "unit": "GB/s", "n_gpus": world, "steps": steps, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": cfg["name"], "tensors": len(ns), "values": total, "s": s,
                   "inputs": (f"a fresh gradient set each step: the workload's steps 0..{P - 1}, "
                              "resident on the device and taken in turn, error buffers "
                              "carried"),
                   "calls": ("one plan call per leg (tlc_compress_batch / "
                             "tlc_decompress_batch)" if use_plan else
                             "one C-ABI call per tensor and leg")
                   + (f"; replayed from CUDA graphs of {reps} steps (the breakdown: of "
                      f"{reps} calls of each leg)" if args.graph else "")},
        "legs": {"compress_ms": round(legs_ms[0], 4),
                 "compress_gbs": round(in_bytes / (legs_ms[0] * 1e-3) / 1e9, 1),
                 "stream_bytes": L, "bits_per_value": round(8 * L / total, 5)},
        "per_tensor_us": round(1e3 * step_ms / len(ns), 3),
        "kernels": {k: {"launches": v[0], "avg_ms": round(v[1] / max(v[0], 1), 5)}
                    for k, v in kern.items() if v[0]},
        "gpu_launches": int(sum(v[0] for v in launches.values())),
        "breakdown": ("legs and kernels: a separate pass of the same steps after the timed "
                      "region, with events between the legs and around every kernel"),
    }
    if args.config == 5:
        res["legs"]["accumulate_ms"] = round(legs_ms[2], 4)
        res["legs"]["accumulate_gbs_of_fp32_input"] = round(
            in_bytes / (legs_ms[2] * 1e-3) / 1e9, 1)
        res["legs"]["accumulate_dense_bytes_frac"] = round(
            (8 * ns[0]) / (legs_ms[2] * 1e-3) / 1e9 / peak, 4)
    else:
        res["legs"]["decompress_ms"] = round(legs_ms[1], 4)
        res["legs"]["decompress_gbs"] = round(in_bytes / (legs_ms[1] * 1e-3) / 1e9, 1)
        res["legs"]["accumulate_ms"] = round(legs_ms[2], 4)
    return res


# ------------------------------------------------------ multi-rank exchange --

def run_exchange(args, rank, world, local):
    """The data-parallel exchange step itself (--exchange): every rank
    compresses its own gradient of the headline workload, the compressed
    streams cross the ranks over NCCL, and every rank decodes them.
    allgather: exchange_step (all-gather of the streams, K = world
    decompress-accumulate); sharded: exchange_step_sharded (all-to-all of
    per-shard streams, server-side aggregate and delta compression,
    all-gather of the delta streams, decode).  Timed with CUDA events on
    the step's stream, the maximum over ranks; one JSON line (rank 0)."""
    import torch

    import gradient_traffic_compression_b200 as tlc
    import synth
    from gradient_traffic_compression_b200.exchange import (exchange_step,
                                                            exchange_step_sharded,
                                                            max_over_ranks, shard_bounds)
    dev = torch.device("cuda", local)
    n = 1 << args.log2n
    xs = [torch.from_numpy(synth.flat_tensor(3, n=n, step=1000 * rank + k)).to(dev)
          for k in range(args.grads)]
    err = torch.zeros(n, dtype=torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    if args.exchange == "allgather":
        acc = torch.zeros(n, dtype=torch.float32, device=dev)
    else:
        b = shard_bounds(n, world)
        server_err = torch.zeros(b[rank + 1] - b[rank], dtype=torch.float32, device=dev)
        y = torch.zeros(n, dtype=torch.float32, device=dev)
    turn = [0]
    last = {}

    def step():
        x = xs[turn[0] % len(xs)]
        turn[0] += 1
        if args.exchange == "allgather":
            lens, _ = exchange_step(x, S_PARAM, err, acc, dev_status=st)
            last["widths"] = [lens]
        else:
            up, down = exchange_step_sharded(x, S_PARAM, err, server_err, y, dev_status=st)
            last["widths"] = [up, down]

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    tlc.tlc_kernel_timing_kinds(["k_quant_zre"])
    tlc.tlc_kernel_timing(True)
    import torch.distributed as dist
    dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    tlc.tlc_kernel_timing(False)
    kern = tlc.tlc_kernel_timing_read()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the exchange")
    ms = t0.elapsed_time(t1) / args.steps
    dom = kern.get("k_quant_zre", (0, 0.0))
    dom_ms = dom[1] / max(dom[0], 1)
    ms, dom_ms = max_over_ranks([ms, dom_ms], device=dev)
    widths = [int(t.max().item()) for t in last["widths"]]
    sent = sum((world - 1) * w for w in widths)
    peak, peak_kind = load_peaks()
    dom_gbs = 12 * n / (dom_ms * 1e-3) / 1e9 if dom_ms else None
    return {
        "metric": METRIC, "value": round(world * 4 * n / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(n, args.log2n) | {
            "parallelism": f"data-parallel exchange over {world} rank(s), NCCL",
            "step": ("exchange_step: compress, all-gather of the streams, K = world "
                     "decompress-accumulate" if args.exchange == "allgather" else
                     "exchange_step_sharded: per-shard compress, all-to-all, aggregate, "
                     "delta compress, all-gather, decode")},
        "exchange": {"form": args.exchange, "slot_widths": widths,
                     "stream_bytes_sent_per_rank_per_step": sent,
                     "bits_per_value_on_the_wire": round(8 * sum(widths) / n, 5)},
        "gpu_launches": int(sum(v[0] for v in kern.values())),
        "roofline": {"bound": "hbm", "kernel": "k_quant_zre",
                     "achieved": round(dom_gbs, 1) if dom_gbs else None, "peak": peak,
                     "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": round(dom_gbs / peak, 4) if dom_gbs else None,
                     "traffic": traffic_for("k_quant_zre", n)},
    }


# ------------------------------------------------------- CPU oracle timing --

def oracle_step(oracle, x, n, acc):
    import numpy as np
    rc, st, e = oracle.compress(x, S_PARAM, np.zeros(n, np.float32))
    rc2, y = oracle.decompress(st, n)
    rc3, acc = oracle.decompress_accumulate([st], n, acc)
    if rc or rc2 or rc3:
        raise RuntimeError(f"oracle status {rc}/{rc2}/{rc3}")
    return st.size, acc


def cpu_sweep():
    """The CPU oracle per direction (median of 3 runs each, one core) over
    the config-3 sweep 2^20..2^24 and on configs 1 and 5 (one of config 5's
    streams, which is what one compress and one decompress see)."""
    import numpy as np
    import oracle
    import synth
    cases = [("config 3", 1 << k, 3, 1.9) for k in range(20, 25)]
    cases += [("config 1", synth.CONFIGS[1]["n"], 1, synth.CONFIGS[1]["s"]),
              ("config 5 (one stream)", synth.CONFIGS[5]["n"], 5, synth.CONFIGS[5]["s"])]
    out = []
    for name, n, cfg, s in cases:
        x = synth.flat_tensor(cfg, n=n)
        err = np.zeros(n, np.float32)
        tc, td = [], []
        for _ in range(3):
            t0 = time.perf_counter()
            rc, st, _ = oracle.compress(x, s, err)
            t1 = time.perf_counter()
            rc2, _ = oracle.decompress(st, n)
            t2 = time.perf_counter()
            if rc or rc2:
                raise RuntimeError(f"oracle status {rc}/{rc2}")
            tc.append(t1 - t0)
            td.append(t2 - t1)
        out.append({"workload": name, "n": int(n),
                    "compress_gbs": round(4 * n / statistics.median(tc) / 1e9, 4),
                    "decompress_gbs": round(4 * n / statistics.median(td) / 1e9, 4),
                    "bits_per_value": round(8 * st.size / n, 4)})
    return out


def cpu_baseline(args):
    """The CPU oracle (single-threaded C, as it stands) on a bounded sample of
    the same workload: repeated compress + decompress + accumulate steps."""
    import numpy as np
    import oracle
    import synth
    ns = 1 << args.cpu_baseline_log2n
    x = synth.flat_tensor(3, n=ns)
    acc = np.zeros(ns, np.float32)
    oracle_step(oracle, x, ns, acc)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_step(oracle, x, ns, acc)
        reps += 1
        el = time.perf_counter() - t0
        if el >= args.cpu_baseline_seconds and reps >= 2:
            break
    return {"value": round(4 * ns * reps / el / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "seconds": round(el, 2),
            "sample": f"{reps} steps of the same workload at n = 2^{args.cpu_baseline_log2n} "
                      "(first-step error buffer), compress + decompress + accumulate",
            "cpu": cpu_model()}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip() + f" ({os.cpu_count()} threads visible)"
    except OSError:
        pass
    return None


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import numpy as np
    import oracle
    import synth
    ns = 1 << min(args.log2n, 24)
    x = synth.flat_tensor(3, n=ns)
    acc = np.zeros(ns, np.float32)
    for _ in range(args.warmup):
        oracle_step(oracle, x, ns, acc)
    t0 = time.perf_counter()
    L = 0
    for _ in range(args.steps):
        L, acc = oracle_step(oracle, x, ns, acc)
    el = time.perf_counter() - t0
    ms = el * 1e3 / args.steps
    v = round(4 * ns / (ms * 1e-3) / 1e9, 4)
    n = 1 << args.log2n
    return {
        "impl": "reference",
        "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(n, args.log2n) | {"parallelism": "single CPU core"},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: the same workload at n = 2^{min(args.log2n, 24)} "
                                   "(a bounded sample of the 2^28 tensor's distribution)",
                         "cpu": cpu_model()},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "bits_per_value": round(8 * L / ns, 5),
    } | ({"cpu_sweep": cpu_sweep()} if args.cpu_sweep else {})


# ---------------------------------------------------------------- traffic ---

def traffic_for(kernel, n):
    """DRAM bytes per launch of `kernel` at size n from the committed ncu
    summary (profiles/dram_traffic.txt), scaled by n; None when there is no
    capture for it or the kernel sources changed since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    from gradient_traffic_compression_b200.build import KERNEL_SOURCES, source_digest
    if kernel not in KERNEL_SOURCES:
        return None
    digest = source_digest(kernel)
    with open(path) as f:
        for line in f:
            t = line.split()
            if len(t) == 4 and not line.startswith("#") and t[0] == kernel:
                n_cap, bytes_cap, dig = int(t[1]), float(t[2]), t[3]
                if dig != digest:
                    return None
                return int(bytes_cap * n / n_cap)
    return None


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    grouped = world > 1 or args.exchange is not None
    if grouped:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(29500 + os.getpid() % 1000))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    try:
        if args.exchange is not None:
            res = run_exchange(args, rank, world, local)
        elif args.config in (1, 3):
            res = run_ours(args, rank, world, local)
        else:
            res = run_config_set(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if grouped:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
