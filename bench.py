#!/usr/bin/env python
"""Benchmark of the OAL causal grouped positive-quadratic attention library on B200.

Headline (one JSON line on rank 0):
  value  = causal PREFILL tokens/s on a Qwen2.5-0.5B-shaped layer: B=1, T=4096, 14 query /
           2 key-value heads, d_h = dv = 64, bf16 inputs (seeded synthetic, same recipe as the
           parity tests), chunk 128.  One step = one oal_prefill call = the whole prefill
           hot path (coefficient expansion, chunk-state builder, readout with the intra-chunk
           dense kernel).  Inputs are resident in HBM.  Between steps, outside the timed
           events, a 256 MB buffer is written and another 256 MB read, so each timed step
           starts on a cold L2 (126 MB) holding no dirty lines (--l2-flush write: the write
           alone).
  e2e    = the same metric through the C ABI's host-buffer call (oal_prefill_host) with
           pinned HOST buffers: every step copies q/k/v host->device, runs the prefill and
           copies yhat device->host, the copies of one segment overlapping the kernels of the
           next (checked once to reproduce the device-resident prefill bit for bit).
  decode = autoregressive decode tokens/s: batch 64, 4096-token context prefilled into the
           packed fp32 states, then single-token steps (L2 flushed between steps).
  roofline = the dominant prefill kernel's achieved rate from the library's CUDA-event trace
           (recorded on the launching stream during the timed steps) against the measured
           peak in MEASURED_PEAKS.json; likewise for the decode kernel against HBM.
  cpu_baseline = the fp64 oracle (oracle/, plain C + OpenMP) on this host's cores, on a
           bounded sample of the same workload (rank 0, N=1 only).

Multi-GPU: one process per GPU (torchrun).  Every rank prefills its own replica of the
layer (independent problems, no data-path collective): weak scaling.  Timing is the max over
ranks of the summed per-step device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "OAL causal prefill tokens/s and decode tokens/s on 1 B200; % of roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
F, W = 2145, 65


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--chunk", type=int, default=128)
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch the prefill's scan and readout kernels in plain stream order "
                         "instead of as programmatic dependents")
    ap.add_argument("--l2-flush", default="write+read", choices=["write+read", "write"],
                    help="between timed steps: write a 256 MB buffer, then (default) read "
                         "another 256 MB so that the write's dirty lines are written back "
                         "outside the timed events")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the small timings of the further paths (Hadamard prefill, "
                         "variable-length batch, dense backward)")
    ap.add_argument("--e2e-segments", type=int, default=4,
                    help="segments of the e2e host-buffer prefill (copies overlap kernels)")
    ap.add_argument("--workload", default="config1", choices=["config1", "config3_16k",
                                                              "config3_32k", "config3_64k"],
                    help="prefill workload (config1 is the headline)")
    ap.add_argument("--no-config2", action="store_true",
                    help="skip the batched 18-layer prefill (B=8, T=4096) measurement")
    ap.add_argument("--config2-steps", type=int, default=3,
                    help="timed passes over the 18 layers of the batched prefill")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def profiled_traffic(workload_name, summary="prefill_tc_config1_kernels.md"):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the kernels
    captured with ncu on the bench workload, from the committed profile summary of the
    current kernels (none: null)."""
    if workload_name != "config1":
        return {}
    path = os.path.join(ROOT, "profiles", summary)
    out = {}
    if os.path.exists(path):
        with open(path) as f:
            for ln in f:
                if ln.startswith("traffic_bytes_per_launch:"):
                    for item in ln.split(":", 1)[1].split():
                        name, val = item.split("=")
                        out[name] = int(val)
    return out


def max_over_ranks(ms, world, device):
    """The job's time: the slowest rank's device-timed milliseconds (all ranks call this)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, units_per_rank, ms):
    """Whole-job throughput: every rank processed units_per_rank units in at most ms."""
    return world * units_per_rank / (ms / 1e3)


def dist_setup(gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}")
    return world, rank, local


def workload(name):
    from positive_quadratic_b200 import inputs as I
    if name == "config1":
        return I.config1(), "qwen2.5-0.5b-layer-prefill B=1 T=4096 Hq=14 Hkv=2 d=64 bf16"
    T = {"config3_16k": 16384, "config3_32k": 32768, "config3_64k": 65536}[name]
    return I.config3(T), f"long-context prefill B=1 T={T} Hq=14 Hkv=2 d=64 bf16"


def to_dev(p, dev, torch):
    dt = torch.bfloat16 if p.dtype == "bf16" else torch.float32
    t = lambda a, d=None: torch.from_numpy(np.ascontiguousarray(a)).to(dev, d)  # noqa: E731
    return t(p.q, dt), t(p.k, dt), t(p.v, dt), t(p.group_id), t(p.L), t(p.G)


def prefill_flops(B, T, Hq, Hkv):
    """Algorithmic prefill work: the eq. (4) state update per key/value head plus the eq. (5)
    readout per query head over D = 2145 packed features and dv + 1 = 65 columns."""
    return 2.0 * B * T * F * W * (Hq + Hkv)


def kernel_work(p, chunk=128):
    """Algorithmic work of each kernel of one tensor-core prefill call (bf16, chunk 128):
    name -> (amount, 'flop' | 'byte').
      delta_tc   eq. (4) chunk deltas: 2 F W flop per token and key/value head
      readout_tc eq. (5) over the prefix state: 2 F W flop per query row with an inter-chunk
                 part (every chunk but the first)
      intra_tc   eqs. (2)-(3) inside a chunk: per causal pair (i, j <= i in the same chunk)
                 2 * 64 (G + 1) flop for the G + 1 factored score products and 2 * 65 for
                 kappa [v; 1]
      scan       bytes: fp32 deltas read once, bf16 state images written once (the 65 live
                 rows of 64 per 64 packed rows), the fp32 final state written once"""
    B, Hq, T, _ = p.q.shape
    Hkv = p.k.shape[1]
    NC = -(-T // chunk)
    rows_inter = max(0, T - chunk)
    pairs = 0
    for c in range(NC):
        n = min(chunk, T - c * chunk)
        pairs += n * (n + 1) // 2
    per_pair = sum(2.0 * 64 * (int(g) + 1) + 2.0 * W for g in p.G)  # summed over heads
    slices = 2176 // 64
    return {
        "delta_tc": (2.0 * B * Hkv * T * F * W, "flop"),
        "readout_tc": (2.0 * B * Hq * rows_inter * F * W, "flop"),
        "intra_tc": (B * pairs * per_pair, "flop"),
        "scan": (B * Hkv * (NC * W * 2176 * 4 + (NC - 1) * slices * W * 64 * 2
                            + 2176 * W * 4), "byte"),
    }


def kernel_rooflines(prof, work, pk, pk_kind, n_steps):
    """Per-kernel achieved rate from the library's CUDA-event trace (name -> (launches, ms))
    against the measured peaks: tensor-core kernels against the bf16 peak, the scan against
    HBM copy bandwidth (its data stays in the L2, so it can read above 1), CUDA-core kernels
    against the fp32 ALU peak."""
    out = {}
    total = sum(t for _, t in prof.values()) or 1.0
    for name, (nl, ms) in prof.items():
        per = ms / nl
        amount, kind = work.get(name, (None, None))
        if amount is None:
            alu = 148 * 128 * 2 * pk.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            out[name] = {"bound": "alu", "avg_launch_ms": per, "peak": alu, "unit": "TFLOP/s",
                         "share": t_share(ms, total)}
            continue
        if kind == "flop":
            ach = amount / (per / 1e3) / 1e12
            out[name] = {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                         "algorithmic_per_launch": amount, "avg_launch_ms": per,
                         "share": t_share(ms, total), "peak_kind": pk_kind}
        else:
            ach = amount / (per / 1e3) / 1e9
            out[name] = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "algorithmic_per_launch": amount,
                         "avg_launch_ms": per, "share": t_share(ms, total), "peak_kind": pk_kind}
    return out


def t_share(ms, total):
    return round(ms / total, 4)


def cpu_baseline(p, budget_s=12.0):
    """The fp64 oracle on the full layer, repeated until about budget_s seconds have passed."""
    import oracle
    tokens, t0, runs = 0, time.perf_counter(), 0
    while True:
        oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
        runs += 1
        tokens += p.q.shape[0] * p.q.shape[2]
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": tokens / el, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"fp64 oracle (H0/H1/H2 recurrence, OpenMP) on the full layer "
                      f"B={p.q.shape[0]} T={p.q.shape[2]} Hq={p.q.shape[1]} x{runs} run(s), "
                      f"{el:.1f} s", "seconds": el}


def cpu_baseline_decode(p, steps=16):
    """The fp64 oracle's decode step on this host's cores: batch and heads of `p`, the state
    of a 16-token prefix (a step's cost does not depend on the context length: the state has
    a fixed size), then `steps` single-token steps continuing it."""
    import oracle
    pre = 16
    sl = lambda a, t0, t1: np.ascontiguousarray(a[:, :, t0:t1])  # noqa: E731
    _, st = oracle.recurrent(sl(p.q, 0, pre), sl(p.k, 0, pre), sl(p.v, 0, pre), p.group_id,
                             p.L, p.G, p.eps, return_state=True)
    t0 = time.perf_counter()
    for t in range(pre, pre + steps):
        _, st = oracle.recurrent(sl(p.q, t, t + 1), sl(p.k, t, t + 1), sl(p.v, t, t + 1),
                                 p.group_id, p.L, p.G, p.eps, state=st, return_state=True)
    el = time.perf_counter() - t0
    B = p.q.shape[0]
    return {"value": B * steps / el, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"fp64 oracle recurrence, batch {B}, {steps} single-token steps after a "
                      f"{pre}-token prefix (a step's cost does not depend on the context), "
                      f"{el:.1f} s", "seconds": el}


def cpu_baseline_long(T=16384):
    """The fp64 oracle on one long-context layer (config 3's shape at T), one run."""
    import oracle
    from positive_quadratic_b200 import inputs as I
    p = I.config3(T)
    t0 = time.perf_counter()
    oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    el = time.perf_counter() - t0
    return {"value": T / el, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"fp64 oracle recurrence on the full layer B=1 T={T} Hq=14, one run, "
                      f"{el:.1f} s", "seconds": el}


def run_reference(args):
    """The reference arm: the fp64 oracle timed on this host's cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    p, desc = workload(args.workload)
    sample_T = 512
    s = p.slice_tokens(0, sample_T)
    for _ in range(args.warmup):
        oracle.recurrent(s.q, s.k, s.v, s.group_id, s.L, s.G, s.eps)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.recurrent(s.q, s.k, s.v, s.group_id, s.L, s.G, s.eps)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = args.steps * sample_T * s.q.shape[0] / tot
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "impl": "reference",
           "config": {"workload": desc, "sample": f"first {sample_T} tokens, all heads",
                      "chunk": args.chunk},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(),
                            "kind": "oracle",
                            "sample": f"fp64 oracle recurrence on the first {sample_T} tokens "
                                      f"of the layer (all 14 heads) per step"},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def host_ahead(torch, steps, us_per_step=150.0):
    """A device-side wait of about `steps` x `us_per_step` microseconds on the current stream
    (a spinning kernel, before the first timed event), during which the host queues the timed
    steps: the device then runs them back to back and never idles waiting for a launch."""
    torch.cuda._sleep(int(steps * us_per_step * 1e-6 * 1.9e9))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist
    from positive_quadratic_b200 import oal

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    pk, pk_kind = peaks()
    oal.lib()
    oal.set_prefill_overlap(not args.no_overlap)

    p, desc = workload(args.workload)
    B, Hq, T, _ = p.q.shape
    Hkv = p.k.shape[1]
    q, k, v, g, L, G = to_dev(p, dev, torch)
    out, state = oal.prefill(q, k, v, g, L, G, p.eps, args.chunk)
    ws = oal.empty_workspace(oal.prefill_workspace_bytes(
        oal.make_shape(B, T, Hq, Hkv, args.chunk, oal.OAL_BF16)), dev)
    flush = L2Flush(torch, dev, args.l2_flush == "write+read")
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    def step():
        oal.prefill(q, k, v, g, L, G, p.eps, args.chunk, out=out, state=state, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
        flush()
    torch.cuda.synchronize()
    assert oal.device_error() == 0

    # ---- timed prefill (device-resident inputs) ----
    # pass 1: the value, with nothing but the step between the events
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    n0 = oal.launch_count()
    with ClockSampler(local) as clk:
        # the device waits (outside the timed events) until the host has queued every step, so
        # that no step's events include time the device spent waiting for the host to launch
        host_ahead(torch, args.steps)
        for s0, s1 in evs:
            s0.record(stream)
            step()
            s1.record(stream)
            flush()
        torch.cuda.synchronize()
    n_launch = oal.launch_count() - n0
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    value = job_rate(world, args.steps * B * T, total_ms)
    # pass 2: the same steps with the library's per-kernel CUDA events on the launching
    # streams (they add a few microseconds per step and keep the programmatic-dependent
    # launches from overlapping), for the per-kernel times and the roofline
    evs2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    oal.profile_read()
    oal.profile_enable(True)
    barrier()
    torch.cuda.synchronize()
    for s0, s1 in evs2:
        s0.record(stream)
        step()
        s1.record(stream)
        flush()
    torch.cuda.synchronize()
    barrier()
    oal.profile_enable(False)
    prof = oal.profile_read()
    traced_ms = sum(a.elapsed_time(b) for a, b in evs2) / args.steps

    # roofline of the dominant prefill kernel: the largest share of the four kernels, which run
    # one after another on the caller's stream (deltas, scan, intra-chunk sums, readout; each
    # a programmatic dependent of the one before)
    per_kernel = kernel_rooflines(prof, kernel_work(p, args.chunk), pk, pk_kind, args.steps)
    roof = None
    if per_kernel:
        serial = list(per_kernel)
        name = max(serial, key=lambda n: per_kernel[n]["share"])
        d = per_kernel[name]
        roof = {"bound": d["bound"], "achieved": d.get("achieved"), "peak": d["peak"],
                "unit": d["unit"], "frac": d.get("frac"),
                "traffic": profiled_traffic(args.workload).get(name), "kernel": name,
                "avg_launch_ms": d["avg_launch_ms"],
                "algorithmic_per_launch": d.get("algorithmic_per_launch"),
                "peak_kind": pk_kind,
                "kernel_shares": {n: v["share"] for n, v in per_kernel.items()},
                "serial_kernels": serial,
                "concurrent_kernels": [n for n in per_kernel if n not in serial],
                "kernels": per_kernel,
                "whole_step_frac_of_bf16_peak": prefill_flops(B, T, Hq, Hkv) /
                (total_ms / args.steps / 1e3) / 1e12 / pk["bf16_tflops"],
                "measured_in": "a second timed pass of the same steps with per-kernel events "
                               f"({traced_ms:.4f} ms per step there)"}

    # ---- e2e through the C ABI with pinned host buffers (oal_prefill_host) ----
    e2e = None
    if not args.no_e2e:
        try:
            e2e = run_e2e(args, dev, torch, oal, p, q, k, v, g, L, G, out, B, T, flush,
                          barrier, stream, world)
        except Exception as exc:  # recorded in the line; the device-resident value stands
            e2e = {"error": repr(exc)[:300]}

    # ---- decode ----
    decode = None
    if not args.no_decode:
        decode = run_decode(args, dev, torch, oal, pk, pk_kind, flush, world, barrier)

    config2 = None
    if not args.no_config2:
        try:
            config2 = run_config2(args, dev, torch, oal, pk, pk_kind, flush, world, barrier)
        except Exception as exc:  # recorded in the line; the headline value stands
            config2 = {"error": repr(exc)[:300]}

    extras = None
    if not args.no_extras:
        extras = run_extras(dev, torch, oal, pk)
    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(p)
        try:  # recorded in the line; the headline value stands either way
            from positive_quadratic_b200 import inputs as I
            if isinstance(decode, dict):
                decode["cpu_baseline"] = cpu_baseline_decode(
                    I.config4(batch=64, context=20, steps=0))
            if isinstance(extras, dict) and isinstance(extras.get("config3_long_context"), dict):
                extras["config3_long_context"]["cpu_baseline_T16384"] = cpu_baseline_long(16384)
        except Exception as exc:
            base["extra_error"] = repr(exc)[:300]

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": desc, "chunk": args.chunk,
                           "schedule": "deltas, scan, intra-chunk sums, readout on one stream"
                           + ("" if args.no_overlap else
                              ", each a programmatic dependent launch of the one before"),
                           "l2": flush.describe(),
                           "launch": "the timed steps are queued while the device waits in a "
                                     "spinning kernel before the first timed event",
                           "parallelism": f"replicas x{world}"},
                "roofline": roof, "e2e": e2e, "gpu_launches": int(n_launch),
                "clocks": clk.summary(), "decode": decode, "config2": config2, "extras": extras,
                "cpu_baseline": base,
                "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


class L2Flush:
    """Evicts the 126 MB L2 between timed steps, outside the timed events.  A 256 MB write
    alone leaves the L2 full of its own dirty lines, which the next timed kernel then has to
    write back to HBM on top of its own traffic; the default therefore follows the write with
    a read of a second 256 MB buffer, so the timed kernel starts on a cold L2 holding only
    clean lines (as a profiler's cache flush leaves it)."""

    def __init__(self, torch, dev, clean: bool):
        self.torch, self.clean = torch, clean
        self.wbuf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.rbuf = (torch.zeros((256 << 20) // 4, dtype=torch.float32, device=dev)
                     if clean else None)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.wbuf.zero_()
        if self.clean:
            self.torch.sum(self.rbuf, dim=0, out=self.sink)

    def describe(self) -> str:
        return ("flushed between steps: 256 MB write, then 256 MB read so no dirty lines remain "
                "(outside timed events)" if self.clean else
                "flushed between steps: 256 MB write (outside timed events)")


def run_e2e(args, dev, torch, oal, p, q, k, v, g, L, G, out, B, T, flush, barrier, stream,
            world):
    """The prefill metric through the C ABI's host-buffer call (oal_prefill_host): pinned
    host q/k/v in, fp32 yhat back, copies inside the timed events."""
    hq = q.cpu().pin_memory()
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=torch.float32, pin_memory=True)
    # segments continue the prefix, which only the tensor-core path (chunk 128) does
    nseg = args.e2e_segments if args.chunk == 128 else 1
    bufs = oal.host_prefill_buffers(hq, hk, hv, g, L, G, args.chunk, nseg, device=dev)
    oal.prefill_from_host(hq, hk, hv, p.eps, bufs, hout)
    torch.cuda.synchronize()
    # the segmented call must reproduce the device-resident prefill exactly
    same = bool(torch.equal(hout, out.cpu())) and oal.device_error() == 0
    if not same:
        bufs = oal.host_prefill_buffers(hq, hk, hv, g, L, G, args.chunk, 1, device=dev)
    for _ in range(3):
        oal.prefill_from_host(hq, hk, hv, p.eps, bufs, hout)
        flush()
    evs2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for s0, s1 in evs2:
        s0.record(stream)
        oal.prefill_from_host(hq, hk, hv, p.eps, bufs, hout)
        s1.record(stream)
        flush()
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs2), world, dev)
    # the copies alone, as the call issues them (in on one stream, out on another, both at
    # once): the PCIe bound the end-to-end number is measured against
    dq, dk, dv = (torch.empty_like(t, device=dev) for t in (hq, hk, hv))
    dout = torch.empty(out.shape, dtype=torch.float32, device=dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def copies(which):
        if which in ("in", "both"):
            with torch.cuda.stream(s_in):
                for d_, h_ in ((dq, hq), (dk, hk), (dv, hv)):
                    d_.copy_(h_, non_blocking=True)
        if which in ("out", "both"):
            with torch.cuda.stream(s_out):
                hout.copy_(dout, non_blocking=True)

    copy_ms = {}
    for which in ("in", "out", "both"):
        copies(which)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            copies(which)
        torch.cuda.synchronize()
        copy_ms[which] = (time.perf_counter() - t0) * 1e3 / args.steps
    h2d = int(sum(t.numel() * t.element_size() for t in (hq, hk, hv)))
    d2h = int(hout.numel() * 4)
    e2e = {"value": job_rate(world, args.steps * B * T, e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h,
           "api": "oal_prefill_host",
           "segments": bufs["segments"],
           "segmented_matches_device_prefill": same,
           "ms_per_step": e_ms / args.steps,
           "copies_alone": {
               "what": "the same pinned copies without kernels, in and out on two streams "
                       "(host wall clock per step)",
               "h2d_ms": copy_ms["in"], "d2h_ms": copy_ms["out"], "both_ms": copy_ms["both"],
               "h2d_gbs": h2d / copy_ms["in"] / 1e6, "d2h_gbs": d2h / copy_ms["out"] / 1e6}}
    return e2e


def run_extras(dev, torch, oal, pk):
    """Small timings of the further paths on this rank (no cross-rank reduction): the
    Hadamard-form prefill, variable-length batches (four streams; one launch per kernel),
    long-context prefill with its chunk-size sweep, and the dense and chunked backward.
    Each is timed with CUDA events after warm-up; a failure is recorded, not raised."""
    from positive_quadratic_b200 import inputs as I
    res = {}

    def timed(fn, reps=5):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    def to(a, d=None):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, d)

    try:  # dense O(T^2) form against the linear-time prefill; the contribution statistic
        pc = I.config1()
        q, k, v = (to(x, torch.bfloat16) for x in (pc.q, pc.k, pc.v))
        g, L, G = to(pc.group_id), to(pc.L), to(pc.G)
        pts = {}
        for T in (1024, 4096):
            qq, kk, vv = (x[:, :, :T].contiguous() for x in (q, k, v))
            ms_d = timed(lambda: oal.dense_ref(qq, kk, vv, g, L, G, pc.eps), reps=2)
            ms_l = timed(lambda: oal.prefill(qq, kk, vv, g, L, G, pc.eps, 128))
            pts[f"T{T}"] = {"dense_ms": ms_d, "linear_ms": ms_l}
        res["dense_vs_linear"] = {"workload": "B=1 Hq=14 Hkv=2 bf16 inputs; oal_dense_ref_gpu "
                                              "(O(T^2), CUDA cores, fp32) against oal_prefill "
                                              "(tensor cores, chunk 128)", "points": pts}
        ms = timed(lambda: oal.contribution_stat(q, k))
        res["contribution_stat"] = {"workload": "eq. (1) chi over B=1 T=4096 Hq=14 Hkv=2 bf16",
                                    "ms": ms}
    except Exception as exc:
        res["dense_vs_linear"] = {"error": repr(exc)[:300]}
    try:  # ungrouped Hadamard form, CUDA cores, chunk 64
        p = I.small_layer(901, B=1, T=2048, Hq=14, Hkv=2, dtype="bf16")
        q, k, v = (to(x, torch.bfloat16) for x in (p.q, p.k, p.v))
        a, b, C = (to(x, torch.float32) for x in oracle_free_hadamard_coefs(14))
        ms = timed(lambda: oal.prefill_hadamard(q, k, v, a, b, C, 64))
        res["hadamard_prefill"] = {"workload": "B=1 T=2048 Hq=14 Hkv=2 bf16, chunk 64 "
                                               "(CUDA cores, fp32)",
                                   "ms": ms, "tokens_per_s": 2048 / (ms / 1e3)}
        p = I.small_layer(907, B=1, T=4096, Hq=14, Hkv=2, dtype="bf16")
        q, k, v = (to(x, torch.bfloat16) for x in (p.q, p.k, p.v))
        ms = timed(lambda: oal.prefill_hadamard(q, k, v, a, b, C, 128))
        res["hadamard_prefill_tc"] = {"workload": "B=1 T=4096 Hq=14 Hkv=2 bf16, chunk 128 "
                                                  "(tensor cores; intra-chunk part through the "
                                                  "feature map)",
                                      "ms": ms, "tokens_per_s": 4096 / (ms / 1e3)}
    except Exception as exc:
        res["hadamard_prefill"] = {"error": repr(exc)[:300]}
    try:  # variable-length batch: 16 sequences of 64..2048 tokens over 4 streams
        rng = np.random.default_rng(902)
        lens = [int(x) for x in rng.integers(64, 2049, size=16)]
        base = I.small_layer(903, B=1, T=1, Hq=14, Hkv=2, dtype="bf16")
        g, L, G = to(base.group_id), to(base.L), to(base.G)
        seqs = [I.small_layer(904 + i, B=1, T=t, Hq=14, Hkv=2, dtype="bf16")
                for i, t in enumerate(lens)]
        qs = [to(s.q[0], torch.bfloat16) for s in seqs]
        ks = [to(s.k[0], torch.bfloat16) for s in seqs]
        vs = [to(s.v[0], torch.bfloat16) for s in seqs]
        streams = [torch.cuda.Stream(device=dev) for _ in range(4)]
        ms = timed(lambda: oal.prefill_varlen(qs, ks, vs, g, L, G, base.eps, 128,
                                              streams=streams))
        res["varlen_prefill"] = {"workload": f"16 sequences, {sum(lens)} tokens, 4 streams, "
                                             "Hq=14 Hkv=2 bf16, chunk 128 (includes packing)",
                                 "ms": ms, "tokens_per_s": sum(lens) / (ms / 1e3)}
        # the same batch, packed once, in one launch per kernel
        q, k, v, _ = oal.pack_sequences(qs, ks, vs)
        ms = timed(lambda: oal.prefill_packed(q, k, v, lens, 14, 2, g, L, G, base.eps))
        res["packed_prefill"] = {"workload": f"the same 16 sequences, {sum(lens)} tokens, "
                                             "one launch per kernel (oal_prefill_packed)",
                                 "ms": ms, "tokens_per_s": sum(lens) / (ms / 1e3)}
        # many short sequences: 64 of 64..320 tokens
        lens2 = [int(x) for x in rng.integers(64, 321, size=64)]
        seqs2 = [I.small_layer(950 + i, B=1, T=t, Hq=14, Hkv=2, dtype="bf16")
                 for i, t in enumerate(lens2)]
        qs2 = [to(s_.q[0], torch.bfloat16) for s_ in seqs2]
        ks2 = [to(s_.k[0], torch.bfloat16) for s_ in seqs2]
        vs2 = [to(s_.v[0], torch.bfloat16) for s_ in seqs2]
        ms_v = timed(lambda: oal.prefill_varlen(qs2, ks2, vs2, g, L, G, base.eps, 128,
                                                streams=streams))
        q2, k2, v2, _ = oal.pack_sequences(qs2, ks2, vs2)
        ms_p = timed(lambda: oal.prefill_packed(q2, k2, v2, lens2, 14, 2, g, L, G, base.eps))
        res["short_sequences"] = {"workload": f"64 sequences of 64..320 tokens ({sum(lens2)} "
                                              "tokens), Hq=14 Hkv=2 bf16, chunk 128",
                                  "varlen_4_streams_ms": ms_v, "packed_one_launch_ms": ms_p,
                                  "packed_tokens_per_s": sum(lens2) / (ms_p / 1e3)}
    except Exception as exc:
        res["varlen_prefill"] = {"error": repr(exc)[:300]}
    try:  # long-context prefill (config 3) and its chunk-size sweep
        sweep = {}
        for T, chunks in ((16384, (64, 128, 256)), (32768, (128,)), (65536, (128,))):
            p = I.config3(T)
            q, k, v, g, L, G = to_dev(p, dev, torch)
            out = torch.empty(1, 14, T, 64, dtype=torch.float32, device=dev)
            for C in chunks:
                ws = oal.empty_workspace(oal.prefill_workspace_bytes(
                    oal.make_shape(1, T, 14, 2, C, oal.OAL_BF16)), dev)
                st = oal.prefill(q, k, v, g, L, G, p.eps, C, out=out, workspace=ws)[1]
                ms = timed(lambda: oal.prefill(q, k, v, g, L, G, p.eps, C, out=out, state=st,
                                               workspace=ws), reps=3)
                sweep[f"T{T}_C{C}"] = {
                    "ms": ms, "tokens_per_s": T / (ms / 1e3),
                    "path": "tensor cores (bf16 operands, fp32 accumulation)"
                    if oal.prefill_path(oal.make_shape(1, T, 14, 2, C, oal.OAL_BF16))
                    == oal.OAL_PATH_TENSOR else "CUDA cores (fp32)",
                    "frac_of_bf16_peak": prefill_flops(1, T, 14, 2) / (ms / 1e3) / 1e12
                    / pk["bf16_tflops"]}
                del ws
            del q, k, v, out
        res["config3_long_context"] = {
            "workload": "B=1 Hq=14 Hkv=2 d=64 bf16, chunk swept at T=16384 (64 and 256 run on "
                        "the fp32 CUDA-core path; 128 is the tensor-core tile height)",
            "points": sweep}
    except Exception as exc:
        res["config3_long_context"] = {"error": repr(exc)[:300]}
    try:  # dense backward, reference scale
        p = I.small_layer(905, B=1, T=256, Hq=14, Hkv=2, dtype="bf16")
        q, k, v = (to(x, torch.bfloat16) for x in (p.q, p.k, p.v))
        g, L, G = to(p.group_id), to(p.L), to(p.G)
        dy = torch.randn(1, 14, 256, 64, device=dev)
        ms = timed(lambda: oal.dense_backward(q, k, v, g, L, G, p.eps, dy), reps=3)
        res["dense_backward"] = {"workload": "B=1 T=256 Hq=14 Hkv=2 bf16 (O(T^2) reference)",
                                 "ms": ms}
        pc = I.config1()
        q, k, v = (to(x, torch.bfloat16) for x in (pc.q, pc.k, pc.v))
        g, L, G = to(pc.group_id), to(pc.L), to(pc.G)
        dy = torch.randn(1, 14, 4096, 64, device=dev)
        ws = oal.backward_workspace(q, k, v)
        ms = timed(lambda: oal.backward(q, k, v, g, L, G, pc.eps, dy, workspace=ws), reps=3)
        res["backward"] = {"workload": "B=1 T=4096 Hq=14 Hkv=2 bf16, chunked O(T) gradients "
                                       "(dq, dk, dv, dL, deps) on CUDA cores in fp32, including "
                                       "the fp32 forward it recomputes",
                           "ms": ms, "tokens_per_s": 4096 / (ms / 1e3)}
    except Exception as exc:
        res["dense_backward"] = {"error": repr(exc)[:300]}
    if oal.device_error() != 0:
        res["device_error"] = True
    return res


def oracle_free_hadamard_coefs(Hq, d=64):
    """Seeded Hadamard-form coefficients with a positive kernel: a in [2, 3), small b,
    C = W W^T / d + I/2 (the benchmark's own draw; no oracle involved)."""
    rng = np.random.default_rng(906)
    a = 2.0 + rng.random(Hq)
    b = 0.1 * rng.standard_normal((Hq, d))
    W = rng.standard_normal((Hq, d, d))
    C = W @ W.transpose(0, 2, 1) / d + 0.5 * np.eye(d)
    return a, b, C


def run_config2(args, dev, torch, oal, pk, pk_kind, flush, world, barrier):
    """Batched prefill of the 18 converted layers (3-20) of a Qwen2.5-0.5B-shaped model:
    B=8, T=4096, 14/2 heads, bf16, each layer with its own seeded inputs, groups and L.  One
    pass = one oal_prefill per layer; tokens/s = B*T tokens through all 18 layers per pass.
    Inputs resident in HBM, the L2 flushed between passes (outside the timed events)."""
    from positive_quadratic_b200 import inputs as I
    layers = []
    for l in range(18):
        p = I.config2_layer(l)
        layers.append(to_dev(p, dev, torch) + (p.eps,))
    q0 = layers[0][0]
    B, Hq, T, _ = q0.shape
    Hkv = layers[0][1].shape[1]
    out = torch.empty(B, Hq, T, 64, dtype=torch.float32, device=dev)
    shape = oal.make_shape(B, T, Hq, Hkv, 128, oal.OAL_BF16)
    ws = oal.empty_workspace(oal.prefill_workspace_bytes(shape), dev)
    states = [oal.prefill(*layers[l][:6], layers[l][6], 128, out=out, workspace=ws)[1]
              for l in range(18)]

    def one_pass():
        for l in range(18):
            q, k, v, g, L, G, eps = layers[l]
            oal.prefill(q, k, v, g, L, G, eps, 128, out=out, state=states[l], workspace=ws)

    one_pass()
    flush()
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.config2_steps)]
    barrier()
    torch.cuda.synchronize()
    for s0, s1 in evs:
        s0.record(stream)
        one_pass()
        s1.record(stream)
        flush()
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev)
    # one more pass with per-kernel events, for the kernel shares only
    oal.profile_read()
    oal.profile_enable(True)
    one_pass()
    torch.cuda.synchronize()
    oal.profile_enable(False)
    prof = oal.profile_read()
    flush()
    per_pass = ms / args.config2_steps
    flops = 18 * prefill_flops(B, T, Hq, Hkv)
    total = sum(t for _, t in prof.values()) or 1.0
    return {"value": job_rate(world, args.config2_steps * B * T, ms), "unit": UNIT,
            "ms_per_pass": per_pass, "passes": args.config2_steps,
            "workload": "18 layers, B=8 T=4096 Hq=14 Hkv=2 d=64 bf16, chunk 128; tokens/s "
                        "through all 18 layers",
            "whole_pass_frac_of_bf16_peak": flops / (per_pass / 1e3) / 1e12 / pk["bf16_tflops"],
            "algorithmic_flop_per_pass": flops, "peak_kind": pk_kind,
            "kernel_shares": {n: round(t / total, 4) for n, (c, t) in prof.items()}}


def run_decode(args, dev, torch, oal, pk, pk_kind, flush, world, barrier):
    """batch 64, context 4096 prefilled (untimed), then args.decode_steps single-token steps."""
    from positive_quadratic_b200 import inputs as I
    nsteps = args.decode_steps
    # tokens for the timed steps and for the traced second pass
    p = I.config4(batch=64, context=4096, steps=2 * nsteps)
    B, Hq, Ttot, _ = p.q.shape
    Hkv = p.k.shape[1]
    q, k, v, g, L, G = to_dev(p, dev, torch)
    ctx = 4096
    _, state = oal.prefill(q[:, :, :ctx].contiguous(), k[:, :, :ctx].contiguous(),
                           v[:, :, :ctx].contiguous(), g, L, G, p.eps, args.chunk)
    ws = oal.decode_workspace(B, Hq, Hkv, dev)
    qs = [q[:, :, t:t + 1].contiguous() for t in range(ctx, Ttot)]
    ks = [k[:, :, t:t + 1].contiguous() for t in range(ctx, Ttot)]
    vs = [v[:, :, t:t + 1].contiguous() for t in range(ctx, Ttot)]
    del q, k, v
    out = torch.empty(B, Hq, 1, 64, dtype=torch.float32, device=dev)
    state0 = state.clone()
    stream = torch.cuda.current_stream()
    for i in range(3):  # warm-up on a scratch copy of the state
        oal.decode_step(qs[i], ks[i], vs[i], state0, ws, out=out)
    torch.cuda.synchronize()
    del state0
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(nsteps)]
    barrier()
    torch.cuda.synchronize()
    # the value: the steps as a caller runs them (no per-kernel events, so the finishing
    # kernel of each step overlaps the tail of its main kernel)
    host_ahead(torch, 16)
    for i, (s0, s1) in enumerate(evs):
        s0.record(stream)
        oal.decode_step(qs[i], ks[i], vs[i], state, ws, out=out)
        s1.record(stream)
        flush()
    torch.cuda.synchronize()
    assert oal.device_error() == 0
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev)
    # the roofline: a second pass over further tokens (same shapes) with the library's
    # per-kernel events on
    n2 = len(qs) - nsteps
    oal.profile_read()
    oal.profile_enable(True)
    for i in range(nsteps, nsteps + n2):
        oal.decode_step(qs[i], ks[i], vs[i], state, ws, out=out)
        flush()
    torch.cuda.synchronize()
    oal.profile_enable(False)
    prof = oal.profile_read()
    assert oal.device_error() == 0
    state_bytes = 2.0 * B * Hkv * F * W * 4   # every packed row read and written once
    io_bytes = B * (Hq + 2 * Hkv) * 64 * 2 + B * Hq * 64 * 4
    kname = "decode"
    kern = prof.get(kname)
    roof = None
    if kern:
        per = kern[1] / kern[0]
        gbs = (state_bytes + io_bytes) / (per / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"], "frac_of_8tbs": gbs / 8000.0,
                "traffic": profiled_traffic("config1", "decode_batch64_sections.md").get(kname),
                "kernel": kname, "avg_launch_ms": per, "peak_kind": pk_kind,
                "algorithmic_bytes_per_launch": state_bytes + io_bytes,
                "measured_in": "a second pass of %d steps with per-kernel events" % n2}
        fin = prof.get("decode_finish")
        if fin:
            roof["finish_kernel_ms"] = fin[1] / fin[0]
        # the whole step (both kernels and the gap between them), untraced
        step_gbs = (state_bytes + io_bytes) / (ms / nsteps / 1e3) / 1e9
        roof["whole_step_gbs"] = step_gbs
        roof["whole_step_frac"] = step_gbs / pk["hbm_gbs"]
        roof["whole_step_frac_of_8tbs"] = step_gbs / 8000.0
    return {"value": job_rate(world, B * nsteps, ms), "unit": UNIT,
            "ms_per_token_step": ms / nsteps, "batch": B, "context": 4096, "steps": nsteps,
            "roofline": roof,
            "workload": "decode batch 64, context 4096, Hq=14 Hkv=2 d=64 bf16 q/k/v, fp32 state",
            "kernel": kname}


if __name__ == "__main__":
    main()
