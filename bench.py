"""Benchmark of the looped gated-delta-rule mixer on B200: tokens*loops/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gdn_prefill]
                    [--order delta_first|decay_first]     # per-key workloads: order of the factors
    python bench.py --impl reference ...        # the fp64 CPU oracle, timed on the host

One step = one looped prefill over the workload's whole batch (all T loops, every chunk
step: gates, Gram products, solve, state GEMMs, outputs), through the C ABI, with inputs
already resident in HBM.  Rank 0 prints one JSON line.  With N > 1 (torchrun, one process
per GPU) every rank runs its own replica of the workload: the (loop, batch, head) units are
independent recurrences, so the path shards with no collective (weak scaling); the only
communication is the timing barrier and the max over ranks.

Extra keys: "decode" (one decode step of the decode workload, timed the same way),
"roofline" (dominant kernel against MEASURED_PEAKS.json), "e2e" (same metric with host
buffers and the copies inside the timed region), "cpu_baseline" (the oracle on a bounded
sample), "clocks" (nvidia-smi sampled during the timed region), "gpu_launches".
"""
import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gated_delta_rule_looped_b200 as lt2  # noqa: E402
from gated_delta_rule_looped_b200 import dist as gdist  # noqa: E402
from gated_delta_rule_looped_b200 import inputs  # noqa: E402

# Algorithmic work per token-head (chunk 64, d = 128; scalar gating): three d x d state
# products 6d^2, the four chunk-local products 8*64*d, the 64x64 solve 64^2/3, counted as
# dense multiply-adds (2 flops each); bytes: q, k, v in + o out (bf16) + alpha + beta (fp32).
FLOP_PER_TOKEN_HEAD = {"scalar": 6 * 128 ** 2 + 8 * 64 * 128 + 64 ** 2 // 3,
                       "per_key": 8 * 128 ** 2 + 16 * 64 * 128 + 64 ** 2 // 3}
BYTES_PER_TOKEN_HEAD = {"scalar": 3 * 256 + 256 + 4 + 4, "per_key": 3 * 256 + 256 + 512 + 4}
# Decode: the fp32 state read and written once, q/k/v in and o out (bf16), alpha, beta.
BYTES_PER_DECODE_UNIT = 2 * 128 * 128 * 4 + 4 * 256 + 8

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = [os.path.join(ROOT, "gated_delta_rule_looped_b200", "csrc", f)
                  for f in ("gdr_prefill_tc.cu", "gdr_prefill_kda_tc.cu", "gdr_decode.cu", "sm100_primitives.cuh")]


def kernel_sources(name, csrc=None):
    """The kernel's source file and every local header it includes, directly or not, in a fixed
    order: kernel code that lives in a shared header changes the kernel as much as its own file."""
    csrc = csrc or os.path.join(ROOT, "gated_delta_rule_looped_b200", "csrc")
    seen, todo = [], [name]
    while todo:
        f = todo.pop(0)
        if f in seen or not os.path.exists(os.path.join(csrc, f)):
            continue
        seen.append(f)
        with open(os.path.join(csrc, f)) as fh:
            todo.extend(re.findall(r'^\s*#\s*include\s+"([^"]+)"', fh.read(), re.M))
    return seen


def kernel_source_hash(name, csrc=None):
    csrc = csrc or os.path.join(ROOT, "gated_delta_rule_looped_b200", "csrc")
    h = hashlib.sha256()
    for f in kernel_sources(name, csrc):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel, source, bytes_launch=None, path=None):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source still
    matches the one that was profiled; else None.  When the benchmarked launch moves a different
    number of algorithmic bytes than the captured one (another workload of the same kernel), the
    captured traffic is scaled by that ratio, since a launch's traffic grows with the token-heads
    it processes.  Returns (bytes or None, a note saying how it was obtained or None)."""
    path = path or PROFILE_TRAFFIC
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(source):
        return None, None
    t = e.get("dram_bytes_per_launch_scaled")
    a = e.get("algorithmic_bytes_per_launch")
    if t is None or bytes_launch is None or not a or a == bytes_launch:
        return t, None
    return t * bytes_launch / a, f"scaled from the capture on {e.get('workload')} by algorithmic bytes per launch"


# ---- clocks during the timed region ------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.samples = []
        self.window = None
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            sel = str(device_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", sel], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [s for (ts, s) in self.samples
                if self.window and self.window[0] - 0.05 <= ts <= self.window[1] + 0.15]
        if not rows:
            rows = [s for (_, s) in self.samples]
        if not rows:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---- distributed plumbing (gated_delta_rule_looped_b200.dist) -----------------------------

def dist_setup(n_gpus):
    world, rank, local = gdist.env_ranks()
    torch.cuda.set_device(local if world > 1 else 0)
    gdist.init("nccl", timeout_s=120, device=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    gdist.barrier(world)


def max_over_ranks(x, world):
    return gdist.max_over_ranks(x, world, device="cuda")


# ---- timed regions -----------------------------------------------------------------------

def timed(fn, steps, warmup, world, sampler=None):
    """W untimed steps, then K steps between a barrier + synchronize on both sides; device
    time from CUDA events on the launching stream, max over ranks."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    barrier(world)
    if sampler is not None:
        sampler.mark(w0, w1)
    ms = e0.elapsed_time(e1) / max(steps, 1)
    return max_over_ranks(ms, world)


def gate_of(w, order):
    if w.gate != "per_key":
        return lt2.LT2_GATE_SCALAR
    return lt2.LT2_GATE_PER_KEY_DECAY_FIRST if order == "decay_first" else lt2.LT2_GATE_PER_KEY


def prefill_case(w, device, order="delta_first"):
    x = inputs.make_inputs(w, seed=0, device=device)
    o = torch.empty(x["v"].shape, dtype=torch.bfloat16, device=device)
    S = torch.empty((w.T, w.B, w.H, w.d, w.d), dtype=torch.float32, device=device)
    dims = lt2.make_dims(w.T, w.B, w.H, w.L, w.d, w.d, lt2.LT2_DTYPE_BF16, gate_of(w, order))
    ws_bytes = lt2.lt2_gdr_prefill_workspace_bytes(dims)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device) if ws_bytes else None

    def step():
        st = lt2.lt2_gdr_prefill(dims, x["q"], x["k"], x["v"], x["alpha"], x["beta"], None, o, S,
                                 ws, ws_bytes)
        if st != lt2.LT2_OK:
            raise lt2.Lt2Error(st, "lt2_gdr_prefill")
    return x, o, S, dims, step


def run_e2e(w, x, dims, steps, warmup, world):
    """Same metric through the C ABI with host buffers: every step copies the inputs from
    pinned host memory, runs the prefill and reads o and the final state back."""
    host = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "alpha", "beta")}
    dev = {n: torch.empty_like(x[n]) for n in host}
    o_d = torch.empty(x["v"].shape, dtype=torch.bfloat16, device="cuda")
    S_d = torch.empty((w.T, w.B, w.H, w.d, w.d), dtype=torch.float32, device="cuda")
    o_h = torch.empty(o_d.shape, dtype=o_d.dtype).pin_memory()
    S_h = torch.empty(S_d.shape, dtype=S_d.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()

    def step():
        for n in host:
            dev[n].copy_(host[n], non_blocking=True)
        st = lt2.lt2_gdr_prefill(dims, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"],
                                 None, o_d, S_d, None, 0)
        if st != lt2.LT2_OK:
            raise lt2.Lt2Error(st, "lt2_gdr_prefill")
        o_h.copy_(o_d, non_blocking=True)
        S_h.copy_(S_d, non_blocking=True)
    ms = timed(step, steps, warmup, world)
    return ms, h2d, d2h


def run_decode(world, steps, warmup):
    w = inputs.workload("decode")
    dev = "cuda"
    hist = inputs.decode_history(w, seed=0, device=dev)
    S = torch.empty((w.T, w.B, w.H, w.d, w.d), dtype=torch.float32, device=dev)
    lt2.prefill(hist["q"], hist["k"], hist["v"], hist["alpha"], hist["beta"], per_key=False, S_out=S)
    del hist
    x = inputs.make_decode_step(w, seed=0, step=0, device=dev)
    o = torch.empty(x["v"].shape, dtype=torch.bfloat16, device=dev)
    dims = lt2.make_dims(w.T, w.B, w.H, 1, w.d, w.d, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR)

    def step():
        st = lt2.lt2_gdr_decode(dims, x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, o)
        if st != lt2.LT2_OK:
            raise lt2.Lt2Error(st, "lt2_gdr_decode")
    ms = timed(step, steps, warmup, world)
    units_per_launch = w.B * w.H
    launch_s = ms * 1e-3 / w.T
    return w, ms, units_per_launch, launch_s


# ---- CPU oracle (reported baseline / reference arm) -----------------------------------------

def oracle_sample(w, target_s=15.0, order="delta_first"):
    """Time the fp64 oracle on a bounded sample of workload w's head-units on this host.
    Returns (tokens*loops per second, threads used, description, single-thread figure): the
    last is one head-unit on one thread, extrapolated to tokens*loops/s."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    threads = oracle.threads(cores)
    L = w.L

    def draw(nunits, seed):
        ws = inputs.workload(w.name, T=1, B=1, H=nunits, L=L)
        x = inputs.make_inputs(ws, seed=seed, device="cpu")
        return [x[n].to(torch.float64).numpy() for n in ("q", "k", "v", "alpha", "beta")]
    # calibrate on one unit, then size the sample to ~target_s of wall time
    a = draw(1, 1)
    t0 = time.perf_counter()
    oracle.prefill_sequential(*a, per_key=(w.gate == "per_key"), nthreads=1, order=order)
    t1 = time.perf_counter() - t0
    per_unit_parallel = t1 / threads
    n = max(threads, int(target_s / max(per_unit_parallel, 1e-6)) // threads * threads)
    n = max(1, min(n, w.units, 64))
    threads = min(threads, n)
    a = draw(n, 2)
    t0 = time.perf_counter()
    oracle.prefill_sequential(*a, per_key=(w.gate == "per_key"), nthreads=threads, order=order)
    dt = time.perf_counter() - t0
    tok_loops = n * L / w.H          # a token*loop needs all H heads
    desc = (f"{n} of {w.units} (loop, batch, head) units of {w.name}, L={L}, fp64 sequential "
            f"oracle, OpenMP over units")
    single = {"value": L / w.H / t1, "unit": "tokens*loops/s", "threads": 1,
              "note": "one head-unit on one thread, extrapolated to the workload"}
    return tok_loops / dt, threads, desc, single


def reference_arm(args, world, rank):
    w = inputs.workload(args.workload)
    metric, unit = metric_of(w)
    if rank != 0:
        return
    vals = []
    desc = threads = None
    single = None
    for _ in range(args.warmup):
        oracle_sample(w, target_s=2.0, order=args.order)
    for _ in range(args.steps):
        v, threads, desc, single = oracle_sample(w, target_s=max(2.0, 20.0 / max(args.steps, 1)), order=args.order)
        vals.append(v)
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, args.gpus, args.order),
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": desc, "single_thread": single},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def metric_of(w):
    return f"looped GDR prefill tokens*loops/s ({w.name})", "tokens*loops/s"


def config_of(w, n_gpus, order="delta_first"):
    gate = w.gate if w.gate != "per_key" or order == "delta_first" else "per_key, decay first"
    return {"workload": w.name, "T": w.T, "B": w.B, "H": w.H, "L": w.L, "d_k": w.d, "d_v": w.d,
            "gate": gate, "chunk": 32 if w.gate == "per_key" else 64, "io_dtype": w.dtype,
            "state_dtype": "f32",
            "parallelism": f"replicas x{n_gpus} (independent head-units, no collective)",
            "l2": "inputs larger than L2 (no flush needed)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gdn_prefill",
                    choices=["gdn_prefill", "kda_prefill", "long_gdn"])
    ap.add_argument("--impl", default="lt2", choices=["lt2", "reference"])
    ap.add_argument("--order", default="delta_first", choices=["delta_first", "decay_first"],
                    help="order of the per-key factors (per-key workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        reference_arm(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return

    world, rank, local = dist_setup(args.gpus)
    lt2.lib()
    w = inputs.workload(args.workload)
    metric, unit = metric_of(w)
    peaks, peak_src = load_peaks()

    x, o, S, dims, step = prefill_case(w, "cuda", args.order)
    sampler = ClockSampler(local) if rank == 0 else None
    ms = timed(step, args.steps, args.warmup, world, sampler)
    if lt2.lt2_gdr_last_device_error() != lt2.LT2_OK:
        raise RuntimeError("device-side timeout during the benchmark")
    clocks = sampler.stop() if sampler else None
    tok_loops = w.T * w.B * w.L * world
    value = gdist.whole_job_rate(w.T * w.B * w.L, world, ms)

    gate = w.gate
    units_per_launch = w.B * w.H
    launch_s = ms * 1e-3 / w.T
    flops_launch = units_per_launch * w.L * FLOP_PER_TOKEN_HEAD[gate]
    bytes_launch = units_per_launch * w.L * BYTES_PER_TOKEN_HEAD[gate]
    kernel, source = (("gdr_prefill_tc_kernel", "gdr_prefill_tc.cu") if gate == "scalar"
                      else ("gdr_prefill_kda_tc_kernel", "gdr_prefill_kda_tc.cu"))
    achieved_tf = flops_launch / launch_s / 1e12
    peak_tf = peaks["bf16_tflops"]
    traffic, traffic_note = traffic_for(kernel, source, bytes_launch)
    roofline = {"bound": "tensor", "kernel": kernel, "achieved": achieved_tf, "peak": peak_tf,
                "unit": "TFLOP/s", "frac": achieved_tf / peak_tf,
                "traffic": traffic,
                "peak_source": f"{peak_src} bf16 dense (fp16 operands run at the same rate)",
                "algorithmic_per_launch": {"flop": flops_launch, "bytes": bytes_launch},
                "hbm": {"achieved": bytes_launch / launch_s / 1e9, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": bytes_launch / launch_s / 1e9 / peaks["hbm_gbs"]},
                "launch_time": "step time / T launches (the T loop launches of a step run back "
                               "to back and overlap through programmatic dependent launch)"}
    if traffic_note:
        roofline["traffic_note"] = traffic_note

    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": config_of(w, world, args.order), "roofline": roofline,
            "gpu_launches": args.steps * w.T}
    if clocks:
        line["clocks"] = clocks

    if not args.no_decode:
        wd, dms, dunits, dlaunch_s = run_decode(world, max(10, args.steps // 4), args.warmup)
        dbytes = dunits * BYTES_PER_DECODE_UNIT
        gbs = dbytes / dlaunch_s / 1e9
        line["decode"] = {"metric": "looped GDR decode tokens*loops/s (decode)",
                          "value": wd.T * wd.B * world / (dms * 1e-3), "unit": "tokens*loops/s",
                          "ms_per_step": dms,
                          "config": {"workload": "decode", "T": wd.T, "B": wd.B, "H": wd.H,
                                     "d": wd.d, "state": "fp32, from a 4096-token prefill"},
                          "roofline": {"bound": "hbm", "kernel": "gdr_decode_kernel",
                                       "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                       "frac": gbs / peaks["hbm_gbs"],
                                       "traffic": traffic_for("gdr_decode_kernel", "gdr_decode.cu")[0],
                                       "peak_source": f"{peak_src} HBM copy"}}

    if not args.no_e2e:
        ems, h2d, d2h = run_e2e(w, x, dims, max(3, args.steps // 20), args.warmup, world)
        line["e2e"] = {"value": tok_loops / (ems * 1e-3), "unit": unit, "ms_per_step": ems,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, threads, desc, single = oracle_sample(w, order=args.order)
        line["cpu_baseline"] = {"value": v, "unit": unit, "cores": threads, "kind": "oracle",
                                "sample": desc, "single_thread": single}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
