"""Benchmark of the looped gated-delta-rule mixer on B200: tokens*loops/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long_gdn]
                    [--extras gdn_prefill,kda_prefill,decode | none]
                    [--order delta_first|decay_first]     # per-key workloads: order of the factors
    python bench.py --impl reference ...        # the fp64 CPU oracle, timed on the host

The headline (`metric`, `value`, `ms_per_step`, `config`, `roofline`, `e2e`, `cpu_baseline`) is
the long-context scalar-gated prefill `long_gdn` (T=8, B=1, H=32, L=65536, d=128), the largest
workload that fits one GPU.  One step = one looped prefill over the workload's whole batch (all
T loops, every chunk step: gates, Gram products, solve, state GEMMs, outputs) through the C ABI,
with inputs already resident in HBM.  The other timed workloads ride along as keys of the same
JSON line, each with its own `ms_per_step`, `value`, `roofline`, `cpu_baseline`, `clocks` and
`gpu_launches`: `gdn_prefill` (T4 B4 H16 L8192, scalar gating), `kda_prefill` (T4 B2 H16
L16384, per-key gating), `decode` (one decode token for T4 B256 H16 from a 4096-token state) and
`fused_gdn_prefill` (gdn_prefill through lt2_gdr_prefill_fused with raw inputs, against the same
steps run as separate passes).

With N > 1 (torchrun, one process per GPU) every rank runs its own replica of each workload: the
(loop, batch, head) units are independent recurrences, so the path shards with no collective
(weak scaling); the only communication is the timing barrier and the max over ranks.  Rank 0
prints one JSON line.
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

HEADLINE = "long_gdn"
EXTRAS = ("gdn_prefill", "kda_prefill", "decode", "fused_gdn_prefill", "swa_prefill", "backward_gdn")

# Algorithmic work per token-head (d = 128), counted as dense multiply-adds (2 flops each).
# Scalar gating, 64-token chunks: three d x d state products 6d^2, the four chunk-local
# products 8*64*d, the 64x64 solve 64^2/3.  Per-key gating (e-form): 8d^2 + 16*64*d + 64^2/3.
# Bytes: q, k, v in + o out (bf16) + alpha (fp32 scalar or d_k vector) + beta (fp32).
FLOP_PER_TOKEN_HEAD = {"scalar": 6 * 128 ** 2 + 8 * 64 * 128 + 64 ** 2 // 3,
                       "per_key": 8 * 128 ** 2 + 16 * 64 * 128 + 64 ** 2 // 3}
BYTES_PER_TOKEN_HEAD = {"scalar": 3 * 256 + 256 + 4 + 4, "per_key": 3 * 256 + 256 + 512 + 4}
# Decode: the fp32 state read and written once, q/k/v in and o out (bf16), alpha, beta.
BYTES_PER_DECODE_UNIT = 2 * 128 * 128 * 4 + 4 * 256 + 8

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Public B200 figures, reported beside the measured ones: ~8 TB/s HBM3e, 2.25 PFLOP/s dense
# bf16/fp16.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}

PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")

KERNELS = {"scalar": ("gdr_prefill_tc_kernel", "gdr_prefill_tc.cu"),
           "per_key": ("gdr_prefill_kda_tc_kernel", "gdr_prefill_kda_tc.cu"),
           "decode": ("gdr_decode_kernel", "gdr_decode.cu"),
           "swa": ("swa_prefill_tc_kernel", "swa_prefill_tc.cu")}


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


# ---- clocks during the timed regions ---------------------------------------------------------

class ClockSampler:
    """nvidia-smi sampled every 100 ms for the whole run; each timed region marks its wall-clock
    window, and `summary` reduces the samples that fall inside a set of windows."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.samples = []
        self.windows = {}
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

    def mark(self, name, t0, t1):
        self.windows.setdefault(name, []).append((t0, t1))

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()

    def summary(self, names=None):
        """Median SM clock, max clock and the throttle reasons seen inside the windows of the
        named regions (all regions when `names` is None)."""
        wins = [w for n, ws in self.windows.items() if names is None or n in names for w in ws]
        rows = [s for (ts, s) in self.samples
                if any(a - 0.05 <= ts <= b + 0.15 for a, b in wins)]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(self.REASONS, r[5:9]):
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

def timed(fn, steps, warmup, world, sampler=None, name="step"):
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
        sampler.mark(name, w0, w1)
    ms = e0.elapsed_time(e1) / max(steps, 1)
    return max_over_ranks(ms, world)


def check_device_status(where):
    st = lt2.lt2_gdr_last_device_error()
    if st != lt2.LT2_OK:
        raise RuntimeError(f"{lt2.lt2_status_string(st)} reported by the device during {where}")


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


def prefill_launches(w):
    """Kernel launches of one prefill step of workload w.  The scalar tensor-core kernel (bf16,
    d = 128) runs every loop in one balanced launch when the units outnumber the SMs and the call
    passes its workspace and S_out, as this benchmark does, and when each CTA's share of the chunks
    touches at most 8 units; otherwise one launch per loop (the library takes the same decision)."""
    if w.gate != "scalar" or w.dtype != "bf16" or w.d != 128:
        return w.T
    units = w.T * w.B * w.H
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    nch = -(-w.L // 64)
    per_cta = -(-units * nch // sms)
    return 1 if units > sms and per_cta <= 6 * nch else w.T


def tensor_roofline(gate, units_per_launch, L, launch_s, peaks, peak_src, launch_note=None):
    """The prefill kernel of one loop launch against the tensor and HBM peaks (measured, and the
    public B200 figures beside them)."""
    kernel, source = KERNELS[gate]
    flops_launch = units_per_launch * L * FLOP_PER_TOKEN_HEAD[gate]
    bytes_launch = units_per_launch * L * BYTES_PER_TOKEN_HEAD[gate]
    achieved_tf = flops_launch / launch_s / 1e12
    achieved_gbs = bytes_launch / launch_s / 1e9
    traffic, traffic_note = traffic_for(kernel, source, bytes_launch)
    r = {"bound": "tensor", "kernel": kernel, "achieved": achieved_tf, "peak": peaks["bf16_tflops"],
         "unit": "TFLOP/s", "frac": achieved_tf / peaks["bf16_tflops"], "traffic": traffic,
         "peak_source": f"{peak_src} bf16 dense burst (fp16 operands run at the same rate)",
         "nominal": {"peak": NOMINAL_PEAKS["bf16_tflops"],
                     "frac": achieved_tf / NOMINAL_PEAKS["bf16_tflops"]},
         "algorithmic_per_launch": {"flop": flops_launch, "bytes": bytes_launch},
         "hbm": {"achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": achieved_gbs / peaks["hbm_gbs"],
                 "nominal": {"peak": NOMINAL_PEAKS["hbm_gbs"],
                             "frac": achieved_gbs / NOMINAL_PEAKS["hbm_gbs"]}},
         "launch_time": launch_note or ("step time / T launches (the T loop launches of a step run back "
                                        "to back and overlap through programmatic dependent launch)")}
    if traffic_note:
        r["traffic_note"] = traffic_note
    return r


def run_prefill(w, args, world, sampler, peaks, peak_src, keep=False):
    """Time workload w's looped prefill.  Returns (entry dict, the case when `keep`)."""
    case = prefill_case(w, "cuda", args.order)
    step = case[-1]
    ms = timed(step, args.steps, args.warmup, world, sampler, w.name)
    check_device_status(w.name)
    nl = prefill_launches(w)
    launch_s = ms * 1e-3 / nl
    note = ("step time: one balanced launch runs every loop (one CTA per SM, an equal share of all "
            "units' chunks each)") if nl == 1 else None
    entry = {"metric": metric_of(w)[0], "value": gdist.whole_job_rate(w.T * w.B * w.L, world, ms),
             "unit": "tokens*loops/s", "ms_per_step": ms, "steps": args.steps,
             "config": config_of(w, world, args.order),
             "roofline": tensor_roofline(w.gate, w.T * w.B * w.H // nl, w.L, launch_s, peaks, peak_src, note),
             "gpu_launches": args.steps * nl}
    if sampler is not None:
        entry["clocks"] = sampler.summary([w.name])
    if keep:
        return entry, case
    del case
    torch.cuda.empty_cache()
    return entry, None


# The fused prologue and output gate (lt2_gdr_prefill_fused), per token-head: the step reads raw
# q, k, v (bf16), the gate logits a, b (fp32) and the output gate logits z (bf16) and writes o
# (bf16).  Run as separate passes around the plain mixer, the same steps move: q, k read and
# written back normalised (4 x 256), a, b read and alpha, beta written (4 x 4), the mixer's own
# bytes, and o, z read and o written back gated (3 x 256).
FUSED_BYTES_PER_TOKEN_HEAD = 3 * 256 + 4 + 4 + 256 + 256
UNFUSED_BYTES_PER_TOKEN_HEAD = 4 * 256 + 4 * 4 + BYTES_PER_TOKEN_HEAD["scalar"] + 3 * 256


def run_fused(args, world, sampler, peaks, peak_src, alpha_scale=0.1):
    """The gdn_prefill workload through lt2_gdr_prefill_fused with raw inputs (every fused step),
    against the same steps as separate passes around the plain call (torch elementwise ops for
    the prologue and the gate, the library's plain prefill for the mixer)."""
    w = inputs.workload("gdn_prefill")
    r = inputs.make_raw_inputs(w, seed=0, device="cuda")
    o = torch.empty(r["v"].shape, dtype=torch.bfloat16, device="cuda")
    S = torch.empty((w.T, w.B, w.H, w.d, w.d), dtype=torch.float32, device="cuda")

    def fused():
        lt2.prefill(r["q"], r["k"], r["v"], r["a"], r["b"], per_key=False, o=o, S_out=S, qk_l2norm=True,
                    gate_logits=True, alpha_scale=alpha_scale, z=r["z"])

    def unfused():
        qn = (r["q"].float() * torch.rsqrt((r["q"].float() ** 2).sum(-1, keepdim=True).clamp_min(1e-24))).to(torch.bfloat16)
        kn = (r["k"].float() * torch.rsqrt((r["k"].float() ** 2).sum(-1, keepdim=True).clamp_min(1e-24))).to(torch.bfloat16)
        al = torch.exp(-torch.nn.functional.softplus(r["a"]) * alpha_scale)
        be = torch.sigmoid(r["b"])
        lt2.prefill(qn, kn, r["v"], al, be, per_key=False, o=o, S_out=S)
        o.copy_((o.float() * torch.sigmoid(r["z"].float())).to(torch.bfloat16))
    ms = timed(fused, args.steps, args.warmup, world, sampler, "fused_gdn_prefill")
    check_device_status("fused_gdn_prefill")
    ms_unfused = timed(unfused, max(3, args.steps // 4), args.warmup, world)
    tokheads = w.T * w.B * w.H * w.L
    entry = {"metric": "looped GDR prefill tokens*loops/s, fused prologue and output gate (gdn_prefill)",
             "value": gdist.whole_job_rate(w.T * w.B * w.L, world, ms), "unit": "tokens*loops/s",
             "ms_per_step": ms, "steps": args.steps,
             "config": dict(config_of(w, world), fused="q/k L2 norm, alpha/beta from logits, sigmoid output gate",
                            alpha_scale=alpha_scale),
             "bytes_per_token_head": {"fused": FUSED_BYTES_PER_TOKEN_HEAD,
                                      "unfused_passes": UNFUSED_BYTES_PER_TOKEN_HEAD},
             "hbm": {"achieved": tokheads * FUSED_BYTES_PER_TOKEN_HEAD / (ms * 1e-3) / 1e9,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": tokheads * FUSED_BYTES_PER_TOKEN_HEAD / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "peak_source": f"{peak_src} HBM copy"},
             "unfused_passes": {"ms_per_step": ms_unfused,
                                "note": "the same steps as separate passes: torch elementwise prologue and "
                                        "output gate around the library's plain prefill"},
             "gpu_launches": args.steps * prefill_launches(w)}
    if sampler is not None:
        entry["clocks"] = sampler.summary(["fused_gdn_prefill"])
    del r, o, S
    torch.cuda.empty_cache()
    return entry


def swa_pairs(L, window):
    """(query, key) pairs inside the windows of one unit: sum over t of min(t + 1, w)."""
    w = min(window, L)
    return w * (w + 1) // 2 + (L - w) * w


def run_swa(args, world, sampler, peaks, peak_src):
    """The sliding-window mixer (lt2_swa_prefill) on the swa_prefill workload, all T loops in one
    launch.  Algorithmic work: 4 d flops per (query, key) pair inside a window (q.k and p v, 2 d
    each); bytes: q, k, v read and o written once (4 x 256 per token-head, bf16)."""
    w = inputs.swa_workload("swa_prefill")
    x = inputs.make_swa_inputs(w, seed=0, device="cuda")
    o = torch.empty_like(x["q"])
    dims = lt2.lt2_swa_dims(w.T, w.B, w.H, w.L, w.d, w.window, 0.0, lt2.LT2_DTYPE_BF16, lt2.LT2_ALGO_AUTO,
                            lt2.LT2_OUT_SAME)

    def step():
        st = lt2.lt2_swa_prefill(dims, x["q"], x["k"], x["v"], o)
        if st != lt2.LT2_OK:
            raise lt2.Lt2Error(st, "lt2_swa_prefill")
    ms = timed(step, args.steps, args.warmup, world, sampler, "swa_prefill")
    check_device_status("swa_prefill")
    launch_s = ms * 1e-3
    flops = w.units * swa_pairs(w.L, w.window) * 4 * w.d
    nbytes = w.units * w.L * 4 * 2 * w.d
    kernel, source = KERNELS["swa"]
    traffic, traffic_note = traffic_for(kernel, source, nbytes)
    tf = flops / launch_s / 1e12
    gbs = nbytes / launch_s / 1e9
    roof = {"bound": "tensor", "kernel": kernel, "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tf / peaks["bf16_tflops"], "traffic": traffic,
            "peak_source": f"{peak_src} bf16 dense burst",
            "nominal": {"peak": NOMINAL_PEAKS["bf16_tflops"], "frac": tf / NOMINAL_PEAKS["bf16_tflops"]},
            "algorithmic_per_launch": {"flop": flops, "bytes": nbytes,
                                       "note": "4 d flops per (query, key) pair inside a window; the "
                                               "kernel also multiplies the masked part of its 64-key "
                                               "blocks, not counted"},
            "hbm": {"achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"]}}
    if traffic_note:
        roof["traffic_note"] = traffic_note
    entry = {"metric": "looped sliding-window attention prefill tokens*loops/s (swa_prefill)",
             "value": gdist.whole_job_rate(w.T * w.B * w.L, world, ms), "unit": "tokens*loops/s",
             "ms_per_step": ms, "steps": args.steps,
             "config": {"workload": w.name, "T": w.T, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "window": w.window,
                        "io_dtype": w.dtype, "scale": "1/sqrt(d)",
                        "parallelism": f"replicas x{world} (independent units, no collective)",
                        "l2": "inputs larger than L2 (no flush needed)"},
             "roofline": roof, "gpu_launches": args.steps}
    if sampler is not None:
        entry["clocks"] = sampler.summary(["swa_prefill"])
    del x, o
    torch.cuda.empty_cache()
    return entry


# Backward pass, per token-head (d_k = d_v = d): the gradient step reads S_{t-1} and S_t and does
# about 20 d^2 flops (G += q dO^T, dq = S dO, three column sums, the dk and dalpha row sums, the
# update of G), and the states it needs cost one forward step, 4 d^2, to recompute.
BW_FLOP_PER_TOKEN_HEAD = 24 * 128 * 128
# Its algorithmic bytes per token-head: q, k, v and dO in bf16, alpha and beta, and the fp32
# gradients dq, dk, dv, dalpha and dbeta (the checkpoints and recomputed states of the workspace
# are the design's, not the problem's).
BW_BYTES_PER_TOKEN_HEAD = 4 * 128 * 2 + 2 * 4 + 3 * 128 * 4 + 2 * 4
# fp32 CUDA-core peak of the part: 148 SMs x 128 fp32 lanes x 2 flops (FMA) x 1.965 GHz
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_backward(args, world, sampler):
    """The backward pass (lt2_gdr_backward, CUDA cores, fp32) on gdn_prefill's shape: gradients of
    every input for upstream gradients of o and of the final state, workspace preallocated."""
    w = inputs.workload("gdn_prefill")
    x = inputs.make_inputs(w, seed=0, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    dO = torch.randn(x["v"].shape, generator=g, device="cuda").to(torch.bfloat16)
    dSL = torch.randn((w.T, w.B, w.H, w.d, w.d), generator=g, device="cuda")
    dims = lt2.make_dims(w.T, w.B, w.H, w.L, w.d, w.d, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR)
    f32 = dict(dtype=torch.float32, device="cuda")
    out = [torch.empty(x["q"].shape, **f32), torch.empty(x["q"].shape, **f32), torch.empty(x["v"].shape, **f32),
           torch.empty(x["alpha"].shape, **f32), torch.empty(x["beta"].shape, **f32), torch.empty(dSL.shape, **f32)]
    ws_bytes = lt2.lt2_gdr_backward_workspace_bytes(dims)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")

    def step():
        st = lt2.lt2_gdr_backward(dims, x["q"], x["k"], x["v"], x["alpha"], x["beta"], None, dO, dSL, *out, ws,
                                  ws_bytes)
        if st != lt2.LT2_OK:
            raise lt2.Lt2Error(st, "lt2_gdr_backward")
    steps = max(3, min(args.steps, 5))
    ms = timed(step, steps, args.warmup, world, sampler, "backward_gdn")
    check_device_status("backward_gdn")
    tokheads = w.T * w.B * w.H * w.L
    tf = tokheads * BW_FLOP_PER_TOKEN_HEAD / (ms * 1e-3) / 1e12
    kernel, source = "gdr_backward_kernel", "gdr_backward.cu"
    traffic, traffic_note = traffic_for(kernel, source, tokheads * BW_BYTES_PER_TOKEN_HEAD)
    entry = {"metric": "looped GDR backward tokens*loops/s (gdn_prefill shape)",
             "value": gdist.whole_job_rate(w.T * w.B * w.L, world, ms), "unit": "tokens*loops/s",
             "ms_per_step": ms, "steps": steps,
             "config": dict(config_of(w, world), **{"pass": "backward", "workspace_bytes": ws_bytes}),
             "roofline": {"bound": "alu", "kernel": kernel, "achieved": tf,
                          "peak": FP32_ALU_PEAK_TFLOPS, "unit": "TFLOP/s", "frac": tf / FP32_ALU_PEAK_TFLOPS,
                          "traffic": traffic,
                          "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz",
                          "algorithmic_per_launch": {"flop": tokheads * BW_FLOP_PER_TOKEN_HEAD,
                                                     "bytes": tokheads * BW_BYTES_PER_TOKEN_HEAD,
                                                     "note": "24 d^2 flops per token-head: the gradient step "
                                                             "and one recomputed forward step; bytes: inputs "
                                                             "and gradients, the workspace's states not counted"}},
             "gpu_launches": steps * 5}
    if traffic_note:
        entry["roofline"]["traffic_note"] = traffic_note + "; the workspace's per-token states are most of it"
    if sampler is not None:
        entry["clocks"] = sampler.summary(["backward_gdn"])
    del x, out, ws, dO, dSL
    torch.cuda.empty_cache()
    return entry


def oracle_backward_sample(target_s=4.0):
    """Time the fp64 backward oracle on this host (one thread): one head-unit of gdn_prefill's
    shape, a prefix of its tokens growing until about `target_s` has passed."""
    from oracle import backward as obw
    w = inputs.workload("gdn_prefill")
    L = 64
    while True:
        ws = inputs.workload("gdn_prefill", T=1, B=1, H=1, L=L)
        x = {n: t.to(torch.float64).numpy() for n, t in inputs.make_inputs(ws, seed=1).items() if t is not None
             and n != "subset"}
        dO = np.random.default_rng(0).normal(size=x["v"].shape)
        t0 = time.perf_counter()
        obw.backward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], dO)
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or L >= w.L:
            break
        L *= 2
    desc = f"one (loop, batch, head) unit of gdn_prefill's shape, the first {L} tokens, fp64 backward oracle"
    return L / dt / w.H, 1, desc


def oracle_swa_sample(target_s=5.0):
    """Time the fp64 oracle of the sliding-window mixer on this host (one thread): one whole unit
    of swa_prefill, repeated until about `target_s` has passed."""
    from oracle import swa as oswa
    w = inputs.swa_workload("swa_prefill")
    ws = inputs.swa_workload("swa_prefill", T=1, B=1, H=1)
    x = {n: t.to(torch.float64).numpy()[0, 0, 0] for n, t in inputs.make_swa_inputs(ws, seed=1).items()}
    rows, reps, L = 0, 0, w.L
    t0 = time.perf_counter()
    while True:
        oswa.prefill(x["q"][:L], x["k"][:L], x["v"][:L], w.window)
        rows += L
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or reps >= 100:
            break
    desc = (f"one (loop, batch, head) unit of swa_prefill, all {L} tokens, {reps} times; fp64 oracle, "
            f"one query at a time")
    return rows / dt / w.H, 1, desc


def run_e2e(w, x, dims, steps, warmup, world):
    """Same metric with host buffers, through the library's host-buffer call (``prefill_host``:
    the C ABI per loop, the loops' copies in and out overlapped with the calls): every step copies
    the inputs from pinned host memory, runs the prefill and writes o and the final state back to
    pinned host memory."""
    names = ("q", "k", "v", "alpha", "beta")
    host = {}
    for n in names:
        host[n] = torch.empty(x[n].shape, dtype=x[n].dtype, pin_memory=True)
        host[n].copy_(x[n])
    o_h = torch.empty(x["v"].shape, dtype=torch.bfloat16, pin_memory=True)
    S_h = torch.empty((w.T, w.B, w.H, w.d, w.d), dtype=torch.float32, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()

    per_key = dims.gate != lt2.LT2_GATE_SCALAR
    order = "decay_first" if dims.gate == lt2.LT2_GATE_PER_KEY_DECAY_FIRST else "delta_first"

    def step():
        lt2.prefill_host(host["q"], host["k"], host["v"], host["alpha"], host["beta"], o_h, S_h,
                         per_key=per_key, order=order)
    ms = timed(step, steps, warmup, world)
    return ms, h2d, d2h


def run_decode(args, world, sampler, peaks, peak_src):
    """One decode step of the decode workload (T4 B256 H16) from the state a 4096-token prefill
    leaves; the state is updated in place, step after step."""
    w = inputs.workload("decode")
    dev = "cuda"
    hist = inputs.decode_history(w, seed=0, device=dev)
    S = torch.empty((w.T, w.B, w.H, w.d, w.d), dtype=torch.float32, device=dev)
    lt2.prefill(hist["q"], hist["k"], hist["v"], hist["alpha"], hist["beta"], per_key=False, S_out=S)
    del hist
    torch.cuda.empty_cache()
    x = inputs.make_decode_step(w, seed=0, step=0, device=dev)
    o = torch.empty(x["v"].shape, dtype=torch.bfloat16, device=dev)
    dims = lt2.make_dims(w.T, w.B, w.H, 1, w.d, w.d, lt2.LT2_DTYPE_BF16, lt2.LT2_GATE_SCALAR)
    S_host = S[0, 0, :8].to("cpu")      # a few units' state for the CPU baseline

    def step():
        st = lt2.lt2_gdr_decode(dims, x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, o)
        if st != lt2.LT2_OK:
            raise lt2.Lt2Error(st, "lt2_gdr_decode")
    nsteps = max(10, args.steps)
    ms = timed(step, nsteps, args.warmup, world, sampler, "decode")
    check_device_status("decode")
    units_per_launch = w.B * w.H
    launch_s = ms * 1e-3 / w.T
    dbytes = units_per_launch * BYTES_PER_DECODE_UNIT
    gbs = dbytes / launch_s / 1e9
    kernel, source = KERNELS["decode"]
    entry = {"metric": "looped GDR decode tokens*loops/s (decode)",
             "value": w.T * w.B * world / (ms * 1e-3), "unit": "tokens*loops/s",
             "ms_per_step": ms, "steps": nsteps,
             "config": {"workload": "decode", "T": w.T, "B": w.B, "H": w.H, "d_k": w.d, "d_v": w.d,
                        "gate": "scalar", "io_dtype": "bf16", "state_dtype": "f32",
                        "state": "fp32, from a 4096-token prefill, updated in place each step",
                        "l2": "1 GiB state read and written per step (larger than L2)"},
             "roofline": {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": peaks["hbm_gbs"],
                          "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                          "traffic": traffic_for(kernel, source)[0],
                          "peak_source": f"{peak_src} HBM copy",
                          "nominal": {"peak": NOMINAL_PEAKS["hbm_gbs"],
                                      "frac": gbs / NOMINAL_PEAKS["hbm_gbs"]},
                          "algorithmic_per_launch": {"bytes": dbytes}},
             "gpu_launches": nsteps * w.T}
    if sampler is not None:
        entry["clocks"] = sampler.summary(["decode"])
    xs = {n: x[n][0, 0, :8].to("cpu") for n in ("q", "k", "v", "alpha", "beta")}
    del S, x, o
    torch.cuda.empty_cache()
    return entry, (w, xs, S_host)


# ---- CPU oracle (reported baseline / reference arm) -----------------------------------------

def oracle_sample(w, target_s=8.0, order="delta_first"):
    """Time the fp64 oracle on a bounded sample of workload w on this host: a calibration on
    one head-unit (one thread, a prefix of at most 1024 tokens) sizes a sample of whole or
    leading-prefix head-units, one per thread, to about `target_s` of wall time.  Returns
    (tokens*loops per second, threads used, description, single-thread figure): the last is
    the calibration, one head-unit on one thread, extrapolated to tokens*loops/s."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    threads = oracle.threads(cores)
    per_key = w.gate == "per_key"

    def draw(nunits, L, seed):
        ws = inputs.workload(w.name, T=1, B=1, H=nunits, L=L)
        x = inputs.make_inputs(ws, seed=seed, device="cpu")
        return [x[n].to(torch.float64).numpy() for n in ("q", "k", "v", "alpha", "beta")]
    L_cal = min(w.L, 1024)
    a = draw(1, L_cal, 1)
    t0 = time.perf_counter()
    oracle.prefill_sequential(*a, per_key=per_key, nthreads=1, order=order)
    per_token = (time.perf_counter() - t0) / L_cal
    L = int(min(w.L, max(64, target_s / max(per_token, 1e-9))))
    n = min(threads, w.units)
    if L == w.L:
        # whole sequences fit: as many rounds of `threads` units as the target allows
        rounds = max(1, int(target_s / max(per_token * w.L, 1e-9)))
        n = min(w.units, 64, threads * rounds)
    threads = min(threads, n)
    a = draw(n, L, 2)
    t0 = time.perf_counter()
    oracle.prefill_sequential(*a, per_key=per_key, nthreads=threads, order=order)
    dt = time.perf_counter() - t0
    tok_loops = n * L / w.H          # a token*loop needs all H heads
    span = f"all {w.L} tokens" if L == w.L else f"the first {L} of {w.L} tokens"
    desc = (f"{n} of {w.units} (loop, batch, head) units of {w.name}, {span} each, fp64 "
            f"sequential oracle, OpenMP over units")
    single = {"value": 1.0 / (per_token * w.H), "unit": "tokens*loops/s", "threads": 1,
              "note": f"one head-unit of {L_cal} tokens on one thread, extrapolated to the workload"}
    return tok_loops / dt, threads, desc, single


def oracle_decode_sample(w, xs, S_host, target_s=4.0):
    """Time the fp64 oracle's decode step on this host: the first units of the decode workload
    (their q, k, v, alpha, beta and prefilled state), repeated to about `target_s`."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    threads = oracle.threads(cores)
    f64 = {n: t.to(torch.float64).numpy() for n, t in xs.items()}
    S = S_host.to(torch.float64).numpy()
    n = S.shape[0]
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.decode_step(f64["q"], f64["k"], f64["v"], f64["alpha"], f64["beta"], S,
                           nthreads=min(threads, n))
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or reps >= 100000:
            break
    units_per_s = reps * n / dt
    desc = (f"decode step of {n} of {w.units} head-units (their prefilled fp32 state), repeated "
            f"{reps} times, fp64 oracle")
    return units_per_s / w.H, min(threads, n), desc


def cpu_entry(w, order, target_s):
    v, threads, desc, single = oracle_sample(w, target_s=target_s, order=order)
    return {"value": v, "unit": "tokens*loops/s", "cores": threads, "kind": "oracle",
            "sample": desc, "single_thread": single}


def reference_arm(args, world, rank):
    """The oracle, as it stands, timed on the host cores on the headline workload: each step a
    bounded sample sized so that the whole --steps/--warmup run ends within a few minutes."""
    w = inputs.workload(args.workload)
    metric, unit = metric_of(w)
    if rank != 0:
        return
    per_step = min(8.0, max(1.0, 150.0 / max(args.steps + args.warmup, 1)))
    vals = []
    desc = threads = single = None
    for _ in range(args.warmup):
        oracle_sample(w, target_s=min(per_step, 2.0), order=args.order)
    for _ in range(args.steps):
        v, threads, desc, single = oracle_sample(w, target_s=per_step, order=args.order)
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
    c = {"workload": w.name, "T": w.T, "B": w.B, "H": w.H, "L": w.L, "d_k": w.d, "d_v": w.d,
         "gate": gate, "chunk": 32 if w.gate == "per_key" else 64, "io_dtype": w.dtype,
         "state_dtype": "f32",
         "parallelism": f"replicas x{n_gpus} (independent head-units, no collective)",
         "l2": "inputs larger than L2 (no flush needed)"}
    if w.overwrite_frac:
        c["overwrites"] = f"alpha = beta = 1 on {w.overwrite_frac:.0%} of the positions"
    return c


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE,
                    choices=["gdn_prefill", "kda_prefill", "long_gdn"],
                    help="headline workload")
    ap.add_argument("--extras", default=",".join(EXTRAS),
                    help="comma-separated workloads timed beside the headline, or 'none'")
    ap.add_argument("--impl", default="lt2", choices=["lt2", "reference"])
    ap.add_argument("--order", default="delta_first", choices=["delta_first", "decay_first"],
                    help="order of the per-key factors (per-key workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    extras = [] if args.extras in ("", "none") else [e for e in args.extras.split(",") if e]
    for e in extras:
        if e not in EXTRAS and e != HEADLINE:
            ap.error(f"unknown extra workload {e!r}")
    extras = [e for e in extras if e != args.workload]

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        reference_arm(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return

    world, rank, local = dist_setup(args.gpus)
    lt2.lib()
    peaks, peak_src = load_peaks()
    sampler = ClockSampler(local) if rank == 0 else None
    cpu = rank == 0 and world == 1 and not args.no_cpu_baseline

    # ---- headline ----
    w = inputs.workload(args.workload)
    head, case = run_prefill(w, args, world, sampler, peaks, peak_src, keep=not args.no_e2e)
    line = {"metric": head["metric"], "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic", "config": head["config"], "roofline": head["roofline"],
            "gpu_launches": head["gpu_launches"]}
    if not args.no_e2e:
        x, _, _, dims, _ = case
        ems, h2d, d2h = run_e2e(w, x, dims, 3, 1, world)
        line["e2e"] = {"value": gdist.whole_job_rate(w.T * w.B * w.L, world, ems),
                       "unit": head["unit"], "ms_per_step": ems, "steps": 3,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "workload": w.name}
        del case, x
        torch.cuda.empty_cache()
    if cpu:
        line["cpu_baseline"] = cpu_entry(w, args.order, target_s=10.0)

    # ---- the other workloads, each with its own timing, roofline and baseline ----
    for name in extras:
        if name == "fused_gdn_prefill":
            entry = run_fused(args, world, sampler, peaks, peak_src)
        elif name == "backward_gdn":
            entry = run_backward(args, world, sampler)
            if cpu:
                v, threads, desc = oracle_backward_sample()
                entry["cpu_baseline"] = {"value": v, "unit": "tokens*loops/s", "cores": threads,
                                         "kind": "oracle", "sample": desc}
        elif name == "swa_prefill":
            entry = run_swa(args, world, sampler, peaks, peak_src)
            if cpu:
                v, threads, desc = oracle_swa_sample()
                entry["cpu_baseline"] = {"value": v, "unit": "tokens*loops/s", "cores": threads,
                                         "kind": "oracle", "sample": desc}
        elif name == "decode":
            entry, (wd, xs, S_host) = run_decode(args, world, sampler, peaks, peak_src)
            if cpu:
                v, threads, desc = oracle_decode_sample(wd, xs, S_host)
                entry["cpu_baseline"] = {"value": v, "unit": "tokens*loops/s", "cores": threads,
                                         "kind": "oracle", "sample": desc}
        else:
            we = inputs.workload(name)
            entry, _ = run_prefill(we, args, world, sampler, peaks, peak_src)
            if cpu:
                entry["cpu_baseline"] = cpu_entry(we, args.order, target_s=6.0)
        line[name] = entry

    if sampler is not None:
        sampler.stop()
        line["clocks"] = sampler.summary([w.name])
        line["clocks_all_regions"] = sampler.summary()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
