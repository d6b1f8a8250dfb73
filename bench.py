#!/usr/bin/env python
"""Benchmark: GPTQ of one Llama-2-7B-shaped decoder layer on B200.

One step = the whole hot path for one decoder layer: accumulate the four
calibration Hessians (H = 2 X^T X over 128 x 2048 = 262,144 bf16 tokens each,
for the attention input, the o_proj input, the MLP input and the down_proj
input), factor each once (damped inverse Cholesky, desc_act permutation), and
sweep all seven linears (q/k/v/o 4096x4096, gate/up 11008x4096, down
4096x11008; 4-bit, group 128, desc_act, static_groups, damp 0.01).  Inputs are
synthetic (seeded Student-t activations, Gaussian weights with 0.5% outliers)
and resident in HBM; at 12 GB they are far larger than L2, so no flush is
needed between steps.

The headline metric is weight columns quantized per second over the layer
(sum of n_in over the seven linears / step time); ms per step is the ms per
decoder layer.  Multi-GPU runs are independent replicas (one layer per rank,
weak scaling); ranks only meet at barriers and at the max-over-ranks timing.

`--impl reference` times the float64 CPU oracle on the same workload, one bounded
piece of the layer per step (pieces at the layer's own shapes, each scaled to the layer
by an exact work ratio), and reports the same metric; `--cpu-full-layer` times the
oracle on the whole layer once, beside the sample's estimate.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ ms/layer & weight-cols/s; Hessian TFLOPS; per-phase roofline fraction"
DATASHEET_BF16_DENSE_TFLOPS = 2250.0
UNIT = "weight-cols/s"


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--config", default="llama7b")
    p.add_argument("--tokens", type=int, default=0, help="override calibration tokens (testing only)")
    p.add_argument("--e2e-steps", type=int, default=6)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--two-phase", action="store_true",
                   help="time the layer with factors and sweeps as two phases instead of the pipelined call")
    p.add_argument("--phase-steps", type=int, default=3,
                   help="untimed-for-the-headline two-phase steps that attribute time to the factor and the sweep")
    p.add_argument("--qlinear", action="store_true",
                   help="measure the linear on the quantized checkpoint (decode, dequantization, GEMM) alone")
    p.add_argument("--qlinear-shape", default="", help="with --qlinear: only the shapes whose name contains this")
    p.add_argument("--cpu-full-layer", action="store_true",
                   help="time the float64 oracle on the whole layer once (minutes of CPU) beside the sample estimate")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    sm_max=d.get("sm_max_mhz", 1965.0), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_max=1965.0, source="fallback")


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [v for v in sm if v > 0.5 * (max(smax) if smax else 1)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workload
WORKLOADS = {
    "tiny": "tiny single linear layer GPTQ (64x256, 512 tokens)",
    "opt125m": "OPT-125m-shaped decoder layer GPTQ (6 linears, 4 Hessians)",
    "llama7b": "Llama-2-7B-shaped decoder layer GPTQ (7 linears, 4 Hessians)",
    "sweep": "4096x11008 down_proj-shaped layer GPTQ (1 linear, 1 Hessian)",
    "llama70b": "Llama-2-70B-shaped decoder layer GPTQ (7 linears, 4 Hessians)",
}


def workload_name(config):
    return f"{config}: {WORKLOADS.get(config, config)}"


def layer_columns(cfg):
    return sum(m.n_in for m in cfg.layers)


def algorithmic_work(cfg, T):
    """Per decoder layer: Hessian flops T*n(n+1) per distinct input, factor 2n^3/3,
    sweep lazy-update flops n_out*n_in^2, and the sweep's minimum HBM bytes."""
    hs = [T * n * (n + 1) for n in cfg.hessian_n]
    fac = [2 * n ** 3 / 3 for n in cfg.hessian_n]
    sw = [m.n_out * m.n_in ** 2 for m in cfg.layers]
    sw_bytes = 0
    for m in cfg.layers:
        G = 1 if cfg.group_size == -1 else m.n_in // cfg.group_size
        sw_bytes += m.n_out * m.n_in * 2 + m.n_in ** 2 * 2 + m.n_out * m.n_in * cfg.bits / 8 + G * m.n_out * 8
    return dict(hessian_flops=hs, factor_flops=fac, sweep_flops=sw, sweep_min_bytes=sw_bytes)


def make_inputs(cfg, T, device, rank):
    import torch

    from post_weight_quantization_layer_b200 import synth
    acts = {}
    for h, n in enumerate(cfg.hessian_n):
        a = synth.acts_for(cfg, h, tokens=T)
        a.seed += 7919 * rank
        acts[h] = a.full(device=device)
    weights = {m.name: synth.weight_for(cfg, m, device=device) for m in cfg.layers}
    torch.cuda.synchronize()
    return acts, weights


def run_native(args, world, rank, local):
    import torch

    import post_weight_quantization_layer_b200 as gq
    from post_weight_quantization_layer_b200 import synth
    from post_weight_quantization_layer_b200.layer import quantize_decoder_layer

    peaks = load_peaks()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[args.config]
    T = args.tokens or cfg.tokens
    acts, weights = make_inputs(cfg, T, dev, rank)
    Hbuf = {h: torch.empty(n, n, dtype=torch.float32, device=dev) for h, n in enumerate(cfg.hessian_n)}
    stream = torch.cuda.current_stream()

    def step(timing=False, pipelined=not args.two_phase):
        return quantize_decoder_layer(acts, weights, cfg.layers, cfg, hessians=Hbuf, timing=timing, stream=stream,
                                      pipelined=pipelined)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    barrier(world)

    props = torch.cuda.get_device_properties(dev)
    gpu_id = getattr(props, "uuid", None)
    gpu_id = f"GPU-{gpu_id}" if gpu_id is not None and not str(gpu_id).startswith("GPU-") else (gpu_id or local)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    n_launch0 = gq.launch_count()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    phase = []
    e0.record(stream)
    for _ in range(args.steps):
        _, t = step(timing=True)
        phase.append(t)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = gq.launch_count() - n_launch0
    clocks = sampler.stop()
    ms_local = e0.elapsed_time(e1) / args.steps
    barrier(world)
    ms = max_over_ranks(ms_local, world, dev)

    cols = layer_columns(cfg)
    value = cols * world / (ms / 1e3)
    work = algorithmic_work(cfg, T)
    fs_ms = statistics.mean(p.factor_sweep_ms for p in phase)
    spread = {"step_ms": [round(f(p.total_ms for p in phase), 3) for f in (min, statistics.median, max)],
              "factor_and_sweep_ms": [round(f(p.factor_sweep_ms for p in phase), 3)
                                      for f in (min, statistics.median, max)]}
    # factor and sweep apart: the timed steps themselves in the two-phase route, else a few
    # extra two-phase steps after the timed region (same inputs, bit-identical results)
    attrib = phase
    if not args.two_phase:
        attrib = [step(timing=True, pipelined=False)[1] for _ in range(max(args.phase_steps, 1))]
    f_ms = statistics.mean(p.factor_ms for p in attrib)
    s_ms = statistics.mean(p.sweep_ms for p in attrib)
    # the Hessian phase and its launches from the two-phase steps, where nothing overlaps them
    h_ms = statistics.mean(p.hessian_ms for p in attrib)
    spread["two_phase_hessian_ms"] = [round(f(p.hessian_ms for p in attrib), 3) for f in (min, statistics.median, max)]
    spread["two_phase_factor_ms"] = [round(f(p.factor_ms for p in attrib), 3) for f in (min, statistics.median, max)]
    spread["two_phase_sweep_ms"] = [round(f(p.sweep_ms for p in attrib), 3) for f in (min, statistics.median, max)]
    launch_ms = [statistics.mean(p.hessian_launch_ms[i] for p in attrib) for i in range(len(cfg.hessian_n))]
    h_flops = sum(work["hessian_flops"])
    h_tflops = h_flops / (sum(launch_ms) / 1e3) / 1e12
    per_launch = [work["hessian_flops"][i] / (launch_ms[i] / 1e3) / 1e12 for i in range(len(launch_ms))]
    f_tflops = sum(work["factor_flops"]) / (f_ms / 1e3) / 1e12
    s_tflops = sum(work["sweep_flops"]) / (s_ms / 1e3) / 1e12
    fp64_peak = measure_fp64_peak(dev)

    roofline = {
        "kernel": "hessian_syrk_kernel (tcgen05 kind::f16, bf16 in, fp32 accumulate)",
        "bound": "tensor",
        "achieved": round(h_tflops, 1),
        "peak": peaks["bf16_sus"],
        "peak_kind": f"bf16 dense sustained ({peaks['source']})",
        "unit": "TFLOP/s",
        "frac": round(h_tflops / peaks["bf16_sus"], 4),
        "traffic": None,
        "algorithmic_flops_per_launch": work["hessian_flops"],
        "per_launch_tflops": [round(x, 1) for x in per_launch],
        "launch_timing": ("the timed steps' launches" if args.two_phase else
                          "launches of the two-phase steps after the timed region (in the pipelined steps "
                          "three of the four Hessians overlap the largest one's factorisation)"),
    }
    traffic = hessian_traffic(cfg, T)
    if traffic is not None:
        # per launch, like `achieved` (the mean over this layer's Hessian launches)
        roofline["traffic"] = round(statistics.mean(traffic["per_launch"]))
        roofline["traffic_per_launch"] = traffic["per_launch"]
        roofline["traffic_source"] = traffic["source"]
        roofline["algorithmic_bytes_per_launch"] = [2 * T * n + 4 * n * n for n in cfg.hessian_n]

    phases = {
        "hessian": {"ms": round(h_ms, 3), "tflops": round(h_tflops, 1),
                    "frac_of_bf16_sustained": round(h_tflops / peaks["bf16_sus"], 4),
                    "frac_of_bf16_burst": round(h_tflops / peaks["bf16"], 4),
                    "frac_of_datasheet_dense_bf16": round(h_tflops / DATASHEET_BF16_DENSE_TFLOPS, 4),
                    "datasheet_note": "2250 TFLOP/s: NVIDIA's dense (non-sparse) bf16 figure for B200 at its "
                                      "boost clock, not measured on this part"},
        "factor_and_sweep": {"ms": round(fs_ms, 3), "pipelined": not args.two_phase,
                             "two_phase_ms": round(f_ms + s_ms, 3),
                             "note": ("timed steps, two phases" if args.two_phase else
                                      "timed steps: from the largest Hessian's completion to the end, overlapping "
                                      "the other Hessians' accumulation") +
                                     "; the hessian, factor and sweep entries come from two-phase steps"
                                     + ("" if args.two_phase else " run after the timed region")},
        "factor": {"ms": round(f_ms, 3), "tflops_fp64": round(f_tflops, 2),
                   "frac_of_fp64_peak": round(f_tflops / fp64_peak, 4)},
        "sweep": {"ms": round(s_ms, 3), "tflops_fp64": round(s_tflops, 2),
                  "frac_of_fp64_peak": round(s_tflops / fp64_peak, 4),
                  "min_hbm_gbs": round(work["sweep_min_bytes"] / (s_ms / 1e3) / 1e9, 1),
                  "frac_of_hbm": round(work["sweep_min_bytes"] / (s_ms / 1e3) / 1e9 / peaks["hbm"], 4)},
        "spread_min_median_max": spread,
        "fp64_peak_tflops": round(fp64_peak, 1),
        "fp64_peak_how": "measured in this run: cuBLAS fp64 GEMM 8192^3 (torch.matmul), best of 3",
    }

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, cfg, acts, weights, dev, stream, world, Hbuf)
    del acts, weights
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, T)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 activations / fp16 weights; fp32 accumulate; fp32+fp64 sweep",
        "data": "synthetic (seeded Student-t activations, Gaussian+outlier weights; no datasets or checkpoints)",
        "config": {"workload": workload_name(args.config),
                   "tokens": T, "bits": cfg.bits, "group_size": cfg.group_size, "desc_act": cfg.desc_act,
                   "static_groups": cfg.static_groups, "damp_percent": cfg.damp_percent,
                   "weight_cols_per_layer": cols, "parallelism": f"replicas x{world}",
                   "l2": "inputs (12 GB of activations) larger than L2; no flush"},
        "ms_per_layer": round(ms, 3),
        "phases": phases,
        "roofline": roofline,
        "gpu_launches": launches,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    return line


def measure_fp64_peak(dev):
    """Denominator of the fp64 phases: this GPU's fp64 GEMM rate, measured with cuBLAS."""
    import torch
    n = 8192
    a = torch.randn(n, n, device=dev, dtype=torch.float64)
    b = torch.randn(n, n, device=dev, dtype=torch.float64)
    a @ b
    torch.cuda.synchronize()
    best = 1e30
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        a @ b
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2 * n ** 3 / (best / 1e3) / 1e12


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "hessian_syrk_traffic.json")


def hessian_traffic(cfg, T):
    """DRAM bytes (read + write) of each Hessian launch of the layer at T tokens, from the
    committed ncu counters of small-case launches of the same kernel (same widths, fewer
    tokens): for each width the counters of two token counts give bytes = a + b * T
    (X is streamed once per token segment group, H written a fixed number of times), which
    is evaluated at T.  None when the file has no capture of a width, or was taken from
    another build of the kernel than this source (its `kernel_sha` field)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("kernel_sha") != kernel_source_sha():
        return None
    per_launch = []
    for n in cfg.hessian_n:
        pts = sorted((c["tokens"], c["dram_bytes"]) for c in d.get("captures", []) if c["n"] == n)
        if len(pts) < 2:
            return None
        (t0, b0), (t1, b1) = pts[0], pts[-1]
        slope = (b1 - b0) / (t1 - t0)
        per_launch.append(round(b1 + slope * (T - t1)))
    caps = ", ".join(f"n={c['n']} T={c['tokens']}" for c in d["captures"])
    return {"per_launch": per_launch,
            "source": f"ncu dram__bytes_read.sum + dram__bytes_write.sum of small-case launches ({caps}), "
                      f"line through two token counts per width evaluated at T={T}; profiles/hessian_syrk_traffic.json"}


def kernel_source_sha():
    """Short hash of the Hessian kernel's sources (the counters belong to this code)."""
    import hashlib
    h = hashlib.sha256()
    for f in ("hessian.cu", "hessian_sched.cuh", "sm100.cuh"):
        with open(os.path.join(ROOT, "post_weight_quantization_layer_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def run_e2e(args, cfg, acts, weights, dev, stream, world, Hbuf):
    """Same metric through the public API with host buffers: every step copies its
    activations and weights from pinned host memory, runs the layer and reads the packed
    results back.  The copies of step k+1 run on a copy stream while step k computes
    (two device buffer sets; a set is refilled only after the step that read it has
    finished), as a calibration pipeline streaming layer after layer would; every step's
    copy lies inside the timed region."""
    import torch

    from post_weight_quantization_layer_b200.layer import quantize_decoder_layer
    h_acts = {h: x.cpu().pin_memory() for h, x in acts.items()}
    h_w = {k: w.cpu().pin_memory() for k, w in weights.items()}
    sets = [({h: torch.empty_like(x) for h, x in acts.items()}, {k: torch.empty_like(w) for k, w in weights.items()})
            for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in h_acts.values()) + \
        sum(w.numel() * w.element_size() for w in h_w.values())
    cs = torch.cuda.Stream(device=dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    for e in freed:
        e.record(stream)

    def issue_copy(b):
        d_acts, d_w = sets[b]
        cs.wait_event(freed[b])
        with torch.cuda.stream(cs):
            for h in h_acts:
                d_acts[h].copy_(h_acts[h], non_blocking=True)
            for k in h_w:
                d_w[k].copy_(h_w[k], non_blocking=True)
        copied[b].record(cs)

    def compute(b):
        d_acts, d_w = sets[b]
        stream.wait_event(copied[b])
        res, _ = quantize_decoder_layer(d_acts, d_w, cfg.layers, cfg, hessians=Hbuf, stream=stream)
        freed[b].record(stream)
        outs = []
        with torch.cuda.stream(stream):
            for r in res.values():
                for t in (r.qweight, r.scales, r.zeros, r.g_idx):
                    outs.append(t.to("cpu", non_blocking=True))
        return outs

    def run(steps):
        start = torch.cuda.Event()
        start.record(stream)
        cs.wait_event(start)  # the first copy starts inside the region timed on `stream`
        issue_copy(0)
        outs = []
        for i in range(steps):
            if i + 1 < steps:
                issue_copy((i + 1) % 2)
            outs = compute(i % 2)
        torch.cuda.synchronize()
        return sum(t.numel() * t.element_size() for t in outs)

    run(2)
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    d2h = run(args.e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
    del sets
    return {"value": round(layer_columns(cfg) * world / (ms / 1e3), 1), "unit": UNIT,
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pipelining": "step k+1's host-to-device copies overlap step k's compute (copy stream, 2 buffer sets)"}


# ------------------------------------------------------------------ CPU oracle baseline
SAMPLE_TOKENS = 8192           # one calibration chunk (the streaming unit of the Hessian)
SAMPLE_SWEEP_BYTES = 64 << 20  # fp64 running weights per sampled sweep: out of cache, like the layer's


class OracleSample:
    """The float64 oracle on a bounded sample of one decoder layer, cut into pieces whose
    shapes are the layer's own, each with the factor that scales it to the whole layer:

    * Hessian h: 2 X^T X of one 8,192-token chunk at the full width n_h; the oracle's
      Hessian of T tokens is the sum of T / 8192 such chunk products (scale T / 8192);
    * factor h: act-order permutation, damping and inverse-Cholesky factor at the full
      width (scale 1; the chunk Hessian is made positive definite by the damping, and the
      factor's cost does not depend on its values);
    * sweep of each distinct linear shape (n_out, n_in): rows of its first linear at the
      full width against that linear's factor, as many rows as make 64 MB of fp64 running
      weights (a working set out of the host's caches, as the whole layer's is; smaller
      samples ran up to 1.8x faster per row); rows are independent given the factor and the
      sweep's time is linear in them (scale: linears of that shape x n_out / rows).

    Inputs are drawn and prepared once (untimed).  `time_piece` times one piece."""

    def __init__(self, cfg, T):
        import numpy as np

        import oracle as O
        from post_weight_quantization_layer_b200 import synth
        self.O, self.np, self.cfg, self.T = O, np, cfg, T
        self.X = {h: synth.acts_for(cfg, h, tokens=SAMPLE_TOKENS).full().double().numpy()
                  for h in range(len(cfg.hessian_n))}
        self.W, self.rows, self.count = {}, {}, {}
        for m in cfg.layers:
            shape = (m.n_out, m.n_in)
            self.count[shape] = self.count.get(shape, 0) + 1
            if any((o.n_out, o.n_in) == shape for o in cfg.layers[:cfg.layers.index(m)]):
                continue  # one piece per distinct shape: its first linear
            rows = min(m.n_out, max(1, SAMPLE_SWEEP_BYTES // (8 * m.n_in)))
            W = synth.weight_for(cfg, m).double().numpy()
            self.W[m.name] = np.ascontiguousarray(W[:rows])
            self.rows[m.name] = rows
        self.H, self.factor = {}, {}
        self.pieces = [("hessian", h) for h in self.X] + [("factor", h) for h in self.X] + \
                      [("sweep", name) for name in self.W]
        self.times = {p: [] for p in self.pieces}

    def scale(self, piece):
        kind, key = piece
        if kind == "hessian":
            return self.T / SAMPLE_TOKENS
        if kind == "factor":
            return 1.0
        m = next(m for m in self.cfg.layers if m.name == key)
        return self.count[(m.n_out, m.n_in)] * m.n_out / self.rows[key]

    def _run(self, piece):
        O, np, cfg = self.O, self.np, self.cfg
        kind, key = piece
        if kind == "hessian":
            self.H[key] = O.hessian(self.X[key])
        elif kind == "factor":
            H = self.H[key]
            perm = O.act_order_perm(H) if cfg.desc_act else np.arange(H.shape[0])
            U = O.inverse_cholesky_upper(O.dampen(H[np.ix_(perm, perm)], cfg.damp_percent))
            self.factor[key] = (perm, U)
        else:
            m = next(m for m in cfg.layers if m.name == key)
            perm, U = self.factor[m.h_index]
            W = self.W[key]
            O.gptq_sweep(W[:, perm], U, cfg.bits, cfg.sym, cfg.group_size, perm, cfg.static_groups, W,
                         cfg.blocksize)

    def time_piece(self, piece):
        """Run one piece (its inputs must exist: Hessian before factor before sweep)."""
        t0 = time.perf_counter()
        self._run(piece)
        dt = time.perf_counter() - t0
        self.times[piece].append(dt)
        return dt

    def run_all(self):
        """Every piece once, in dependency order (the cpu_baseline measurement)."""
        for p in self.pieces:
            self.time_piece(p)

    def layer_seconds(self):
        """Whole-layer oracle seconds from the mean time of each piece times its scale."""
        return sum(statistics.mean(self.times[p]) * self.scale(p) for p in self.pieces if self.times[p])

    def spent(self):
        return sum(sum(v) for v in self.times.values())

    def describe(self):
        parts = {"hessian": [], "factor": [], "sweep": []}
        for p in self.pieces:
            if self.times[p]:
                rows = f" ({self.rows[p[1]]} rows)" if p[0] == "sweep" else ""
                parts[p[0]].append(f"{p[1]}{rows} {statistics.mean(self.times[p]):.2f} s x{self.scale(p):.4g}")
        return (f"float64 oracle on the host cores, pieces of the layer at its own shapes, each timed and "
                f"scaled to the layer: Hessian of one {SAMPLE_TOKENS}-token chunk per input (scale T/{SAMPLE_TOKENS}): "
                + ", ".join(parts["hessian"]) + "; factor at full width per input: " + ", ".join(parts["factor"]) +
                "; sweep per distinct linear shape at full width (rows for 64 MB of running weights; scale "
                "linears of the shape x n_out/rows): " + ", ".join(parts["sweep"]) +
                f"; {self.spent():.1f} s of CPU work timed")


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(cfg, T):
    smp = OracleSample(cfg, T)
    smp.run_all()
    total = smp.layer_seconds()
    return {"value": round(layer_columns(cfg) / total, 3), "unit": UNIT, "cores": cpu_cores(),
            "kind": "oracle", "sample": smp.describe(), "s_per_layer_extrapolated": round(total, 1)}


def run_reference(args, world, rank):
    """The oracle as the reference arm: rank 0 alone.  Each step is one piece of the layer
    sample (OracleSample), taken round-robin, so a step is a bounded amount of CPU work;
    ms_per_step is the time the steps actually took, and the layer-time estimate comes
    from the per-piece times scaled to the layer (any piece no timed step reached is
    taken from the set-up pass, which times every piece once)."""
    if rank != 0:
        return None
    from post_weight_quantization_layer_b200 import synth
    cfg = synth.CONFIGS[args.config]
    T = args.tokens or cfg.tokens
    smp = OracleSample(cfg, T)
    smp.run_all()  # set-up: every piece's inputs and one timing of each
    setup = {p: list(v) for p, v in smp.times.items()}
    for p in smp.pieces:
        smp.times[p] = []
    k = 0
    for _ in range(max(args.warmup, 0)):
        smp._run(smp.pieces[k % len(smp.pieces)])
        k += 1
    step_s = []
    for _ in range(args.steps):
        step_s.append(smp.time_piece(smp.pieces[k % len(smp.pieces)]))
        k += 1
    for p in smp.pieces:
        if not smp.times[p]:
            smp.times[p] = setup[p]
    layer_s = smp.layer_seconds()
    value = layer_columns(cfg) / layer_s
    ms = 1e3 * statistics.mean(step_s) if step_s else 0.0
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(args.config),
                   "tokens": T},
        "step_is": "one piece of the oracle's layer sample (round-robin over "
                   f"{len(smp.pieces)} pieces); ms_per_step is measured",
        "s_per_layer_extrapolated": round(layer_s, 1),
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": smp.describe()},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_cpu_full_layer(args):
    """Calibration of the sample: the oracle on the WHOLE decoder layer once (all tokens,
    all rows; several minutes of CPU), next to the sample's estimate in the same run."""
    import numpy as np

    import oracle as O
    from post_weight_quantization_layer_b200 import synth
    cfg = synth.CONFIGS[args.config]
    T = args.tokens or cfg.tokens
    smp = OracleSample(cfg, T)
    smp.run_all()
    est = smp.layer_seconds()
    del smp
    phase = {"hessian": 0.0, "factor": 0.0, "sweep": 0.0}
    factors = {}
    for h, n in enumerate(cfg.hessian_n):
        acts = synth.acts_for(cfg, h, tokens=T)
        H = np.zeros((n, n))
        for i in range(acts.n_chunks):
            X = acts.get_chunk(i).double().numpy()
            t0 = time.perf_counter()
            H += O.hessian(X)
            phase["hessian"] += time.perf_counter() - t0
        t0 = time.perf_counter()
        perm = O.act_order_perm(H) if cfg.desc_act else np.arange(n)
        U = O.inverse_cholesky_upper(O.dampen(H[np.ix_(perm, perm)], cfg.damp_percent))
        phase["factor"] += time.perf_counter() - t0
        factors[h] = (perm, U)
        del H
    for m in cfg.layers:
        W = synth.weight_for(cfg, m).double().numpy()
        perm, U = factors[m.h_index]
        t0 = time.perf_counter()
        O.gptq_sweep(W[:, perm], U, cfg.bits, cfg.sym, cfg.group_size, perm, cfg.static_groups, W, cfg.blocksize)
        phase["sweep"] += time.perf_counter() - t0
    full = sum(phase.values())
    return {"impl": "oracle-full-layer", "config": args.config, "tokens": T, "cores": cpu_cores(),
            "s_per_layer_measured": round(full, 1), "phases_s": {k: round(v, 1) for k, v in phase.items()},
            "value_measured": round(layer_columns(cfg) / full, 3), "unit": UNIT,
            "s_per_layer_sample_estimate": round(est, 1), "estimate_over_measured": round(est / full, 3)}


def run_qlinear(args):
    """The linear on the quantized checkpoint (4-bit, group 128; act order, and for decoding also
    without it and with the act-order checkpoint's inputs sorted by group), measured alone on Llama-shaped weights quantized by the library itself: the decode kernel (M = 1 and 4 rows; HBM-bound: bytes =
    packed codes + fp16 scales + packed zero points + g_idx + X + Y) against the measured
    copy bandwidth, the dequantization (bytes = the checkpoint read + the 16-bit weight
    written) likewise, and the tensor-core GEMM (2 M N K flops) against the measured bf16
    rate.  Device time: the call's launches captured once in a CUDA graph and replayed, CUDA
    events around each replay, 3 warm-ups, the median of 20; decode also reports the wall time
    of one call through the Python binding (call_us, host overhead included).  Weights are
    re-read every launch (decode shapes below L2 are reported as such)."""
    import torch

    import post_weight_quantization_layer_b200 as gq
    from post_weight_quantization_layer_b200 import synth
    from post_weight_quantization_layer_b200._native import lib
    peaks = load_peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    def timed(fn, reps=20):
        """Device time of one fn() (median over reps), its launches replayed from a CUDA graph
        so that the host-side cost of the Python call is not in the number."""
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        try:
            with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
                fn()
        except RuntimeError as e:  # not capturable: time back-to-back calls instead
            print(f"graph capture failed ({e}); timing 20 queued calls", file=sys.stderr)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            e1.synchronize()
            return e0.elapsed_time(e1) / reps
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        del g
        return statistics.median(ts)

    def call_timed(fn, reps=20):
        """Wall time of one call through the Python binding, host overhead included."""
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            t0 = time.perf_counter()
            fn()
            torch.cuda.synchronize()
            ts.append(time.perf_counter() - t0)
        return statistics.median(ts) * 1e3

    out = {"mode": "qlinear", "unit_decode": "GB/s", "unit_gemm": "TFLOP/s", "hbm_peak_gbs": peaks["hbm"],
           "bf16_peak_tflops": peaks["bf16"], "peaks": peaks["source"], "shapes": []}
    bits, g = 4, 128
    shapes = (("7b q_proj", 4096, 4096), ("7b gate_proj", 4096, 11008), ("7b down_proj", 11008, 4096),
              ("70b gate_proj", 8192, 28672), ("70b down_proj", 28672, 8192))
    for name, n_in, n_out in shapes:
        if args.qlinear_shape and args.qlinear_shape not in name:
            continue
        # a real checkpoint of the library's own making: Hessian, GPTQ with act order, export
        W = synth.outlier_weight(n_out, n_in, 11, device=dev)
        H = torch.zeros(n_in, n_in, device=dev)
        acts = synth.StudentTActs(n_in, 2 * n_in, 12, dtype=torch.bfloat16)
        for i in range(acts.n_chunks):
            gq.accumulate_hessian(acts.get_chunk(i, device=dev), H)
        from post_weight_quantization_layer_b200.export import export_layer
        ck = export_layer(gq.quantize_layer(W, H, bits, g, 0.01, True, True, False, 128), bits)
        ck_mono = export_layer(gq.quantize_layer(W, H, bits, g, 0.01, True, False, False, 128), bits)
        del W, H
        G = ck["scales"].shape[0]
        wbytes = n_in * n_out * bits // 8 + G * n_out * (2 + bits / 8) + n_in * 4
        row = {"shape": name, "n_in": n_in, "n_out": n_out, "weight_bytes": int(wbytes)}
        ck_re = gq.reorder_act_order(ck, bits)  # the act-order checkpoint with its inputs sorted by group
        for tag, c in (("", ck), ("_monotone_groups", ck_mono), ("_act_order_reordered", ck_re)):
            for M in (1, 4):
                X = torch.randn(M, n_in, device=dev).to(torch.bfloat16)
                Y = torch.empty(M, n_out, device=dev, dtype=torch.bfloat16)
                fn = lambda: gq.quantized_linear(X, c, bits, out=Y)  # noqa: E731
                ms = timed(fn)
                gbs = (wbytes + M * (n_in + n_out) * 2) / (ms / 1e3) / 1e9
                row[f"decode_m{M}{tag}"] = {"us": round(ms * 1e3, 1), "gbs": round(gbs, 1),
                                            "frac_of_hbm": round(gbs / peaks["hbm"], 3),
                                            "l2_resident": wbytes < 100e6,
                                            "call_us": round(call_timed(fn) * 1e3, 1)}
        Wd = torch.empty(n_out, n_in, dtype=torch.bfloat16, device=dev)
        ms = timed(lambda: lib().gptq_dequantize_weight(ck["qweight"].data_ptr(), ck["qzeros"].data_ptr(),
                                                         ck["scales"].data_ptr(), ck["g_idx"].data_ptr(), G, n_in,
                                                         n_out, bits, 2, Wd.data_ptr(),
                                                         torch.cuda.current_stream().cuda_stream))
        gbs = (wbytes + n_in * n_out * 2) / (ms / 1e3) / 1e9
        row["dequant"] = {"us": round(ms * 1e3, 1), "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm"], 3)}
        for M in (2048, 16384):
            X = torch.randn(M, n_in, device=dev).to(torch.bfloat16)
            Y = torch.empty(M, n_out, device=dev, dtype=torch.bfloat16)
            ms = timed(lambda: gq.quantized_linear(X, ck, bits, out=Y), reps=10)
            tf = 2 * M * n_in * n_out / (ms / 1e3) / 1e12
            row[f"gemm_m{M}"] = {"ms": round(ms, 3), "tflops": round(tf, 1), "frac_of_bf16_burst": round(tf / peaks["bf16"], 3)}
            del X, Y
        out["shapes"].append(row)
        del ck, Wd
        torch.cuda.empty_cache()
    return out


def main():
    args = parse_args()
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.qlinear:
            line = run_qlinear(args) if rank == 0 else None
        elif args.cpu_full_layer:
            line = run_cpu_full_layer(args) if rank == 0 else None
        elif args.impl == "reference":
            line = run_reference(args, world, rank)
        else:
            line = run_native(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
