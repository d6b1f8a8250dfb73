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

`--impl reference` times the float64 CPU oracle on a bounded sample of the same
workload and reports the same metric (extrapolated per phase by work).
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

    def step(timing=False):
        return quantize_decoder_layer(acts, weights, cfg.layers, cfg, hessians=Hbuf, timing=timing, stream=stream)

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
    h_ms = statistics.mean(p.hessian_ms for p in phase)
    f_ms = statistics.mean(p.factor_ms for p in phase)
    s_ms = statistics.mean(p.sweep_ms for p in phase)
    launch_ms = [statistics.mean(p.hessian_launch_ms[i] for p in phase) for i in range(len(cfg.hessian_n))]
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
    }
    traffic = load_traffic() if args.config == "llama7b" and T == cfg.tokens else None
    if traffic is not None and len(traffic) == len(launch_ms):
        # per launch, like `achieved` (the mean over this layer's Hessian launches)
        roofline["traffic"] = round(statistics.mean(traffic))
        roofline["traffic_per_launch"] = traffic
        roofline["traffic_source"] = "ncu dram__bytes_read.sum + dram__bytes_write.sum, " \
                                     "profiles/hessian_syrk_dram_llama7b_layer.md"

    phases = {
        "hessian": {"ms": round(h_ms, 3), "tflops": round(h_tflops, 1),
                    "frac_of_bf16_sustained": round(h_tflops / peaks["bf16_sus"], 4)},
        "factor": {"ms": round(f_ms, 3), "tflops_fp64": round(f_tflops, 2),
                   "frac_of_fp64_peak": round(f_tflops / fp64_peak, 4)},
        "sweep": {"ms": round(s_ms, 3), "tflops_fp64": round(s_tflops, 2),
                  "frac_of_fp64_peak": round(s_tflops / fp64_peak, 4),
                  "min_hbm_gbs": round(work["sweep_min_bytes"] / (s_ms / 1e3) / 1e9, 1),
                  "frac_of_hbm": round(work["sweep_min_bytes"] / (s_ms / 1e3) / 1e9 / peaks["hbm"], 4)},
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
        "config": {"workload": f"{args.config}: Llama-2-7B-shaped decoder layer GPTQ (7 linears, 4 Hessians)",
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


def load_traffic():
    """DRAM bytes (read + write) per Hessian launch of one decoder layer, from the committed
    ncu summary of the same bench command (profiles/hessian_syrk_dram_llama7b_layer.md)."""
    path = os.path.join(ROOT, "profiles", "hessian_syrk_dram_llama7b_layer.md")
    try:
        with open(path) as f:
            for ln in f:
                if ln.startswith("traffic_bytes_per_launch:"):
                    return [float(x) for x in ln.split(":", 1)[1].strip().strip("[]").split(",")]
    except OSError:
        pass
    return None


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
def oracle_sample(cfg, T, budget_scale=1.0):
    """Time the float64 oracle on a bounded sample and extrapolate each phase to the
    full decoder layer along its cost structure: the Hessian by T*n^2 (a sample of
    tokens), the factor by n^3 (a smaller Hessian), the sweep by rows (full-width
    rows of each distinct n_in; rows are independent given the factor).
    Returns (seconds per layer, description, seconds spent)."""
    import numpy as np

    import oracle as O
    from post_weight_quantization_layer_b200 import synth

    spent = 0.0
    n0 = cfg.hessian_n[0]
    ts = max(256, int(1024 * budget_scale))
    X = synth.acts_for(cfg, 0, tokens=ts).full().double().numpy()
    t0 = time.perf_counter()
    H = O.hessian(X)
    t_h = time.perf_counter() - t0
    h_scale = sum(T * n * n for n in cfg.hessian_n) / (ts * n0 * n0)

    nf = min(n0, 2048 if budget_scale < 2 else 4096)
    t0 = time.perf_counter()
    O.inverse_cholesky_upper(O.dampen(H[:nf, :nf], cfg.damp_percent))
    t_f = time.perf_counter() - t0
    f_scale = sum(n ** 3 for n in cfg.hessian_n) / nf ** 3
    spent += t_h + t_f

    # Sweep: full-width rows per distinct n_in, with a valid upper-triangular factor
    # (a scaled identity; the sweep's cost does not depend on the factor's values).
    rows = max(16, int(128 * budget_scale))
    t_s_total = 0.0
    parts = []
    for n_in in sorted({m.n_in for m in cfg.layers}):
        W = synth.outlier_weight(rows, n_in, 5).double().numpy()
        U = np.eye(n_in) * 0.5
        t0 = time.perf_counter()
        O.gptq_sweep(W, U, cfg.bits, cfg.sym, cfg.group_size, np.arange(n_in), cfg.static_groups, W,
                     cfg.blocksize)
        dt = time.perf_counter() - t0
        spent += dt
        total_rows = sum(m.n_out for m in cfg.layers if m.n_in == n_in)
        t_s_total += dt * total_rows / rows
        parts.append(f"{rows}x{n_in} in {dt:.2f} s (x{total_rows / rows:.0f} rows)")
    total = t_h * h_scale + t_f * f_scale + t_s_total
    desc = (f"oracle float64 on host cores: Hessian of {ts} tokens x {n0} in {t_h:.2f} s (x{h_scale:.0f} by T*n^2), "
            f"factor n={nf} in {t_f:.2f} s (x{f_scale:.1f} by n^3), sweep " + ", ".join(parts) +
            f"; sample {spent:.1f} s of CPU work")
    return total, desc, spent


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(cfg, T):
    total, desc, _ = oracle_sample(cfg, T, 4.0)
    return {"value": round(layer_columns(cfg) / total, 3), "unit": UNIT, "cores": cpu_cores(),
            "kind": "oracle", "sample": desc, "s_per_layer_extrapolated": round(total, 1)}


def run_reference(args, world, rank):
    """The oracle as the reference arm: rank 0 alone, each step a bounded sample."""
    if rank != 0:
        return None
    from post_weight_quantization_layer_b200 import synth
    cfg = synth.CONFIGS[args.config]
    T = args.tokens or cfg.tokens
    for _ in range(max(args.warmup, 0)):
        oracle_sample(cfg, T, 0.5)
    tot = []
    desc = ""
    for _ in range(args.steps):
        t, desc, _ = oracle_sample(cfg, T, 0.5)
        tot.append(t)
    s = statistics.mean(tot)
    value = layer_columns(cfg) / s
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * s, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.config}: Llama-2-7B-shaped decoder layer GPTQ (7 linears, 4 Hessians)",
                   "tokens": T},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
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
