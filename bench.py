"""Throughput of the Muon step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama3|gpt2|moe|single]
                    [--impl ours|reference] [--no-e2e] [--no-cpu-baseline]

One "step" is one Muon optimizer step over the whole matrix set of the
workload: momentum/Nesterov/norm/cast, five quintic Newton-Schulz iterations
on the tensor cores, scale + weight decay + write. Default workload: the
Llama-3-8B hidden-matrix set (224 matrices, 6.98 G elements, bf16 grads,
fp32 params and momenta), synthetic inputs generated on the device from
seeds (workloads/). Inputs (70 GB) are far larger than L2, so no L2 flush is
needed between steps.

Metric: Muon steps/s for the whole job (weak scaling: with N GPUs every rank
runs its own full set, no collective on the data path), with NS TFLOP/s
(nominal 5 (4 s^2 l + 2 s^3) per matrix) and its fraction of peak.
Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle (the reference arm of this
method) on a bounded sample of the same workload, scaled to steps/s.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    "llama3": (W.CONFIG_LLAMA, W.llama3_8b_shapes, "bf16", "Llama-3-8B hidden matrices: 32 x {q 4096x4096, "
               "k 1024x4096, v 1024x4096, o 4096x4096, gate 14336x4096, up 14336x4096, down 4096x14336}"),
    "llama3_layer": (W.CONFIG_LLAMA, W.llama3_layer_shapes, "bf16", "one Llama-3-8B layer: {q 4096x4096, "
                     "k 1024x4096, v 1024x4096, o 4096x4096, gate 14336x4096, up 14336x4096, down 4096x14336}"),
    "gpt2": (W.CONFIG_GPT2, W.gpt2_shapes, "fp32", "GPT-2-small hidden matrices: 12 x {QKV 2304x768, "
             "O 768x768, up 3072x768, down 768x3072}"),
    "moe": (W.CONFIG_MOE, W.moe_shapes, "bf16", "MoE layer: 128 experts x {gate 2048x7168, up 2048x7168, "
            "down 7168x2048}"),
    "single": (W.CONFIG_SINGLE, W.single_shapes, "fp32", "one 256x512 gradient"),
}
LR, BETA, WD = 2e-4, 0.95, 0.1
NS_STEPS = 5
METRIC = "Muon steps/sec and NS TFLOP/s (% of B200 dense BF16 peak) per matrix set"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in ("muon_newton_schulz_03_b200/csrc/ns_tcgen05.cu", "muon_newton_schulz_03_b200/csrc/common.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def tensor_peak(peaks, peak_src, timed_ms):
    """The dense bf16 peak a timed region is held to: the sustained figure (a
    seconds-long loop under the power cap) for a region of a second or more,
    the burst figure for a shorter one. Returns (TFLOP/s, description)."""
    if timed_ms >= 1000.0:
        return (peaks["bf16_tflops_sustained"],
                f"{peak_src} sustained dense bf16 (timed region of {timed_ms / 1e3:.1f} s, inside a long run)")
    return peaks["bf16_tflops"], f"{peak_src} burst dense bf16 (timed region of {timed_ms:.0f} ms)"


def profiled_traffic(workload):
    """DRAM bytes per launch of the Newton-Schulz kernel from a committed ncu
    summary, if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"ns_phase_kernel_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        line = line.strip().strip("|").strip()
        if line.startswith("kernel_source_hash:"):
            vals["hash"] = line.split(":", 1)[1].strip()
        if line.startswith("traffic_bytes_per_launch:"):
            vals["traffic"] = float(line.split(":", 1)[1].strip())
    if vals.get("hash") == kernel_source_hash() and "traffic" in vals:
        return vals["traffic"]
    return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9], parts[4]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for nm, v in zip(names, r[2]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline and reference arm)
# ---------------------------------------------------------------------------

_ORACLE_INPUTS = {}


def oracle_inputs(workload, first_index):
    """The oracle's inputs for matrix `first_index` of the workload's set
    (generated once per process)."""
    key = (workload, first_index)
    if key not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[key] = _make_oracle_inputs(workload, first_index)
    return _ORACLE_INPUTS[key]


def _make_oracle_inputs(workload, first_index):
    import numpy as np
    config, shapes_fn, gdt, _ = WORKLOADS[workload]
    m, n = shapes_fn()[first_index]
    vals = W.set_values(config, shapes_fn(), gdt == "bf16", indices=[first_index])
    p, g, mom = vals[first_index]
    return p, g, np.zeros((m, n))


def time_oracle_class(workload, shape):
    """Seconds the float64 oracle takes for one Muon step of one matrix of
    this shape class (the class's first matrix in the set)."""
    from oracle import muon_oracle as O
    _, shapes_fn, _, _ = WORKLOADS[workload]
    count, first = W.shape_classes(shapes_fn())[shape]
    p, g, m = oracle_inputs(workload, first)
    t0 = time.perf_counter()
    O.muon_step_matrix(p, g, m, lr=LR, beta=BETA, wd=WD, ns_steps=NS_STEPS)
    return time.perf_counter() - t0


def set_seconds(workload, class_seconds):
    """Extrapolated seconds for the whole set: sum over shape classes of
    (matrices of that class) x (measured seconds for one of them)."""
    _, shapes_fn, _, _ = WORKLOADS[workload]
    classes = W.shape_classes(shapes_fn())
    return sum(classes[s][0] * t for s, t in class_seconds.items())


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((d.get("num_threads") or 0) for d in info) or os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(workload):
    """One oracle step on one matrix of every shape class of the set,
    extrapolated to the set by the class counts."""
    _, shapes_fn, _, _ = WORKLOADS[workload]
    classes = W.shape_classes(shapes_fn())
    secs = {s: time_oracle_class(workload, s) for s in classes}
    total = set_seconds(workload, secs)
    measured = sum(secs.values())
    return {"value": 1.0 / total, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
            "extrapolated": True, "measured_s": measured, "set_s": total,
            "sample": "float64 NumPy oracle, one Muon step of one matrix of every shape class "
                      + ", ".join(f"{m}x{n} ({classes[(m, n)][0]} in the set): {t:.2f} s"
                                  for (m, n), t in secs.items())
                      + "; set time = sum of count x class time"}


def run_reference(args):
    """The reference arm: the float64 CPU oracle. Step k times one matrix of
    shape class k mod C (C classes in the set), so every class is measured
    about K / C times; the reported step time is the sum over classes of
    (count in set) x (median time of that class). Warm-up steps run the
    cheapest class."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    _, shapes_fn, _, desc = WORKLOADS[args.workload]
    classes = list(W.shape_classes(shapes_fn()))
    cheapest = min(classes, key=lambda s: W.ns_flops(*s))
    for _ in range(args.warmup):
        time_oracle_class(args.workload, cheapest)
    per_class = {s: [] for s in classes}
    measured = 0.0
    for k in range(max(args.steps, len(classes))):
        s = classes[k % len(classes)]
        dt = time_oracle_class(args.workload, s)
        per_class[s].append(dt)
        measured += dt
    med = {s: statistics.median(v) for s, v in per_class.items()}
    ms = set_seconds(args.workload, med) * 1e3
    value = 1e3 / ms
    cores = blas_threads()
    sample = ("each step: one Muon step of the float64 oracle on one matrix of one shape class, classes in turn "
              + ", ".join(f"{m}x{n} x{len(per_class[(m, n)])} (median {med[(m, n)]:.2f} s)" for (m, n) in classes)
              + "; set time = sum of count in set x class median")
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "extrapolated": True, "measured_s": measured,
        "config": {"workload": desc, "matrices": len(shapes_fn()), "ns_steps": NS_STEPS},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle", "extrapolated": True,
                         "measured_s": measured, "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def executed_flops(shapes, steps, gram=False, pair=False):
    """FLOPs the tensor cores execute per Muon step: every listed tile is a
    BM x 256 x K product (K padded to 64), the symmetric phases list only the
    upper tiles; matrices on the on-chip small path count their nominal
    FLOPs."""
    import muon_newton_schulz_03_b200 as muon
    plan = muon.plan_query(shapes, "bf16", True, pair)
    bm = 256 if pair else 128

    def phase(tiles, use_l):
        f = 0.0
        for (mat, _, _) in tiles:
            m, n = shapes[mat][:2]
            k = max(m, n) if use_l else min(m, n)
            f += 2.0 * bm * 256 * (-(-k // 64) * 64)
        return f

    g, p, c = phase(plan["tiles"][0], True), phase(plan["tiles"][1], False), phase(plan["tiles"][2], False)
    if gram:
        two, one = steps // 2, steps % 2
        per = two * (g + 5 * p + c) + one * (g + p + c)
    else:
        per = steps * (g + p + c)
    small = sum(W.ns_flops(shapes[i][0], shapes[i][1], steps) for i in plan["small"])
    return per + small


def all_ranks_ok(torch, dist, device, flag):
    """True when `flag` holds on every rank (one all-reduce of the minimum),
    so every rank takes the same branch on an error path."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return bool(flag)
    t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def max_over_ranks(torch, dist, value, device):
    """Largest value over all ranks (timing is reported as the slowest rank)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def make_inputs(torch, workload, device, rank):
    config, shapes_fn, gdt, _ = WORKLOADS[workload]
    shapes = shapes_fn()
    gdtype = torch.bfloat16 if gdt == "bf16" else torch.float32
    params, grads, moms = [], [], []
    for i, (m, n) in enumerate(shapes):
        seed = W.seed_for(config, i // 7, i % 7) + 7919 * rank
        grads.append(W.gradient_gpu(config, m, n, seed, device, gdtype))
        params.append(W.param_gpu(m, n, seed, device))
        moms.append(torch.zeros((m, n), dtype=torch.float32, device=device))
    torch.cuda.synchronize()
    return shapes, params, grads, moms, gdtype


def run_ours(args):
    import torch
    import torch.distributed as dist
    import muon_newton_schulz_03_b200 as muon

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()

    shapes, params, grads, moms, gdtype = make_inputs(torch, args.workload, device, rank)
    count = len(shapes)
    gram = args.ns_algorithm == "gram"
    nominal = W.total_ns_flops(shapes, NS_STEPS, gram)
    algorithmic = W.total_ns_flops_symmetric(shapes, NS_STEPS, gram)
    gbytes = 2 if gdtype == torch.bfloat16 else 4
    k1_bytes = sum(W.step_bytes(m, n, gbytes)[0] for m, n in shapes)
    k4_bytes = sum(W.step_bytes(m, n, gbytes)[1] for m, n in shapes)

    opt = muon.Muon(device=local, cta_pair=args.cta_pair, ns_algorithm=args.ns_algorithm)
    stream = torch.cuda.current_stream()
    stepper = opt
    if args.layerwise:
        # One matrix set for the whole job: each rank updates the matrices it
        # owns and broadcasts them (layer-wise distributed Muon).
        from muon_newton_schulz_03_b200.distributed import LayerwiseMuon
        if world == 1:
            dist.init_process_group("nccl", init_method="tcp://127.0.0.1:29511", rank=0, world_size=1,
                                    device_id=device)
        stepper = LayerwiseMuon(opt)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        stepper.step(params, grads, moms, lr=LR, beta=BETA, wd=WD, ns_steps=NS_STEPS)
    torch.cuda.synchronize()
    code, ew, nf = opt.status()
    if not all_ranks_ok(torch, dist, device, code == 0):
        raise RuntimeError(f"device status {code} after warm-up on this or another rank (error word {ew}, "
                           f"non-finite {nf})")
    launches_per_step = opt.last_launch_count()

    opt.profile_enable(args.steps)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            stepper.step(params, grads, moms, lr=LR, beta=BETA, wd=WD, ns_steps=NS_STEPS)
        end.record(stream)
        torch.cuda.synchronize()
    barrier()
    elapsed_ms = start.elapsed_time(end)
    prof = opt.profile_read()
    opt.profile_enable(0)
    code, ew, nf = opt.status()
    if not all_ranks_ok(torch, dist, device, code == 0):
        raise RuntimeError(f"device status {code} after timing on this or another rank (error word {ew}, "
                           f"non-finite {nf})")

    ms_step = max_over_ranks(torch, dist, elapsed_ms / args.steps, device)

    # The same step captured once in a CUDA graph and replayed (no host work
    # per step: launch overhead and host-side checks drop out).
    graph_ms = None
    if not args.layerwise and not args.no_graph:
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            opt.step(params, grads, moms, lr=LR, beta=BETA, wd=WD, ns_steps=NS_STEPS)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            opt.step(params, grads, moms, lr=LR, beta=BETA, wd=WD, ns_steps=NS_STEPS)
        for _ in range(2):
            graph.replay()
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(args.steps):
            graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
        graph_ms = max_over_ranks(torch, dist, start.elapsed_time(end) / args.steps, device)
        del graph
        code, ew, nf = opt.status()
        if not all_ranks_ok(torch, dist, device, code == 0):
            raise RuntimeError(f"device status {code} after graph replay on this or another rank (error word {ew}, "
                               f"non-finite {nf})")

    by_kind = {}
    for kind, ms in prof:
        by_kind.setdefault(kind, []).append(ms)
    ns_ms = sum(sum(by_kind.get(k, [])) for k in ("ns_gram", "ns_poly", "ns_comb", "ns_sym")) / args.steps
    ns_launches = sum(len(by_kind.get(k, [])) for k in ("ns_gram", "ns_poly", "ns_comb", "ns_sym"))
    k1_ms = statistics.mean(by_kind["momentum_norm"]) if by_kind.get("momentum_norm") else None
    k4_ms = statistics.mean(by_kind["apply"]) if by_kind.get("apply") else None
    ns_tflops = nominal / (ns_ms * 1e-3) / 1e12 if ns_ms > 0 else None
    ns_tflops_alg = algorithmic / (ns_ms * 1e-3) / 1e12 if ns_ms > 0 else None
    executed = executed_flops(shapes, NS_STEPS, gram, args.cta_pair)
    ns_tflops_exec = executed / (ns_ms * 1e-3) / 1e12 if ns_ms > 0 else None
    avg_ns_launch_ms = ns_ms * args.steps / ns_launches if ns_launches else None
    per_launch_flops = algorithmic * args.steps / ns_launches if ns_launches else None

    clocks = clk.summary()

    # e2e: the same step through the host-buffer entry point (params, grads
    # and momenta in pinned host memory; copies inside the timed region).
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(torch, muon, opt, shapes, params, grads, moms, args, device, world, dist)

    opt.close()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload)

    if rank == 0:
        value = (1 if args.layerwise else world) * 1e3 / ms_step
        # The committed captures are of the single-CTA kernel, standard form.
        traffic = None if (gram or args.cta_pair) else profiled_traffic(args.workload)
        peak_tf, peak_note = tensor_peak(peaks, peak_src, ms_step * args.steps)
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "steps/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "strong" if args.layerwise else "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {
                "workload": WORKLOADS[args.workload][3],
                "matrices": count,
                "elements": W.total_elements(shapes),
                "grad_dtype": "bf16" if gdtype == torch.bfloat16 else "fp32",
                "param_dtype": "fp32",
                "ns_steps": NS_STEPS,
                "lr": LR, "beta": BETA, "nesterov": True, "wd": WD, "scale": "moonlight 0.2*sqrt(max(m,n))",
                "l2": "inputs larger than L2 (params, momenta, grads resident in HBM, no flush needed)",
                "parallelism": (f"layer-wise ownership over {world} GPUs + broadcast (strong)" if args.layerwise
                                else f"replica per GPU x{world} (weak)"),
                "ns_tiles": "256x256 CTA pair (cta_group::2)" if args.cta_pair else "128x256 single CTA",
                "ns_algorithm": ("Gram form, segments of 2 steps" if gram else "standard"),
            },
            "ns_tflops_nominal": ns_tflops,
            "ns_frac_of_datasheet_bf16": (ns_tflops / DATASHEET_BF16_TFLOPS) if ns_tflops else None,
            "ns_frac_of_measured_bf16": (ns_tflops / peak_tf) if ns_tflops else None,
            "matrices_per_s": count * value,
            "ns_ms_per_step": ns_ms,
            "elementwise": {
                "momentum_norm_ms": k1_ms, "momentum_norm_gbs": (k1_bytes / (k1_ms * 1e-3) / 1e9) if k1_ms else None,
                "apply_ms": k4_ms, "apply_gbs": (k4_bytes / (k4_ms * 1e-3) / 1e9) if k4_ms else None,
                # no apply kernel ran: the last combine wrote p' itself
                "apply_fused": k4_ms is None,
                "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src,
            },
            "roofline": {
                "kernel": "ns_phase_kernel (tcgen05 Newton-Schulz phases, all matrices per launch)",
                "bound": "tensor",
                "achieved": ns_tflops_alg,
                "peak": peak_tf,
                "unit": "TFLOP/s",
                "frac": (ns_tflops_alg / peak_tf) if ns_tflops_alg else None,
                "traffic": traffic,
                "peak_source": peak_note,
                "flops_per_launch": per_launch_flops,
                "achieved_nominal": ns_tflops,
                "achieved_executed": ns_tflops_exec,
                "frac_executed": (ns_tflops_exec / peak_tf) if ns_tflops_exec else None,
                "executed_definition": "tile FLOPs the tensor cores run: listed tiles x BM x 256 x K (K padded "
                                       "to 64); symmetric phases list upper tiles only",
                "avg_launch_ms": avg_ns_launch_ms,
                "flops_definition": ("the method's own work, symmetric products on one triangle: Gram form "
                                     "3 s^2 l + 5 s^3 per two-step segment, 3 s^2 l + s^3 per one-step segment"
                                     if gram else "the method's own work: 3 s^2 l + s^3 per matrix per iteration "
                                     "(Gram and polynomial symmetric, one triangle; combine 2 s^2 l)"),
                "nominal_definition": ("nominal 4 s^2 l + 2 s^3 per matrix per iteration, the dense count of the "
                                       "north-star gate (achieved_nominal; ns_frac_of_datasheet_bf16)"),
            },
            "graph": ({"ms_per_step": graph_ms, "value": (1 if args.layerwise else world) * 1e3 / graph_ms,
                       "unit": "steps/s", "note": "one step captured in a CUDA graph, replayed"}
                      if graph_ms else None),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_e2e(torch, muon, opt, shapes, params, grads, moms, args, device, world, dist):
    """Steps/s through muon_step_host with host buffers (copies included)."""
    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    def all_ok(flag):
        # Every rank takes the same path: the decision is the minimum over ranks.
        if world == 1:
            return bool(flag)
        t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MIN)
        return bool(t.item())

    # The host copies of every rank on this node must fit in host memory with
    # room to spare; otherwise no rank runs this leg.
    need = sum(t.numel() * t.element_size() for t in list(params) + list(grads) + list(moms))
    local_ranks = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:  # pragma: no cover - psutil missing
        avail = 0
    if not all_ok(need * local_ranks <= 0.8 * avail):
        return {"value": None, "unit": "steps/s",
                "error": f"host memory: {local_ranks} ranks x {need / 1e9:.1f} GB of pinned buffers would not fit"}
    hp, hg, hm, err = [], [], [], None
    try:
        hp = [pinned_copy(p) for p in params]
        hg = [pinned_copy(g) for g in grads]
        hm = [pinned_copy(m) for m in moms]
    except Exception as e:  # pragma: no cover - host memory limits
        err = str(e)
    if not all_ok(err is None):
        del hp, hg, hm
        return {"value": None, "unit": "steps/s", "error": f"pinned host buffers unavailable: {err or 'on another rank'}"}
    h2d = sum(t.numel() * t.element_size() for t in hp + hg + hm)
    d2h = sum(t.numel() * t.element_size() for t in hp + hm)
    # Free the device-resident copies so the staging area fits.
    del params[:], grads[:], moms[:]
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()
    steps = max(1, min(args.steps, args.e2e_steps))
    opt.step_host(hp, hg, hm, lr=LR, beta=BETA, wd=WD, ns_steps=NS_STEPS)   # warm: staging allocation
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        opt.step_host(hp, hg, hm, lr=LR, beta=BETA, wd=WD, ns_steps=NS_STEPS)
    end.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, dist, start.elapsed_time(end) / steps, device)
    code, ew, _ = opt.status()
    if not all_ok(code == 0):
        return {"value": None, "unit": "steps/s", "error": f"device status {code} on this or another rank"}
    return {"value": world * 1e3 / ms, "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms, "steps": steps,
            "path": "muon_step_host: params, grads, momenta in pinned host memory; up to 32 chunks pipelined over "
                    "copy-in, compute and copy-out streams; the caller's stream waits for the last copy-out"}


def run_sweep(args):
    """NS-only sweep: bf16 X with log-uniform singular values in [1e-4, 1],
    five steps, every (m, n, batch) point of the sweep; one JSON line whose
    `sweep` list holds nominal NS TFLOP/s per point."""
    import torch
    import muon_newton_schulz_03_b200 as muon
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()
    batches = set(int(b) for b in args.sweep_batches.split(","))
    opt = muon.Muon(device=device.index, cta_pair=args.cta_pair)
    points = []
    for (m, n, batch) in W.sweep_points():
        if batch not in batches:
            continue
        base = W.gradient_gpu(W.CONFIG_SWEEP, m, n, W.seed_for(W.CONFIG_SWEEP, m, n), device, torch.bfloat16)
        ld = muon.round_up(n, 8)
        xin = []
        for b in range(batch):
            buf = torch.zeros((m, ld), dtype=torch.bfloat16, device=device)
            buf[:, :n] = base if b % 2 == 0 else -base
            xin.append(buf)
        del base
        xout = [torch.empty((m, ld), dtype=torch.bfloat16, device=device) for _ in range(batch)]
        shapes = [(m, n)] * batch
        opt.newton_schulz(xin, xout, shapes, None, ns_steps=NS_STEPS)        # plan, workspace, maps
        torch.cuda.synchronize()
        reps = 3
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(reps):
            opt.newton_schulz(xin, xout, shapes, None, ns_steps=NS_STEPS)
        end.record()
        torch.cuda.synchronize()
        ms_eager = start.elapsed_time(end) / reps
        # The same call captured in a CUDA graph: the device time without the
        # per-call host work (argument checks and marshalling of `batch`
        # tensors), which dominates the eager time of small batched points.
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            opt.newton_schulz(xin, xout, shapes, None, ns_steps=NS_STEPS)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            opt.newton_schulz(xin, xout, shapes, None, ns_steps=NS_STEPS)
        graph.replay()
        torch.cuda.synchronize()
        # About 100 ms of replays (3 to 50): a short point's replays then
        # queue back to back, and the first one's launch latency does not
        # weigh on its mean.
        greps = max(3, min(50, int(100.0 / max(ms_eager, 1e-3))))
        start.record()
        for _ in range(greps):
            graph.replay()
        end.record()
        torch.cuda.synchronize()
        ms = start.elapsed_time(end) / greps
        del graph
        flops = batch * W.ns_flops(m, n, NS_STEPS)
        tf = flops / (ms * 1e-3) / 1e12
        points.append({"m": m, "n": n, "batch": batch, "ms": ms, "ms_eager": ms_eager, "replays": greps, "tflops_nominal": tf,
                       "frac_datasheet": tf / DATASHEET_BF16_TFLOPS, "frac_measured": tf / peaks["bf16_tflops"]})
        del xin, xout
        torch.cuda.empty_cache()
    code, ew, _ = opt.status()
    opt.close()
    if code != 0:
        raise RuntimeError(f"device status {code} (error word {ew})")
    vals = sorted(p["tflops_nominal"] for p in points)
    line = {"metric": "NS-only TFLOP/s (nominal 5 (4 s^2 l + 2 s^3)) per sweep point", "value": vals[len(vals) // 2],
            "unit": "TFLOP/s (median over points)", "n_gpus": 1, "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": W.describe(W.CONFIG_SWEEP), "ns_steps": NS_STEPS,
                                            "timing": "CUDA-graph replay of the call (ms); eager call (ms_eager)",
                                            "batches": sorted(batches), "peak_source": peak_src},
            "sweep": points}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["sweep"], default="llama3")
    ap.add_argument("--sweep-batches", default="1,4,16,64,256")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--layerwise", action="store_true",
                    help="one matrix set per job, whole matrices owned by ranks, broadcast after the update")
    ap.add_argument("--cta-pair", action="store_true",
                    help="tiled phases on CTA pairs (256 x 256 tiles, cta_group::2) instead of single CTAs")
    ap.add_argument("--ns-algorithm", choices=["standard", "gram"], default="standard",
                    help="form of the Newton-Schulz iteration (the Gram form iterates on the s x s Gram)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)   # at least three untimed steps
    if args.workload == "sweep":
        return run_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
