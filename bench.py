#!/usr/bin/env python
"""SparseGPT per-layer prune time and weights/s on B200.

One step prunes the OPT-125M-shaped layer (W 768 x 768 fp32, X 262,144 x 768
bf16 = 128 sequences x 2,048 tokens) twice from its activations, once 2:4 and
once unstructured at 50%: each run is a full layer prune through the C ABI
(Hessian accumulation, damping and factorisation, blocked OBS sweep, and for
2:4 the packing). Inputs are resident in HBM; W is restored and L2 is flushed
between steps (untimed). Device time per step comes from CUDA events on the
launching stream; with N GPUs every rank prunes its own replica and the
slowest rank's time counts (weak scaling, no collectives on the data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SparseGPT per-layer prune time & weights/s on 1 B200; % of HBM/tensor roofline"
UNIT = "weights/s"
CONFIG = "opt125m_768"
WORKLOADS = {
    "layer256": "256x256 layer, 2048 tokens, 2:4",
    "llama7b_down": ("Llama-7B MLP down-proj: W 4096x11008 fp32, X 131072x11008 bf16 (lognormal sigma=1.5, "
                     "0.5% outlier channels x50), 2:4"),
    "llama7b_q": ("Llama-7B q_proj: W 4096x4096 fp32, X 262144x4096 bf16, unstructured 50/70/80% "
                  "(three layer prunes per step)"),
    "profile_4096": "4096x4096 layer, 32768 tokens, 2:4 (profiler captures)",
    "qwen3_32b_block": ("Qwen3-32B-shaped block: q 5120->8192, k/v 5120->1024, o 8192->5120, gate/up "
                        "5120->25600, down 25600->5120, 131072 tokens, 2:4; H and U shared by q/k/v and by "
                        "gate/up (4 Hessians, 7 sweeps per step)"),
}
WORKLOAD = ("OPT-125M-shaped linear layer: W 768x768 fp32 ~N(0,1/768); X 262144x768 bf16 "
            "(128 seqs x 2048 tokens, lognormal(sigma=1) channel scales, 1% outlier channels x20); "
            "two layer prunes per step from X: 2:4 and unstructured 50%; blocksize 128; damp 0.01")
WORKLOADS[CONFIG] = WORKLOAD


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config", default=CONFIG, help="workload (default: the OPT-125M-shaped layer)")
    return ap.parse_args()


# DRAM bytes (read + write) of one hessian_tc_kernel launch, from the ncu
# capture summarised in profiles/hessian_tc_kernel_opt125m_768.md; re-capture
# when the kernel changes.
HESSIAN_TRAFFIC = {"opt125m_768": 407.6e6}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks during the timed region."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        props = torch.cuda.get_device_properties(device_index)
        self.bus = None
        try:
            self.bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        except AttributeError:
            pass
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        if self.bus:
            mine = [r for r in rows if r[0].upper().endswith(self.bus[-12:].upper())]
            rows = mine or rows
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 4 + i and r[4 + i].strip() == "Active"})
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


# ------------------------------------------------------------------ oracle

def cpu_baseline(spec, X_cpu, W_cpu, budget_tokens=32768):
    """The float64 oracle as it stands, on a bounded sample of the workload:
    the Hessian over the first `budget_tokens` tokens (time scaled to the full
    token count), damping, factorisation, sweep and packing in full, for
    both runs. Returns (weights/s, seconds, cores, sample description)."""
    import numpy as np

    import oracle
    from workloads import bf16_bits_to_f64

    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    n = spec.n_tok
    t_sample = min(budget_tokens, n)
    Xs = bf16_bits_to_f64(X_cpu[:t_sample]).numpy()
    W0 = W_cpu.numpy().astype(np.float64)
    total = 0.0
    for run in spec.runs:
        t0 = time.perf_counter()
        H = oracle.hessian(Xs)
        t_h = (time.perf_counter() - t0) * (n / t_sample)
        t0 = time.perf_counter()
        oracle.prune_layer(W0, H=H, pattern=run, blocksize=128, damp_ratio=0.01)
        total += t_h + (time.perf_counter() - t0)
    weights = spec.weights * len(spec.runs)
    sample = (f"per run: Hessian over {t_sample} of {n} tokens, time scaled x{n / t_sample:g}; "
              f"damping, factor, sweep and 2:4 pack in full; runs {list(spec.runs)}")
    return weights / total, total, cores, sample


def reference_arm(args, spec):
    """--impl reference: the oracle timed as it stands on the host cores."""
    import torch

    from workloads import gen_activations, gen_weights
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    X = gen_activations(spec, device="cpu", count=32768)
    W = gen_weights(spec)
    times = []
    cores = 1
    sample = ""
    for i in range(args.warmup + args.steps):
        v, t, cores, sample = cpu_baseline(spec, X, W, budget_tokens=8192)
        if i >= args.warmup:
            times.append(t)
    t = sum(times) / len(times)
    value = spec.weights * len(spec.runs) / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    del torch
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ranks

def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time: every rank contributes its own device time and
    all ranks receive the maximum (one all-reduce, outside the timed region)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(weights_per_rank_step: int, steps: int, world: int, t_slowest: float) -> dict:
    """Whole-job throughput of `world` replicas (weak scaling): all ranks'
    units over the slowest rank's time."""
    total = weights_per_rank_step * steps * world
    return {"value": total / t_slowest, "ms_per_step": t_slowest * 1e3 / steps}


# ------------------------------------------------------------------ native

def main():
    args = parse()
    from workloads import CONFIGS
    if args.impl == "reference":
        reference_arm(args, CONFIGS[CONFIG][0])
        return

    import torch
    import torch.distributed as dist

    import post_pruning_b200 as pp
    from workloads import gen_activations, gen_weights

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    stream = torch.cuda.current_stream()
    # A job is one activation input: its Hessian and factor are computed once,
    # then every weight matrix reading that input is swept (and 2:4 packed).
    # The OPT-125M workload prunes its layer twice from X (one job per run);
    # the Qwen3-32B block has four inputs shared by q/k/v, o, gate/up, down.
    jobs = []
    specs = CONFIGS[args.config]
    if len(specs) == 1:
        sp = specs[0]
        X = gen_activations(sp, device=dev)
        for run in sp.runs:
            jobs.append((sp, X, [(sp, pp.Params(run))]))
    else:
        by_x = {}
        for sp in specs:
            by_x.setdefault(sp.x_key, []).append(sp)
        for key, group in by_x.items():
            X = gen_activations(group[0], device=dev)
            jobs.append((group[0], X, [(sp, pp.Params(sp.runs[0])) for sp in group]))
    layers = []      # (W0, W, LayerGraphs)
    job_graphs = []
    for xs, X, mats in jobs:
        first = None
        gl = []
        for sp, p in mats:
            W0 = gen_weights(sp, device=dev)
            W = W0.clone()
            if first is None:
                b = pp.LayerBuffers.allocate(sp.d_out, sp.d_in, xs.n_tok, dev)
                g = pp.LayerGraphs(b, W, X, p)
                first = b
            else:
                b = pp.LayerBuffers.sharing(first, sp.d_out, dev)
                g = pp.LayerGraphs(b, W, None, p, phases=("prune", "pack"))
            layers.append((W0, W, g))
            gl.append(g)
        job_graphs.append(gl)
    weights_per_step = sum(sp.weights for _, _, mats in jobs for sp, _ in mats)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    PH = pp.LayerGraphs.PHASES

    def one_step(ev=None):
        # ev[j][phase] pairs of events around every graph of job j
        for j, gl in enumerate(job_graphs):
            for g in gl:
                for name in g.phases:
                    if ev is not None:
                        ev[j][name][0].record(stream)
                    g.graphs[name].replay()
                    if ev is not None:
                        ev[j][name][1].record(stream)

    def prep():
        for W0, W, _ in layers:
            W.copy_(W0)
        flush.zero_()

    for _ in range(args.warmup):
        prep()
        one_step()
    torch.cuda.synchronize()
    for _, _, g in layers:
        pp.raise_on_info(g.bufs.info, where="warm-up")

    def mk():
        return (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    # one event pair per (job, phase); graphs of the same phase in a job share it
    evs = [[{name: mk() for name in PH} for _ in job_graphs] for _ in range(args.steps)]
    step_ev = [mk() for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)               # let the sampler produce its first line
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = pp.kernel_launches()
    wall0 = time.perf_counter()
    phase = {name: 0.0 for name in PH}
    for s_ in range(args.steps):
        prep()
        step_ev[s_][0].record(stream)
        for j, gl in enumerate(job_graphs):
            for name in PH:
                e0, e1 = evs[s_][j][name]
                ran = False
                for g in gl:
                    if name in g.graphs:
                        if not ran:
                            e0.record(stream)
                            ran = True
                        g.graphs[name].replay()
                if ran:
                    e1.record(stream)
        step_ev[s_][1].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    launches = pp.kernel_launches() - launches0 + args.steps * sum(sum(g.kernels.values()) for _, _, g in layers)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    for _, _, g in layers:
        pp.raise_on_info(g.bufs.info, where="timed steps")

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    for s_ in range(args.steps):
        for j, gl in enumerate(job_graphs):
            for name in PH:
                if any(name in g.graphs for g in gl):
                    e0, e1 = evs[s_][j][name]
                    phase[name] += e0.elapsed_time(e1)
    phase = {k: v / args.steps for k, v in phase.items()}
    t_rank = max_over_ranks(sum(step_ms) / 1e3, dist if world > 1 else None, dev)
    agg = aggregate(weights_per_step, args.steps, world, t_rank)
    value, ms_per_step = agg["value"], agg["ms_per_step"]
    spec = jobs[0][0]
    n_hess = len(jobs)
    n, d = spec.n_tok, spec.d_in

    # roofline of the dominant kernel: the tensor-core Hessian (one launch per job)
    hbm, bf16_burst, bf16_sust, peak_kind = peaks()
    hess_flops = sum(xs.n_tok * xs.d_in * (xs.d_in + 1) for xs, _, _ in jobs)
    achieved = hess_flops / (phase["hessian"] * 1e-3) / 1e12
    roofline = {"kernel": "hessian_tc_kernel", "bound": "tensor", "achieved": achieved,
                "peak": bf16_burst, "unit": "TFLOP/s", "frac": achieved / bf16_burst,
                "traffic": HESSIAN_TRAFFIC.get(args.config), "traffic_unit": "bytes per launch",
                "peak_kind": f"{peak_kind} bf16 burst",
                "work": f"n*d*(d+1) = {hess_flops / n_hess:.4g} flop per launch (upper triangle incl. "
                        f"diagonal), {n_hess} launches per step"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "input_dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOADS.get(args.config, args.config), "name": args.config,
                   "weights_per_step": weights_per_step,
                   "launch": "each phase of each layer replayed as a captured CUDA graph",
                   "l2": "flushed between steps (256 MiB write, untimed); every X exceeds the 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "phases_ms_per_step": phase,
        "roofline": roofline,
        "gpu_launches": launches,
        "clocks": clk,
        "wall_s_timed": wall,
    }

    # end to end through the public API with host buffers (rank-local), for
    # workloads whose layers each read their own input
    single = all(len(m) == 1 for _, _, m in jobs)
    if not args.no_e2e and single:
        hp = [(pp.HostPruner(sp.d_out, sp.d_in, xs.n_tok, dev), p, xs, sp) for xs, _, ((sp, p),) in jobs]
        X_host = {id(X): X.cpu().pin_memory() for _, X, _ in jobs}
        W_host = [layers[k][0].cpu().pin_memory() for k in range(len(layers))]
        xs_of = [X for _, X, _ in jobs]

        # Each distinct input is copied from the host once per step, into one
        # of two device buffers on a copy stream, while the previous step's
        # prunes run on the compute stream from the other buffer; the layers
        # that read the same input prune from that copy.
        keys = list({id(X): X for X in xs_of}.keys())
        xbuf = {key: [torch.empty_like(X_host[key], device=dev) for _ in range(2)] for key in keys}
        copy_s, comp_s = torch.cuda.Stream(), torch.cuda.Stream()
        ready = [torch.cuda.Event() for _ in range(2)]
        free = [torch.cuda.Event() for _ in range(2)]
        step_no = [0]

        def e2e_step():
            b = step_no[0] & 1
            step_no[0] += 1
            with torch.cuda.stream(copy_s):
                copy_s.wait_event(free[b])          # the step two back is done with this buffer
                for key in keys:
                    xbuf[key][b].copy_(X_host[key], non_blocking=True)
                ready[b].record(copy_s)
            with torch.cuda.stream(comp_s):
                comp_s.wait_event(ready[b])
                for k, (h, p, xs, sp) in enumerate(hp):
                    h.enqueue(W_host[k], None, p, X_device=xbuf[id(xs_of[k])][b])
                free[b].record(comp_s)

        for _ in range(max(1, args.warmup // 2)):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ks = max(1, args.steps // 2)
        e0.record(copy_s)
        comp_s.wait_event(e0)
        for _ in range(ks):
            e2e_step()
        e1.record(comp_s)
        torch.cuda.synchronize()
        for h, _, _, _ in hp:
            pp.raise_on_info(h.bufs.info, where="e2e")
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist if world > 1 else None, dev)
        x_bytes = sum(X.numel() * X.element_size() for X in {id(X): X for X in xs_of}.values())
        line["e2e"] = {"value": weights_per_step * ks * world / t_e2e, "unit": UNIT,
                       "h2d_bytes_per_step": x_bytes + sum(h.W.numel() * 4 for h, _, _, _ in hp),
                       "d2h_bytes_per_step": sum(h.d2h_bytes(p) for h, p, _, _ in hp),
                       "ms_per_step": t_e2e * 1e3 / ks,
                       "note": ("every step copies each distinct X and every W from pinned host memory "
                                "and each layer's results back; the next step's X copy overlaps this "
                                "step's pruning (two device buffers)")}

    if rank == 0 and world == 1 and not args.no_cpu_baseline and len(specs) == 1:
        v, t, cores, sample = cpu_baseline(spec, jobs[0][1][:32768].cpu(), layers[0][0].cpu())
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": sample, "seconds": t}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
