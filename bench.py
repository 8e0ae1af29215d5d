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
WORKLOAD = ("OPT-125M-shaped linear layer: W 768x768 fp32 ~N(0,1/768); X 262144x768 bf16 "
            "(128 seqs x 2048 tokens, lognormal(sigma=1) channel scales, 1% outlier channels x20); "
            "two layer prunes per step from X: 2:4 and unstructured 50%; blocksize 128; damp 0.01")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


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
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"],
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


# ------------------------------------------------------------------ native

def main():
    args = parse()
    from workloads import CONFIGS
    spec = CONFIGS[CONFIG][0]
    if args.impl == "reference":
        reference_arm(args, spec)
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
    X = gen_activations(spec, device=dev)
    W0 = gen_weights(spec, device=dev)
    runs = [pp.Params(r) for r in spec.runs]
    r, d, n = spec.d_out, spec.d_in, spec.n_tok
    bufs = [pp.LayerBuffers.allocate(r, d, n, dev) for _ in runs]
    Ws = [W0.clone() for _ in runs]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def one_step(ev=None):
        for k, (p, b, W) in enumerate(zip(runs, bufs, Ws)):
            info = b.info
            pp.info_clear(info)
            if ev is not None:
                ev[k][0].record(stream)
            pp.hessian_zero(b.H)
            pp.hessian_accumulate(b.H, X, b.ws, info)
            if ev is not None:
                ev[k][1].record(stream)
            pp.factor(b.H, n, p.damp, b.U, b.ws, info)
            if ev is not None:
                ev[k][2].record(stream)
            b.row_loss.zero_()
            pp.prune(W, b.U, p, b.mask, b.ws, info, row_loss=b.row_loss)
            if ev is not None:
                ev[k][3].record(stream)
            if p.is_nm:
                pp.pack24(W, b.mask, b.values, b.meta, info)
            if ev is not None:
                ev[k][4].record(stream)

    def prep():
        for W in Ws:
            W.copy_(W0)
        flush.zero_()

    for _ in range(args.warmup):
        prep()
        one_step()
    torch.cuda.synchronize()
    for b in bufs:
        pp.raise_on_info(b.info, where="warm-up")

    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in runs] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = pp.kernel_launches()
    wall0 = time.perf_counter()
    for s in range(args.steps):
        prep()
        one_step(evs[s])
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    launches = pp.kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    for b in bufs:
        pp.raise_on_info(b.info, where="timed steps")

    # per-step device time and phase breakdown
    step_ms = [sum(e[k][0].elapsed_time(e[k][4]) for k in range(len(runs))) for e in evs]
    phase = {"hessian": 0.0, "factor": 0.0, "sweep": 0.0, "pack": 0.0}
    names = list(phase)
    for e in evs:
        for k in range(len(runs)):
            for j, nm in enumerate(names):
                phase[nm] += e[k][j].elapsed_time(e[k][j + 1])
    phase = {k: v / args.steps for k, v in phase.items()}
    t_rank = sum(step_ms) / 1e3
    if world > 1:
        t = torch.tensor([t_rank], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        t_rank = float(t.item())
    weights = spec.weights * len(runs) * args.steps * world
    value = weights / t_rank
    ms_per_step = t_rank * 1e3 / args.steps

    # roofline of the dominant kernel: the tensor-core Hessian (one launch per run)
    hbm, bf16_burst, bf16_sust, peak_kind = peaks()
    hess_ms = phase["hessian"] / len(runs)
    hess_flops = n * d * (d + 1)            # the symmetric half X^T X needs
    achieved = hess_flops / (hess_ms * 1e-3) / 1e12
    roofline = {"kernel": "hessian_tc_kernel", "bound": "tensor", "achieved": achieved,
                "peak": bf16_burst, "unit": "TFLOP/s", "frac": achieved / bf16_burst,
                "traffic": None, "peak_kind": f"{peak_kind} bf16 burst",
                "work": f"n*d*(d+1) = {hess_flops:.4g} flop per launch (upper triangle incl. diagonal)"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "input_dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "per_gpu_layers_per_step": len(runs),
                   "l2": "flushed between steps (256 MiB write, untimed); X is 403 MB > 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "per_layer_ms": {p.pattern: sum(e[k][0].elapsed_time(e[k][4]) for e in evs) / args.steps
                         for k, p in enumerate(runs)},
        "phases_ms_per_step": phase,
        "roofline": roofline,
        "gpu_launches": launches,
        "clocks": clk,
        "wall_s_timed": wall,
    }

    # end to end through the public API with host buffers (rank-local)
    if not args.no_e2e:
        hp = [pp.HostPruner(r, d, n, dev) for _ in runs]
        X_host = X.cpu().pin_memory()
        W_host = W0.cpu().pin_memory()
        for _ in range(max(1, args.warmup // 2)):
            for p, h in zip(runs, hp):
                h.enqueue(W_host, X_host, p)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ks = max(1, args.steps // 2)
        e0.record(stream)
        for _ in range(ks):
            for p, h in zip(runs, hp):
                h.enqueue(W_host, X_host, p)
        e1.record(stream)
        torch.cuda.synchronize()
        for h in hp:
            pp.raise_on_info(h.bufs.info, where="e2e")
        t_e2e = e0.elapsed_time(e1) / 1e3
        if world > 1:
            t = torch.tensor([t_e2e], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            t_e2e = float(t.item())
        line["e2e"] = {"value": spec.weights * len(runs) * ks * world / t_e2e, "unit": UNIT,
                       "h2d_bytes_per_step": sum(h.h2d_bytes() for h in hp),
                       "d2h_bytes_per_step": sum(h.d2h_bytes(p) for h, p in zip(hp, runs)),
                       "ms_per_step": t_e2e * 1e3 / ks,
                       "note": "each run copies W and X from pinned host memory and its results back"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, t, cores, sample = cpu_baseline(spec, X[:32768].cpu(), W0.cpu())
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": sample, "seconds": t}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
