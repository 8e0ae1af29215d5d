#!/usr/bin/env python
"""SparseGPT per-layer prune time and weights/s on B200.

Default workload: one Qwen3-32B-shaped decoder block, 131,072 calibration
tokens, every linear layer pruned 2:4 from its activations. One step prunes
all seven matrices (q 5120->8192, k/v 5120->1024, o 8192->5120, gate/up
5120->25600, down 25600->5120; 487,587,840 weights): for each of the four
distinct inputs the Hessian H = X^T X and the damped factorisation run once,
then every matrix that reads that input is swept (blocked OBS, 2:4 masks on
the compensated weights, lazy trailing updates) and packed (values + 2-bit
metadata), all through the C ABI. Inputs are resident in HBM (11.5 GB of
bf16 activations, far above the 126 MB L2); W is restored and L2 flushed
between steps (untimed). Device time per step comes from CUDA events on the
launching stream; with N GPUs every rank prunes its own replica and the
slowest rank's time counts (weak scaling, no collectives on the data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--config qwen3_32b_block|opt125m_768|llama7b_down|llama7b_q|...]

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
CONFIG = "qwen3_32b_block"
WORKLOADS = {
    "layer256": "256x256 layer, 2048 tokens, 2:4",
    "opt125m_768": ("OPT-125M-shaped linear layer: W 768x768 fp32 ~N(0,1/768); X 262144x768 bf16 "
                    "(128 seqs x 2048 tokens, lognormal(sigma=1) channel scales, 1% outlier channels x20); "
                    "two layer prunes per step from X: 2:4 and unstructured 50%; blocksize 128; damp 0.01"),
    "llama7b_down": ("Llama-7B MLP down-proj: W 4096x11008 fp32, X 131072x11008 bf16 (lognormal sigma=1.5, "
                     "0.5% outlier channels x50), 2:4"),
    "llama7b_q": ("Llama-7B q_proj: W 4096x4096 fp32, X 262144x4096 bf16, unstructured 50/70/80% "
                  "(three layer prunes per step)"),
    "profile_4096": "4096x4096 layer, 32768 tokens, 2:4 (profiler captures)",
    "qwen3_32b_block": ("Qwen3-32B-shaped decoder block, 2:4 along d_in: q 5120->8192, k/v 5120->1024, "
                        "o 8192->5120, gate/up 5120->25600, down 25600->5120 (487,587,840 weights); "
                        "X 131072 tokens per distinct input, bf16, lognormal(sigma=1) channel scales with 1% "
                        "outlier channels x20, independent draws for the attention, o, MLP and down inputs; "
                        "W fp32 ~N(0,1/d_in); H and U computed once for q/k/v and once for gate/up "
                        "(4 Hessians + 4 factorisations + 7 sweeps and 2:4 packs per step); blocksize 128; "
                        "damp 0.01"),
}

# Oracle sample (cpu_baseline and the reference arm): per distinct input the
# first SAMPLE_TOKENS tokens of its leading SAMPLE_D channels; the Hessian of
# that slice, its damped factorisation, and the sweep and pack of SAMPLE_ROWS
# evenly spaced rows of each matrix over those channels. Each time is scaled
# to the full workload: Hessian x (n / tokens) x (d / SAMPLE_D)^2, factor x
# (d / SAMPLE_D)^3, sweep x (d_out / rows) x (d / SAMPLE_D). The sweep's
# scaling is linear in d although its trailing product grows as d^2, so the
# scaled oracle time is, if anything, too short for the wide layers.
SAMPLE_TOKENS = 512
SAMPLE_D = 3072
SAMPLE_ROWS = 8


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config", default=CONFIG, help="workload (default: the Qwen3-32B-shaped block)")
    ap.add_argument("--pattern", default=None,
                    help="prune every matrix with this pattern instead (e.g. 16:64, unstructured:0.5)")
    ap.add_argument("--qbits", type=int, default=0,
                    help="joint sparsification and quantization of the kept weights to this many bits")
    ap.add_argument("--driver", choices=["sequential", "parallel"], default="sequential",
                    help="mode of the multi-layer driver (config qwen3_32b_mlp_block)")
    ap.add_argument("--width", type=int, default=25600, help="d_in of configs hessian and factor")
    ap.add_argument("--tokens", type=int, default=131072, help="tokens of configs hessian and factor")
    return ap.parse_args()


# DRAM bytes (read + write) per step of each phase's kernels: the
# dram__bytes_read.sum + dram__bytes_write.sum of every launch of one step of
# the workload in one ncu capture, summed per phase; null for workloads and
# overrides without a capture.
TRAFFIC = {"qwen3_32b_block": {"hessian": 217.46e9, "factor": 160.14e9, "prune": 66.30e9, "pack": 2.87e9}}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained") or p["bf16_tflops"], "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# TF32 tensor rate over bf16 (nominal dense figures 1.1 and 2.25 PFLOP/s).
TF32_OVER_BF16 = 1.1 / 2.25


def group_by_input(specs):
    """{x_key: [specs reading that input]} in order of first appearance."""
    by_x = {}
    for sp in specs:
        by_x.setdefault(sp.x_key, []).append(sp)
    return by_x


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

def host_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def oracle_sample_inputs(specs):
    """What the oracle sample reads, generated on the host: the first
    SAMPLE_TOKENS tokens x SAMPLE_D channels of each distinct input and
    SAMPLE_ROWS evenly spaced rows (first SAMPLE_D columns) of every weight
    matrix, as float64."""
    from workloads import bf16_bits_to_f64, gen_activations, gen_weights
    xs, ws, rows = {}, {}, {}
    for key, group in group_by_input(specs).items():
        sp = group[0]
        X = gen_activations(sp, device="cpu", count=min(SAMPLE_TOKENS, sp.n_tok))
        xs[key] = bf16_bits_to_f64(X[:, :min(SAMPLE_D, sp.d_in)]).numpy()
    for sp in specs:
        step = max(1, sp.d_out // SAMPLE_ROWS)
        r = list(range(0, sp.d_out, step))[:SAMPLE_ROWS]
        rows[sp.name] = r
        ws[sp.name] = gen_weights(sp, rows=r)[:, :min(SAMPLE_D, sp.d_in)].numpy().astype("float64")
    return xs, ws, rows


def oracle_sample_time(specs, xs, ws, rows) -> float:
    """The float64 oracle, as it stands, on the bounded sample; returns the
    time scaled to one whole step of the workload (seconds)."""
    import oracle
    total = 0.0
    for key, group in group_by_input(specs).items():
        sp0 = group[0]
        n, d = sp0.n_tok, sp0.d_in
        X = xs[key]
        ds = X.shape[1]
        t0 = time.perf_counter()
        H = oracle.hessian(X)
        total += (time.perf_counter() - t0) * (n / X.shape[0]) * (d / ds) ** 2
        t0 = time.perf_counter()
        Hd, _ = oracle.damp(H, 0.01)
        U = oracle.inverse_cholesky_upper(Hd)
        total += (time.perf_counter() - t0) * (d / ds) ** 3
        for sp in group:
            for run in sp.runs:
                t0 = time.perf_counter()
                out = oracle.sweep(ws[sp.name], U, run, 128)
                if run == "2:4":
                    oracle.pack24(out["W"], out["mask"])
                total += (time.perf_counter() - t0) * (sp.d_out / len(rows[sp.name])) * (d / ds)
    return total


def oracle_sample_text(specs) -> str:
    return (f"per distinct input, its first {SAMPLE_TOKENS} tokens x first min(d, {SAMPLE_D}) channels: "
            f"Hessian (time x n_tok/{SAMPLE_TOKENS} x (d/{SAMPLE_D})^2), damping and factorisation "
            f"(time x (d/{SAMPLE_D})^3), and per matrix and run the sweep (+ 2:4 pack) of {SAMPLE_ROWS} evenly "
            f"spaced rows over those channels (time x d_out/{SAMPLE_ROWS} x d/{SAMPLE_D}, linear in d although "
            f"the trailing product grows as d^2); numpy float64, {len(specs)} matrices")


def cpu_baseline(specs, repeats=2):
    """The oracle timed on the host cores over the bounded sample."""
    xs, ws, rows = oracle_sample_inputs(specs)
    times = [oracle_sample_time(specs, xs, ws, rows) for _ in range(repeats)]
    t = sum(times) / len(times)
    weights = sum(sp.weights * len(sp.runs) for sp in specs)
    return weights / t, t, host_cores(), oracle_sample_text(specs) + f"; mean of {repeats} evaluations"


def reference_arm(args, specs, workload):
    """--impl reference: the oracle, as it stands, on the host cores. Each
    step times the bounded sample; ms_per_step is that measured time, value
    the whole workload's weights over the time scaled to it."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    xs, ws, rows = oracle_sample_inputs(specs)
    scaled, wall = [], []
    for i in range(args.warmup + args.steps):
        w0 = time.perf_counter()
        t = oracle_sample_time(specs, xs, ws, rows)
        if i >= args.warmup:
            scaled.append(t)
            wall.append(time.perf_counter() - w0)
    t_full = sum(scaled) / len(scaled)
    weights = sum(sp.weights * len(sp.runs) for sp in specs)
    value = weights / t_full
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(wall) / len(wall) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload, "name": args.config},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                         "sample": oracle_sample_text(specs),
                         "scaled_ms_per_step": t_full * 1e3,
                         "note": "ms_per_step is the measured time of one step's sample; value divides the "
                                 "whole workload's weights by the sample time scaled to it"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
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


# ------------------------------------------------------------------ rooflines

def phase_rooflines(jobs, phase_ms, sustained: bool, traffic=None) -> dict:
    """Achieved rate of each phase against its bound, from the algorithmic
    work of the phase (per step) and its measured time (per step).

    hessian  bf16 tensor: n*d*(d+1) flop per input (the upper triangle with
             the diagonal; symmetric tiles are what the kernel issues).
    factor   FP32-accurate products on tensor cores (three TF32 products per
             fp32 product): 2/3*d^3 flop per input (reverse Cholesky d^3/3 +
             triangular inverse d^3/3); peak = TF32 rate / 3.
    prune    sweep + selection + lazy trailing update: the larger of the
             sweep's 12*r*d HBM bytes (W in, W out, errors) and the trailing
             update's r*(d^2 - d*B) flop at the FP32-accurate rate.
    pack     HBM: 6.25 bytes per weight (W and mask in, values and metadata
             out).
    """
    hbm, bf16_burst, bf16_sust, kind = peaks()
    bf16 = bf16_sust if sustained else bf16_burst
    which = "sustained" if sustained else "burst"
    fp32acc = bf16 * TF32_OVER_BF16 / 3.0
    B = 128
    h_flops = sum(xs.n_tok * xs.d_in * (xs.d_in + 1) for xs, _, _ in jobs)
    f_flops = sum(2.0 / 3.0 * xs.d_in ** 3 for xs, _, _ in jobs)
    sweep_bytes = sum(12.0 * sp.d_out * sp.d_in for _, _, mats in jobs for sp, _ in mats)
    trail_flops = sum(float(sp.d_out) * (sp.d_in ** 2 - sp.d_in * B) for _, _, mats in jobs for sp, _ in mats)
    pack_bytes = sum(6.25 * sp.d_out * sp.d_in for _, _, mats in jobs for sp, p in mats
                     if p.is_nm and p.nm == (2, 4))
    out = {}

    def entry(name, bound, achieved, peak, unit, work, extra=None):
        e = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
             "frac": achieved / peak if peak else None, "traffic": (traffic or {}).get(name),
             "work_per_step": work}
        e.update(extra or {})
        out[name] = e

    t = phase_ms.get("hessian", 0.0) * 1e-3
    if t > 0:
        entry("hessian", "tensor", h_flops / t / 1e12, bf16, "TFLOP/s",
              f"{h_flops:.4g} flop (n*d*(d+1) per distinct input)",
              {"kernel": "hessian_tc_kernel", "peak_kind": f"{kind} bf16 {which}"})
    t = phase_ms.get("factor", 0.0) * 1e-3
    if t > 0:
        entry("factor", "tensor", f_flops / t / 1e12, fp32acc, "TFLOP/s",
              f"{f_flops:.4g} flop (2/3*d^3 per distinct input)",
              {"kernel": "gemm_tf32x3_kernel + diag_factor_kernel + chain_step_kernel",
               "peak_kind": f"{kind} bf16 {which} x {TF32_OVER_BF16:.3f} (TF32) / 3 (products per fp32 product)"})
    t = phase_ms.get("prune", 0.0) * 1e-3
    if t > 0:
        t_roof = max(sweep_bytes / (hbm * 1e9), trail_flops / (fp32acc * 1e12))
        entry("prune", "hbm+tensor", t_roof / t, 1.0, "fraction of roofline time",
              f"sweep {sweep_bytes:.4g} B; trailing {trail_flops:.4g} flop",
              {"kernel": "sweep_kernel + gemm_tf32x3_kernel (+ select_kernel)",
               "roofline_ms": t_roof * 1e3, "measured_ms": t * 1e3,
               "sweep_hbm_gbs": sweep_bytes / t / 1e9, "trailing_tflops": trail_flops / t / 1e12,
               "peak_kind": f"{kind} HBM {hbm} GB/s; FP32-accurate tensor {fp32acc:.4g} TFLOP/s"})
    t = phase_ms.get("pack", 0.0) * 1e-3
    if t > 0 and pack_bytes:
        entry("pack", "hbm", pack_bytes / t / 1e9, hbm, "GB/s", f"{pack_bytes:.4g} B (6.25 per weight)",
              {"kernel": "pack24_kernel", "peak_kind": f"{kind} HBM copy"})
    return out


# ------------------------------------------------------------------ native

def main():
    args = parse()
    from workloads import CONFIGS
    if args.config in EXTRA_BENCHES:
        EXTRA_BENCHES[args.config](args)
        return
    specs = CONFIGS[args.config]
    if args.pattern:
        specs = [sp.with_(runs=(args.pattern,)) for sp in specs]
    workload = WORKLOADS.get(args.config, args.config)
    if args.pattern or args.qbits:
        workload += f" [pattern {args.pattern or 'as listed'}, quantized to {args.qbits} bits]" if args.qbits else \
            f" [pattern {args.pattern}]"
    if args.impl == "reference":
        reference_arm(args, specs, workload)
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
    # A single-layer workload with several runs prunes its layer once per run
    # from X (one job per run).
    jobs = []
    if len(specs) == 1:
        sp = specs[0]
        X = gen_activations(sp, device=dev)
        for run in sp.runs:
            jobs.append((sp, X, [(sp, pp.Params(run, qbits=args.qbits))]))
    else:
        for key, group in group_by_input(specs).items():
            X = gen_activations(group[0], device=dev)
            jobs.append((group[0], X, [(sp, pp.Params(sp.runs[0], qbits=args.qbits)) for sp in group]))
    layers = []      # (W0, W, LayerGraphs, spec, params)
    job_graphs = []
    for xs, X, mats in jobs:
        first = None
        gl = []
        for sp, p in mats:
            W0 = gen_weights(sp, device=dev)
            W = W0.clone()
            if first is None:
                b = pp.LayerBuffers.allocate(sp.d_out, sp.d_in, xs.n_tok, dev, nm=p.nm if p.is_nm else (2, 4))
                g = pp.LayerGraphs(b, W, X, p)
                first = b
            else:
                b = pp.LayerBuffers.sharing(first, sp.d_out, dev, nm=p.nm if p.is_nm else (2, 4))
                g = pp.LayerGraphs(b, W, None, p, phases=("prune", "pack"))
            layers.append((W0, W, g, sp, p))
            gl.append(g)
        job_graphs.append(gl)
    weights_per_step = sum(sp.weights for _, _, mats in jobs for sp, _ in mats)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    PH = pp.LayerGraphs.PHASES

    def prep():
        for W0, W, _, _, _ in layers:
            W.copy_(W0)
        flush.zero_()

    def step_replay(evs_step=None, evs_mat=None):
        # evs_step[j][phase]: one event pair around all graphs of that phase of
        # job j; evs_mat[(j, m)][phase]: one pair around matrix m's graph
        for j, gl in enumerate(job_graphs):
            for name in PH:
                ran = False
                for m, g in enumerate(gl):
                    if name in g.graphs:
                        if evs_step is not None and not ran:
                            evs_step[j][name][0].record(stream)
                        ran = True
                        mev = evs_mat[(j, m)].get(name) if evs_mat is not None else None
                        if mev is not None:
                            mev[0].record(stream)
                        g.graphs[name].replay()
                        if mev is not None:
                            mev[1].record(stream)
                if ran and evs_step is not None:
                    evs_step[j][name][1].record(stream)

    for _ in range(args.warmup):
        prep()
        step_replay()
    torch.cuda.synchronize()
    for _, _, g, _, _ in layers:
        pp.raise_on_info(g.bufs.info, where="warm-up")

    def mk():
        return (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    evs = [[{name: mk() for name in PH} for _ in job_graphs] for _ in range(args.steps)]
    evs_mat = [{(j, m): {name: mk() for name in ("prune", "pack")} for j, gl in enumerate(job_graphs)
                for m in range(len(gl))} for _ in range(args.steps)]
    step_ev = [mk() for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)               # let the sampler produce its first line
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = pp.kernel_launches()
    wall0 = time.perf_counter()
    for s_ in range(args.steps):
        prep()
        step_ev[s_][0].record(stream)
        step_replay(evs[s_], evs_mat[s_])
        step_ev[s_][1].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    launches = pp.kernel_launches() - launches0 + args.steps * sum(sum(g.kernels.values()) for _, _, g, _, _ in layers)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    for _, _, g, _, _ in layers:
        pp.raise_on_info(g.bufs.info, where="timed steps")

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    phase = {name: 0.0 for name in PH}
    per_job = [{name: 0.0 for name in PH} for _ in job_graphs]
    for s_ in range(args.steps):
        for j, gl in enumerate(job_graphs):
            for name in PH:
                if any(name in g.graphs for g in gl):
                    e0, e1 = evs[s_][j][name]
                    ms = e0.elapsed_time(e1)
                    phase[name] += ms
                    per_job[j][name] += ms
    phase = {k: v / args.steps for k, v in phase.items()}
    per_job = [{k: v / args.steps for k, v in pj.items() if v} for pj in per_job]
    per_matrix = []
    for j, (xs, _, mats) in enumerate(jobs):
        for m, (sp, _) in enumerate(mats):
            g = job_graphs[j][m]
            row = {"matrix": sp.name, "d_out": sp.d_out, "d_in": sp.d_in}
            for name in ("prune", "pack"):
                if name in g.graphs:
                    row[f"{name}_ms"] = sum(evs_mat[s_][(j, m)][name][0].elapsed_time(evs_mat[s_][(j, m)][name][1])
                                            for s_ in range(args.steps)) / args.steps
            per_matrix.append(row)
    t_rank = max_over_ranks(sum(step_ms) / 1e3, dist if world > 1 else None, dev)
    agg = aggregate(weights_per_step, args.steps, world, t_rank)
    value, ms_per_step = agg["value"], agg["ms_per_step"]

    sustained = ms_per_step * args.steps > 2000.0     # seconds-long run: the power-capped peak applies
    roof = phase_rooflines([(xs, X, mats) for xs, X, mats in jobs], phase, sustained,
                           None if (args.pattern or args.qbits) else TRAFFIC.get(args.config))
    dominant = max(roof, key=lambda k: phase.get(k, 0.0))
    roofline = dict(roof[dominant])
    roofline["phase"] = dominant
    roofline["share_of_step"] = phase[dominant] / ms_per_step

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "input_dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload, "name": args.config,
                   "weights_per_step": weights_per_step,
                   "launch": "each phase of each layer replayed as a captured CUDA graph",
                   "l2": "flushed between steps (256 MiB write, untimed); every X exceeds the 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "phases_ms_per_step": phase,
        "phases_ms_per_input": [{"input": f"{xs.d_in}-wide ({', '.join(sp.name for sp, _ in mats)})", **pj}
                                for (xs, _, mats), pj in zip(jobs, per_job)],
        "phases_ms_per_matrix": per_matrix,
        "ms_per_step_median": statistics.median(step_ms),
        # the same step from H (the Hessian phase left out): factor, sweep, pack
        "from_H": {"value": weights_per_step * world / ((ms_per_step - phase["hessian"]) * 1e-3),
                   "unit": UNIT, "ms_per_step": ms_per_step - phase["hessian"]},
        "roofline": roofline,
        "rooflines": roof,
        "gpu_launches": launches,
        "clocks": clk,
        "wall_s_timed": wall,
    }

    # end to end through the public API with host buffers (rank-local): every
    # step copies each distinct X and every W from pinned host memory, prunes
    # each input's first matrix with sgpt_prune_layer (Hessian, factor,
    # sweep, pack) and the matrices sharing its H and U with sgpt_prune and
    # sgpt_pack_nm, and copies every pruned W, mask, value and metadata array
    # back into pinned host memory. Three streams: uploads (h2d), pruning
    # (comp) and downloads (d2h); step s+1's uploads and step s's downloads
    # overlap step s's pruning. Each W, mask and packed output has two device
    # buffers (steps alternate), so an upload never overwrites what a
    # download of the step before still reads.
    if not args.no_e2e:
        h2d_s, comp_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        distinct = {}                 # jobs that read the same X share one copy of it
        x_of_job = [distinct.setdefault(id(X), len(distinct)) for _, X, _ in jobs]
        X_dev = {id(X): X for _, X, _ in jobs}
        X_host = [X_dev[k].cpu().pin_memory() for k in distinct]
        xbuf = [[torch.empty_like(Xh, device=dev) for _ in range(2)] for Xh in X_host]
        ready = [torch.cuda.Event() for _ in range(2)]      # step's inputs are on the device
        free = [torch.cuda.Event() for _ in range(2)]       # step's outputs are on the host
        done = [torch.cuda.Event() for _ in layers]        # layer pruned (per step)
        pin = dict(pin_memory=True)
        host, devb = [], []     # per layer: pinned host tensors; two sets of device buffers
        for W0, W, g, sp, p in layers:
            b = g.bufs
            pk = b.packs(p)
            host.append({"W_in": W0.cpu().pin_memory(),
                         "W_out": torch.empty(W.shape, dtype=W.dtype, **pin),
                         "mask": torch.empty(b.mask.shape, dtype=b.mask.dtype, **pin),
                         "values": torch.empty(b.values.shape, dtype=b.values.dtype, **pin) if pk else None,
                         "meta": torch.empty(b.meta.shape, dtype=b.meta.dtype, **pin) if pk else None})
            devb.append([{"W": torch.empty_like(W), "mask": torch.empty_like(b.mask),
                          "values": torch.empty_like(b.values) if pk else None,
                          "meta": torch.empty_like(b.meta) if pk else None} for _ in range(2)])
        h2d = sum(Xh.numel() * Xh.element_size() for Xh in X_host) + sum(h["W_in"].numel() * 4 for h in host)
        d2h = sum(sum(t.numel() * t.element_size() for k, t in h.items() if k != "W_in" and t is not None)
                  for h in host)
        step_no = [0]

        def e2e_step():
            bsel = step_no[0] & 1
            step_no[0] += 1
            with torch.cuda.stream(h2d_s):
                h2d_s.wait_event(free[bsel])        # step s-2's outputs in these buffers are on the host
                for j, Xh in enumerate(X_host):
                    xbuf[j][bsel].copy_(Xh, non_blocking=True)
                for k, h in enumerate(host):
                    devb[k][bsel]["W"].copy_(h["W_in"], non_blocking=True)
                ready[bsel].record(h2d_s)
            with torch.cuda.stream(comp_s):
                comp_s.wait_event(ready[bsel])
                k = 0
                for j, (xs, _, mats) in enumerate(jobs):
                    for m_i, (sp, p) in enumerate(mats):
                        g, bd = layers[k][2], devb[k][bsel]
                        b = g.bufs
                        pack = b.packs(p)
                        if m_i == 0:
                            pp.prune_layer(bd["W"], b.H, b.U, p, bd["mask"], b.ws, b.info,
                                           X=xbuf[x_of_job[j]][bsel], values=bd["values"], meta=bd["meta"],
                                           row_loss=b.row_loss)
                        else:
                            pp.info_clear(b.info)
                            b.row_loss.zero_()
                            pp.prune(bd["W"], b.U, p, bd["mask"], b.ws, b.info, row_loss=b.row_loss)
                            if pack:
                                pp.pack_nm(bd["W"], bd["mask"], *p.nm, bd["values"], bd["meta"], b.info)
                        done[k].record(comp_s)
                        k += 1
            with torch.cuda.stream(d2h_s):
                for k, h in enumerate(host):
                    d2h_s.wait_event(done[k])
                    bd = devb[k][bsel]
                    for key in ("W", "mask", "values", "meta"):
                        if bd[key] is not None:
                            h["W_out" if key == "W" else key].copy_(bd[key], non_blocking=True)
                free[bsel].record(d2h_s)

        for _ in range(max(2, args.warmup // 2)):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ks = max(2, args.steps // 2)
        e0.record(h2d_s)
        for _ in range(ks):
            e2e_step()
        e1.record(d2h_s)
        torch.cuda.synchronize()
        for _, _, g, _, _ in layers:
            pp.raise_on_info(g.bufs.info, where="e2e")
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist if world > 1 else None, dev)
        line["e2e"] = {"value": weights_per_step * ks * world / t_e2e, "unit": UNIT,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": t_e2e * 1e3 / ks, "steps": ks,
                       "note": ("every step copies each distinct X and every W from pinned host memory and "
                                "every pruned W, mask, N:M values and metadata back into pinned host memory; "
                                "uploads, pruning and downloads run on three streams, so step s+1's uploads "
                                "and step s's downloads overlap step s's pruning (two device buffers per "
                                "input and output)")}
        del xbuf, devb

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, t, cores, sample = cpu_baseline(specs)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": sample, "scaled_seconds_per_step": t}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ other rows

def _events(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def bench_mlp_block(args):
    """The multi-layer driver on one Qwen3-32B-shaped MLP block (hidden 5120,
    intermediate 25600, 131,072 tokens, 2:4 unless --pattern): gate and up
    pruned from the block input, the down input formed with the pruned (or,
    --driver parallel, dense) gate and up, down pruned from it, the block
    output formed; every step restores the dense weights (untimed). Also
    times the driver's forward product alone (sgpt_linear_bf16 of the same
    shape as gate) for its roofline."""
    import torch

    import post_pruning_b200 as pp
    from workloads import LayerSpec, gen_activations, gen_weights
    dev = torch.device("cuda")
    h, f, n = 5120, 25600, 131072
    spec = LayerSpec("mlp_in", d_in=h, d_out=f, n_tok=n, sigma=1.0, p_out=0.01, f_out=20.0, x_key=2)
    X = gen_activations(spec, device=dev)
    W0 = [gen_weights(spec.with_(w_key=4), device=dev), gen_weights(spec.with_(w_key=5), device=dev),
          gen_weights(LayerSpec("down", d_in=f, d_out=h, n_tok=n, w_key=6), device=dev)]
    W = [w.clone() for w in W0]
    masks = (torch.empty(f, h // 32, dtype=torch.int32, device=dev), torch.empty(f, h // 32, dtype=torch.int32,
             device=dev), torch.empty(h, f // 32, dtype=torch.int32, device=dev))
    X_next = torch.empty(n, h, dtype=torch.bfloat16, device=dev)
    ws = pp.mlp_block_workspace(h, f, n)
    info = pp.new_info()
    p = pp.Params(args.pattern or "2:4", qbits=args.qbits)
    mode = pp.DRIVER_PARALLEL if args.driver == "parallel" else pp.DRIVER_SEQUENTIAL
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    def step():
        pp.prune_mlp_block(*W, masks, X, p, X_next, ws, info, mode=mode)

    def prep():
        for w, w0 in zip(W, W0):
            w.copy_(w0)
        flush.zero_()
    for _ in range(args.warmup):
        prep()
        step()
    pp.raise_on_info(info)
    evs = [_events(torch) for _ in range(args.steps)]
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    l0 = pp.kernel_launches()
    for e0, e1 in evs:
        prep()
        e0.record(st)
        step()
        e1.record(st)
    torch.cuda.synchronize()
    launches = pp.kernel_launches() - l0
    clk = clocks.stop()
    pp.raise_on_info(info)
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    weights = 3 * h * f
    # the forward product alone: x Wg^T, n x h x f
    Wb = torch.empty(f, h, dtype=torch.bfloat16, device=dev)
    pp.to_bf16(W0[0], Wb, info)
    Y = torch.empty(n, f, device=dev)
    for _ in range(3):
        pp.linear_bf16(X, Wb, Y, info)
    e0, e1 = _events(torch)
    e0.record(st)
    for _ in range(10):
        pp.linear_bf16(X, Wb, Y, info)
    e1.record(st)
    torch.cuda.synchronize()
    g_ms = e0.elapsed_time(e1) / 10
    g_flops = 2.0 * n * h * f
    hbm, bf16_burst, bf16_sust, kind = peaks()
    line = {"metric": "multi-layer driver: one MLP block pruned layer by layer, weights/s", "value": weights / ms * 1e3,
            "unit": "weights/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "f32 (forward products bf16)", "data": "synthetic",
            "config": {"workload": f"Qwen3-32B-shaped MLP block h={h} f={f}, {n} tokens, {p.pattern}, "
                                   f"driver {args.driver}", "name": "qwen3_32b_mlp_block"},
            "gpu_launches": launches,
            "forward_gemm": {"kernel": "gemm_tc_kernel<bf16>", "shape": f"{n}x{h} * {h}x{f}", "ms": g_ms,
                             "achieved": g_flops / g_ms / 1e9, "unit": "TFLOP/s", "peak": bf16_burst,
                             "frac": g_flops / g_ms / 1e9 / bf16_burst, "peak_kind": f"{kind} bf16 burst"},
            "clocks": clk}
    print(json.dumps(line), flush=True)


def bench_consumer(args):
    """The 2:4 consumer: Y = X W^T from the packed 2:4 form of the Qwen3-32B
    down-proj (5120 x 25600) on the sparse tensor cores, against the dense
    tensor-core product of the same (unpacked, bf16) weights; 8192 tokens."""
    import torch

    import post_pruning_b200 as pp
    dev = torch.device("cuda")
    d_out, d_in, n = 5120, 25600, 8192
    g = torch.Generator(device=dev).manual_seed(0)
    W = torch.randn(d_out, d_in, device=dev, generator=g)
    keep = torch.zeros(d_out, d_in // 4, 4, dtype=torch.bool, device=dev)
    keep.scatter_(2, torch.rand(d_out, d_in // 4, 4, device=dev, generator=g).topk(2, dim=2).indices, True)
    keep = keep.reshape(d_out, d_in)
    W = torch.where(keep, W, torch.zeros_like(W))
    bits = (keep.reshape(d_out, d_in // 32, 32).to(torch.int64) << torch.arange(32, device=dev)).sum(2)
    mask = torch.where(bits >= 2 ** 31, bits - 2 ** 32, bits).to(torch.int32)   # the same 32 bits as int32
    info = pp.new_info()
    vals = torch.empty(d_out, d_in // 2, device=dev)
    meta = torch.empty(d_out, d_in // 32, dtype=torch.int32, device=dev)
    pp.pack24(W, mask, vals, meta, info)
    vb = torch.empty(d_out, d_in // 2, dtype=torch.bfloat16, device=dev)
    pp.to_bf16(vals, vb, info)
    Wb = torch.empty(d_out, d_in, dtype=torch.bfloat16, device=dev)
    pp.to_bf16(W, Wb, info)
    X = torch.randn(n, d_in, device=dev, generator=g).to(torch.bfloat16)
    Y = torch.empty(n, d_out, device=dev)
    pp.raise_on_info(info)
    tiles = pp.sparse24_meta_tiles(meta, d_in)      # once per weight matrix, timed apart below
    st = torch.cuda.current_stream()
    out = {}
    for name, fn in (("sparse24", lambda: pp.sparse24_linear(vb, tiles, X, Y, info)),
                     ("dense", lambda: pp.linear_bf16(X, Wb, Y, info)),
                     ("tile_meta", lambda: pp.sparse24_meta_tiles(meta, d_in, out=tiles))):
        for _ in range(args.warmup):
            fn()
        e0, e1 = _events(torch)
        e0.record(st)
        for _ in range(args.steps):
            fn()
        e1.record(st)
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / args.steps
    pp.raise_on_info(info)
    flops = 2.0 * n * d_in * d_out
    hbm, bf16_burst, bf16_sust, kind = peaks()
    line = {"metric": "2:4 consumer: Y = X W^T from the packed 2:4 form, dense-equivalent TFLOP/s",
            "value": flops / out["sparse24"] / 1e9, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": out["sparse24"], "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"X {n}x{d_in} bf16, W {d_out}x{d_in} 2:4 (values bf16 + 2-bit metadata)",
                       "name": "consumer_qwen_down"},
            "dense_ms": out["dense"], "dense_tflops": flops / out["dense"] / 1e9,
            "tile_meta_ms": out["tile_meta"],
            "speedup_vs_dense": out["dense"] / out["sparse24"],
            "peak": {"bf16_dense": bf16_burst, "sparse_2to4_nominal": 2 * bf16_burst, "kind": f"{kind} burst"}}
    print(json.dumps(line), flush=True)


def bench_hessian(args):
    """The Hessian kernel alone: H = X^T X for X [tokens x width] bf16 with
    the Qwen-block channel-scale distribution (sgpt_hessian_compute), for
    per-kernel timing and profiler captures at a chosen size."""
    import torch

    import post_pruning_b200 as pp
    from workloads import LayerSpec, gen_activations
    dev = torch.device("cuda")
    spec = LayerSpec("hessian", d_in=args.width, d_out=128, n_tok=args.tokens, sigma=1.0, p_out=0.01, f_out=20.0,
                     x_key=3)
    X = gen_activations(spec, device=dev)
    H = torch.empty(args.width, args.width, device=dev)
    ws = pp.workspace(128, args.width, args.tokens)
    info = pp.new_info()
    st = torch.cuda.current_stream()
    for _ in range(args.warmup):
        pp.hessian_compute(H, X, ws, info)
    e0, e1 = _events(torch)
    e0.record(st)
    for _ in range(args.steps):
        pp.hessian_compute(H, X, ws, info)
    e1.record(st)
    torch.cuda.synchronize()
    pp.raise_on_info(info)
    ms = e0.elapsed_time(e1) / args.steps
    flops = float(args.tokens) * args.width * (args.width + 1)
    hbm, bf16_burst, bf16_sust, kind = peaks()
    print(json.dumps({"metric": "Hessian H = X^T X alone, TFLOP/s (n*d*(d+1) flop)", "value": flops / ms / 1e9,
                      "unit": "TFLOP/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
                      "config": {"workload": f"X {args.tokens} x {args.width} bf16", "name": "hessian"},
                      "peak": bf16_burst, "frac": flops / ms / 1e9 / bf16_burst, "peak_kind": f"{kind} bf16 burst"}),
          flush=True)


def bench_factor(args):
    """The factorisation alone: U = chol(H_d^-1) of the Hessian of X [tokens
    x width] (sgpt_factor, damping included), for per-phase timing and
    profiler captures at a chosen size."""
    import torch

    import post_pruning_b200 as pp
    from workloads import LayerSpec, gen_activations
    dev = torch.device("cuda")
    spec = LayerSpec("factor", d_in=args.width, d_out=128, n_tok=args.tokens, sigma=1.0, p_out=0.01, f_out=20.0,
                     x_key=3)
    X = gen_activations(spec, device=dev)
    H = torch.empty(args.width, args.width, device=dev)
    U = torch.empty_like(H)
    ws = pp.workspace(128, args.width, args.tokens)
    info = pp.new_info()
    pp.hessian_compute(H, X, ws, info)
    del X
    st = torch.cuda.current_stream()
    for _ in range(args.warmup):
        pp.factor(H, args.tokens, 0.01, U, ws, info)
    e0, e1 = _events(torch)
    e0.record(st)
    for _ in range(args.steps):
        pp.factor(H, args.tokens, 0.01, U, ws, info)
    e1.record(st)
    torch.cuda.synchronize()
    pp.raise_on_info(info)
    ms = e0.elapsed_time(e1) / args.steps
    flops = 2.0 / 3.0 * float(args.width) ** 3
    hbm, bf16_burst, bf16_sust, kind = peaks()
    rate = bf16_burst * TF32_OVER_BF16 / 3.0
    print(json.dumps({"metric": "factorisation U = chol(H_d^-1) alone, FP32-accurate TFLOP/s (2/3 d^3 flop)",
                      "value": flops / ms / 1e9, "unit": "TFLOP/s", "ms_per_step": ms, "steps": args.steps,
                      "warmup": args.warmup,
                      "config": {"workload": f"H of X {args.tokens} x {args.width} bf16", "name": "factor"},
                      "peak": rate, "frac": flops / ms / 1e9 / rate,
                      "peak_kind": f"{kind} bf16 burst x {TF32_OVER_BF16:.3f} (TF32) / 3 (products per fp32 product)"}),
          flush=True)


EXTRA_BENCHES = {"qwen3_32b_mlp_block": bench_mlp_block, "consumer_qwen_down": bench_consumer,
                 "hessian": bench_hessian, "factor": bench_factor}


if __name__ == "__main__":
    main()
