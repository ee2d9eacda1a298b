#!/usr/bin/env python
"""Throughput of the Muon weight update on B200: full Mamba-2 130M optimizer steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mamba2-130m|mamba2-2k] [--mode replicas|sharded]

One step = the whole hot path over every in_proj (24 x 3352 x 768) and
out_proj (24 x 768 x 1536) matrix of a Mamba-2 130M model, in one
muon_step_groups call: momentum + Nesterov + Frobenius norm, 5 quintic
Newton-Schulz iterations (three tensor-core products each), shape scale and
decoupled weight decay applied to W.  Gradients are synthetic (Gaussian bulk
+ rank-4 spike, bf16), redrawn per step from a pool of pre-generated sets
resident in HBM; W and M persist across steps.

Multi-GPU (torchrun): every rank runs its own full step on its own GPU (the
matrices of different models/ranks are independent -- weak scaling, no
collective on the data path); time is the max over ranks.  `--mode sharded`
instead splits ONE model's step over the ranks by matrix ownership
(reduce-scatter of gradients, owned step, all-gather of weights; strong scaling).

Prints ONE JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
(the baseline arm) on rank 0 over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Muon steps/s and Newton-Schulz TFLOP/s (% of bf16 peak), Mamba-2 130M shapes"
UNIT = "steps/s"
QUINTIC = (3.4445, -4.7750, 2.0315)
K_ITERS = 5
HP = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7)
GRAD_SETS = 4

WORKLOADS = {
    # name: list of (label, count, rows, cols)
    "mamba2-130m": [("out_proj", 24, 768, 1536), ("in_proj", 24, 3352, 768)],
    "mamba2-2k": [("out_proj", 48, 2048, 4096), ("in_proj", 48, 8768, 2048)],
}
WORKLOAD_NAMES = {
    "mamba2-130m": "full Mamba-2 130M Muon step: in_proj 24x3352x768 + out_proj 24x768x1536 bf16, "
                   "5 quintic NS iterations, one muon_step_groups call",
    "mamba2-2k": "scaled Mamba-2-style d_model 2048: in_proj 48x8768x2048 + out_proj 48x2048x4096 bf16, "
                 "5 quintic NS iterations",
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- work counts
def ns_flops(groups, k=K_ITERS):
    """Algorithmic NS flops: per iteration m^2 n (symmetric Gram) + m^3 (symmetric A^2) + 2 m^2 n (B X)."""
    tot = 0
    for _, L, R, C in groups:
        m, n = min(R, C), max(R, C)
        tot += L * k * (3 * m * m * n + m ** 3)
    return tot


def ns_dense_flops(groups, k=K_ITERS):
    tot = 0
    for _, L, R, C in groups:
        m, n = min(R, C), max(R, C)
        tot += L * k * (4 * m * m * n + 2 * m ** 3)
    return tot


def elements(groups):
    return sum(L * R * C for _, L, R, C in groups)


def momentum_bytes(groups):
    """Algorithmic bytes of the momentum pass: G 2 + M 4 (read) + M 4 + U 2 (write) per element."""
    return 12 * elements(groups)


def apply_bytes(groups):
    """Algorithmic bytes of the apply pass: O 2 (read) + W 2 (read) + W 2 (write) per element (bf16)."""
    return 6 * elements(groups)


def step_bytes_algorithmic(groups):
    """Algorithmic HBM bytes of the elementwise part of one step: G 2 + M 4 (read) + M 4 + U 2 (write)
    + W 2 (read) + W 2 (write) = 16 B per element (the un-normalised U is the Newton-Schulz input)."""
    return 16 * elements(groups)


def roofline_step_ms(groups, tflops, hbm_gbs):
    """Shortest possible step: the Newton-Schulz flops at the tensor peak plus the elementwise bytes at
    the HBM peak (the two cannot overlap less than this, and need not overlap more)."""
    return ns_flops(groups) / (tflops * 1e12) * 1e3 + step_bytes_algorithmic(groups) / (hbm_gbs * 1e9) * 1e3


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text):
    """Source without comments, trailing blanks or empty lines (a capture stays valid across comment edits)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = []
    for line in text.splitlines():
        line = re.sub(r"//.*$", "", line).rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def gemm_source_hash():
    """sha256 (16 hex digits) of the NS kernel's code: gemm.cu, gemm.h, device_utils.cuh without comments."""
    h = hashlib.sha256()
    for f in ("gemm.cu", "gemm.h", "device_utils.cuh"):
        with open(os.path.join(ROOT, "spectral_optimizer_state_b200", "csrc", f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per GEMM launch from the committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"ns_gemm_kernel.{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("gemm_source_sha256") != gemm_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.lines = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- inputs
def make_inputs(groups, device, sets=GRAD_SETS, pinned_host=False):
    import torch

    from synthetic import group_inputs, group_weights
    if elements(groups) > 200_000_000:
        return make_inputs_device(groups, device, sets, pinned_host)
    Ws, Ms, Gsets, Ghost = [], [], [], []
    for g, (_, L, R, C) in enumerate(groups):
        Ws.append([torch.from_numpy(w).to(torch.bfloat16).to(device) for w in group_weights(3, g, L, R, C)])
        Ms.append([torch.zeros((R, C), dtype=torch.float32, device=device) for _ in range(L)])
    for s in range(sets):
        per_group, per_group_host = [], []
        for g, (_, L, R, C) in enumerate(groups):
            gs = group_inputs(3, s, g, L, R, C)
            per_group.append([torch.from_numpy(x).to(torch.bfloat16).to(device) for x in gs])
            if pinned_host and s == 0:
                per_group_host.append([torch.from_numpy(x).to(torch.bfloat16).pin_memory() for x in gs])
        Gsets.append(per_group)
        if pinned_host and s == 0:
            Ghost = per_group_host
    return Ws, Ms, Gsets, Ghost


def device_spike_gradient(R, C, gen, device, std=1e-3, rank=4, factor=10.0, dtype=None):
    """Gaussian N(0, std^2) bulk plus a rank-4 spike at `factor` times the bulk's top edge
    std (sqrt(R) + sqrt(C)), drawn on the device (the host recipe's distribution, another stream)."""
    import torch
    g = torch.randn((R, C), device=device, generator=gen) * std
    u, ru = torch.linalg.qr(torch.randn((R, rank), device=device, generator=gen))
    v, rv = torch.linalg.qr(torch.randn((C, rank), device=device, generator=gen))
    u = u * torch.sign(torch.diagonal(ru))
    v = v * torch.sign(torch.diagonal(rv))
    g += factor * std * (R ** 0.5 + C ** 0.5) * (u @ v.T)
    return g.to(dtype if dtype is not None else torch.bfloat16)


def make_inputs_device(groups, device, sets, pinned_host):
    """Large workloads: seeded weights and spike gradients drawn on the device (the host generator
    would take minutes for 1.3 G elements), one gradient set."""
    import torch
    gen = torch.Generator(device=device).manual_seed(3000)
    Ws, Ms, G1, Ghost = [], [], [], []
    for g, (_, L, R, C) in enumerate(groups):
        Ws.append([(torch.randn((R, C), device=device, generator=gen) * 0.02).to(torch.bfloat16) for _ in range(L)])
        Ms.append([torch.zeros((R, C), dtype=torch.float32, device=device) for _ in range(L)])
        G1.append([device_spike_gradient(R, C, gen, device) for _ in range(L)])
        if pinned_host:
            Ghost.append([t.cpu().pin_memory() for t in G1[-1]])
    return Ws, Ms, [G1] * sets, Ghost


# ---------------------------------------------------------------- oracle arm
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def blas_vendor():
    try:
        from threadpoolctl import threadpool_info
        for d in threadpool_info():
            if d.get("user_api") == "blas":
                return f"{d.get('internal_api')} {d.get('version')}"
    except Exception:
        pass
    return "unknown"


def oracle_one_thread_seconds(groups):
    """Seconds of the fp64 oracle for one matrix of the first group with BLAS held to one thread."""
    import oracle
    from synthetic import group_inputs, group_weights
    from threadpoolctl import threadpool_limits
    _, _, R, C = groups[0]
    G = group_inputs(3, 0, 0, 1, R, C)[0].astype(np.float64)
    W = group_weights(3, 0, 1, R, C)[0].astype(np.float64)
    with threadpool_limits(limits=1, user_api="blas"):
        t0 = time.perf_counter()
        oracle.muon_step(W, G, np.zeros((R, C)), [QUINTIC] * K_ITERS, **HP)
        return time.perf_counter() - t0


def oracle_sample(groups, budget_s=12.0, max_per_group=96):
    """Time the fp64 oracle on whole matrices of one step until ~budget_s; returns steps/s and a label."""
    import oracle
    from synthetic import group_inputs, group_weights
    coeffs = [QUINTIC] * K_ITERS
    done = {lbl: 0 for lbl, *_ in groups}
    t_total = 0.0
    frac = 0.0
    total_mats = sum(L for _, L, _, _ in groups)
    for i in range(max_per_group):
        for g, (lbl, L, R, C) in enumerate(groups):
            G = group_inputs(3, 0, g, 1, R, C)[0].astype(np.float64)
            W = group_weights(3, g, 1, R, C)[0].astype(np.float64)
            M = np.zeros((R, C))
            t0 = time.perf_counter()
            oracle.muon_step(W, G, M, coeffs, **HP)
            t_total += time.perf_counter() - t0
            done[lbl] += 1
            frac += 1.0 / total_mats
        if t_total >= budget_s:
            break
    sample = (" + ".join(f"{n} {lbl}" for lbl, n in done.items())
              + " matrices, alternating groups, until about 12 s of fp64 NumPy (oracle.muon_step)")
    return frac / t_total, sample, t_total


def measure_spectral(mu, Ws, Gs, Ms, groups, stream, peaks, pi_iters=8, min_iters=16, reps=5):
    """Spectral diagnostics and the capped step on every group of the workload (device-timed)."""
    import torch

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    w_bytes = sum(L * R * C * 2 for _, L, R, C in groups)
    dev = Ws[0][0].device
    vecs = []
    for g, (_, L, R, C) in enumerate(groups):
        u = [torch.zeros(R, device=dev) for _ in range(L)]
        v = [torch.ones(C, device=dev) for _ in range(L)]
        y = [torch.ones(min(R, C), device=dev) for _ in range(L)]
        vecs.append((u, v, y, torch.zeros(L, device=dev), torch.zeros(L, device=dev), torch.zeros(L, device=dev)))

    # checked and marshalled once, as a training loop holding these tensors would
    plans = [mu.spectral_plan(Ws[g], vecs[g][0], vecs[g][1], vecs[g][3], vecs[g][2], vecs[g][4])
             for g in range(len(groups))]

    def power():
        for plan in plans:
            plan.power_iteration(iters=pi_iters, stream=stream)

    def min_sv():
        for plan in plans:
            plan.min_singular(iters=min_iters, stream=stream)

    def plain():
        for g in range(len(groups)):
            mu.step(Ws[g], Gs[g], Ms[g], stream=stream, **HP)

    def capped():
        for g in range(len(groups)):
            u, v, _, _, _, alpha = vecs[g]
            mu.step_capped(Ws[g], Gs[g], Ms[g], u, v, alpha, stream=stream, **HP)

    pi_ms = timed(power)
    min_ms = timed(min_sv)
    plain_ms = timed(plain)
    cap_ms = timed(capped)
    st, _ = mu.status()
    assert st == 0, f"device status {st}"
    kappa = [float((vecs[g][3] / vecs[g][4]).max()) for g in range(len(groups))]
    pi_gbs = pi_iters * w_bytes / (pi_ms / 1e3) / 1e9
    min_gbs = (min_iters + 1) * w_bytes / (min_ms / 1e3) / 1e9
    hbm = peaks["hbm_gbs"]
    return {
        "bound": "hbm",
        "note": ("passes over W; algorithmic bytes: one pass over W per power iteration (u and W^T u "
                 "come from the same pass, since W^T u = W^T (W v) / |W v|), one per shifted iteration + 1 "
                 "(X X^T y formed in one pass: rows of a tall W, column slabs of a wide one); "
                 "one group's W (<= 124 MB at 130M) can stay in the 126 MB L2 between passes"),
        "power_iteration": {"iters": pi_iters, "ms": pi_ms, "achieved_gbs": pi_gbs, "frac": pi_gbs / hbm},
        "min_singular": {"iters": min_iters, "ms": min_ms, "achieved_gbs": min_gbs, "frac": min_gbs / hbm,
                         "max_kappa_estimate": kappa},
        "capped_step_ms": cap_ms, "plain_step_ms": plain_ms, "cap_overhead_ms": cap_ms - plain_ms,
        "step_entry": "muon_step / muon_step_capped per group (not the fused two-group call)",
    }


GEMM_KINDS = ("gram", "poly", "update", "ns_fused")


def measure_fp32(mu, groups, device, stream, peaks, reps=20):
    """The fp32 path on the same shapes: fp32 W and G, every Newton-Schulz operand split into three
    bf16 planes and six plane products accumulated per contraction (so 6x the bf16 tensor work)."""
    import torch
    gen = torch.Generator(device=device).manual_seed(3100)
    W = [[torch.randn((R, C), device=device, generator=gen) * 0.02 for _ in range(L)] for _, L, R, C in groups]
    G = [[device_spike_gradient(R, C, gen, device, dtype=torch.float32) for _ in range(L)] for _, L, R, C in groups]
    M = [[torch.zeros((R, C), device=device) for _ in range(L)] for _, L, R, C in groups]

    def step():
        mu.step_groups([(W[g], G[g], M[g]) for g in range(len(groups))], stream=stream, **HP)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    mu.profile_read(reset=True)
    mu.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    mu.profile_enable(False)
    prof = mu.profile_read(reset=True)
    st, _ = mu.status()
    assert st == 0, f"device status {st}"
    ms = e0.elapsed_time(e1) / reps
    ns_ms = sum(prof[k][1] for k in GEMM_KINDS) / reps
    alg = ns_flops(groups)
    plane_tf = 6 * alg / (ns_ms / 1e3) / 1e12
    del W, G, M
    return {"steps_per_s": 1000.0 / ms, "ms_per_step": ms, "ns_ms_per_step": ns_ms,
            "ns_algorithmic_tflops": alg / (ns_ms / 1e3) / 1e12,
            "plane_product_tflops": plane_tf,
            "plane_product_frac_of_bf16_peak": {"burst": plane_tf / peaks["bf16_tflops"],
                                                "sustained": plane_tf / peaks["bf16_tflops_sustained"]},
            "steps": reps,
            "note": ("fp32 W, G and M; each Newton-Schulz operand as three bf16 planes, six plane products "
                     "per contraction on the bf16 tensor cores (6x the algorithmic flops)")}


def steady_state_run(step_fn, stream, mu, gpu_id, ms_per_step, groups, peaks, min_s=1.0, max_steps=20000):
    """The same step repeated for at least `min_s` seconds after the timed region, with the SM clock
    sampled meanwhile: the steady state under the power cap, for reading the short timed region."""
    import torch
    n = int(min(max_steps, max(1, min_s * 1.2 * 1000.0 / max(ms_per_step, 1e-3))))
    clocks = ClockSampler(gpu_id)
    mu.profile_read(reset=True)
    mu.profile_enable(True)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        step_fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    mu.profile_enable(False)
    prof = mu.profile_read(reset=True)
    ms = e0.elapsed_time(e1)
    ns_ms = sum(prof[k][1] for k in GEMM_KINDS)
    tf = ns_flops(groups) * n / (ns_ms / 1e3) / 1e12
    out = {"steps": n, "seconds": ms / 1e3, "steps_per_s": n / (ms / 1e3), "ns_tflops": tf,
           "ns_frac_of_bf16_peak": {"burst": tf / peaks["bf16_tflops"],
                                    "sustained": tf / peaks["bf16_tflops_sustained"]},
           "clocks": clk}
    if clk.get("sm_mhz"):
        # work per SM clock, which the power cap's clock changes do not move
        out["ns_flop_per_sm_clock"] = ns_flops(groups) * n / (ns_ms / 1e3) / (clk["sm_mhz"] * 1e6) / 148
    return out


def run_reference(args, groups, rank):
    if rank != 0:
        return
    per_step = []
    labels = None
    coeffs = [QUINTIC] * K_ITERS
    import oracle
    from synthetic import group_inputs, group_weights
    total_mats = sum(L for _, L, _, _ in groups)
    mats = []
    for g, (lbl, L, R, C) in enumerate(groups):
        mats.append((g, lbl, R, C, group_inputs(3, 0, g, 1, R, C)[0].astype(np.float64),
                     group_weights(3, g, 1, R, C)[0].astype(np.float64)))
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for (g, lbl, R, C, G, W) in mats:  # one matrix of each group per step
            oracle.muon_step(W, G, np.zeros((R, C)), coeffs, **HP)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            per_step.append(dt)
    frac = len(mats) / total_mats
    value = frac * len(per_step) / sum(per_step)
    labels = (" + ".join(f"1 {m[1]}" for m in mats) + f" matrix per step (oracle.muon_step, fp64 NumPy); "
              f"steps/s extrapolated from {len(mats)} of the step's {total_mats} matrices")
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": labels,
                         "extrapolated": True, "matrices_timed_per_step": len(mats),
                         "matrices_per_step": total_mats,
                         "seconds_per_timed_step": sum(per_step) / max(len(per_step), 1)},
        "extrapolated": True,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(args):
    return {"workload": WORKLOAD_NAMES[args.workload], "ns_iterations": K_ITERS,
            "coefficients": list(QUINTIC), "hparams": HP, "parallelism": f"replicas x{args.gpus} (independent matrices)",
            "grad_sets_in_hbm": GRAD_SETS,
            "l2": "inputs larger than L2: each step streams G, M and W (%.2f GB)" % (
                elements(WORKLOADS[args.workload]) * 8 / 1e9)}


# ---------------------------------------------------------------- sharded data parallelism
def run_sharded(args, groups, world, rank, local, device):
    """Strong scaling of one model: ShardedMuon over `world` ranks -- an in-place NCCL reduce-scatter
    of the gradients to the matrices' owners, the owners' libmuon step (the 1/N average folded into
    its momentum pass), an in-place all-gather of the weights.  Each rank's local gradient is
    refreshed from a resident copy before every step (a backward pass would write it there); only
    opt.step() is timed, per part, with CUDA events on the launching stream."""
    import torch
    import torch.distributed as dist
    from spectral_optimizer_state_b200.sharded import ShardedMuon
    shapes = [(R, C) for _, L, R, C in groups for _ in range(L)]
    opt = ShardedMuon(shapes, dtype=torch.bfloat16, device=device, coeffs=[QUINTIC] * K_ITERS, **HP)
    gen = torch.Generator(device=device).manual_seed(3000)  # identical weights on every rank
    for w in opt.weights:
        w.copy_((torch.randn(w.shape, device=device, generator=gen) * 0.02).to(torch.bfloat16))
    gen_r = torch.Generator(device=device).manual_seed(3300 + rank)  # this rank's own gradients
    local_g = [device_spike_gradient(R, C, gen_r, device) for (R, C) in shapes]
    stream = torch.cuda.current_stream()
    parts = ("reduce_scatter", "local_step", "all_gather")
    n_ev = args.steps * 4
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]

    def refresh():
        for g, src in zip(opt.grads, local_g):
            g.copy_(src)

    for _ in range(args.warmup):
        refresh()
        opt.step()
    st, _ = opt.local_step.muon.status() if opt.owned else (0, [])
    assert st == 0, f"device status {st}"
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        refresh()
        marks = iter(evs[4 * i:4 * i + 4])
        opt.step(mark=lambda phase: next(marks).record(stream))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    per_part = {p: 0.0 for p in parts}
    for i in range(args.steps):
        e = evs[4 * i:4 * i + 4]
        for j, p in enumerate(parts):
            per_part[p] += e[j].elapsed_time(e[j + 1])
    ms_local = sum(per_part.values())
    ms = max_over_ranks(ms_local, world, device)
    parts_max = {p: max_over_ranks(v, world, device) / args.steps for p, v in per_part.items()}
    nbytes = opt.owned_bytes()
    line = {
        "metric": METRIC, "value": args.steps / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_dict(args), parallelism=f"sharded x{world} (reduce-scatter -> owned step -> all-gather)"),
        "matrices_per_s": args.steps / (ms / 1e3) * len(shapes),
        "ms_per_step_by_part": parts_max,
        "owned_matrices": len(opt.owned),
        "bytes_per_rank": {"reduce_scatter_in": nbytes["reduce_scatter_bytes"],
                           "all_gather_out": nbytes["all_gather_bytes"],
                           "momentum_state": nbytes["momentum_bytes"]},
        "note": "one model's step, total work fixed as N grows; timed region = opt.step() only",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    opt.local_step.muon.close()


# ---------------------------------------------------------------- ranks
def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's value (one all-reduce on `device`); the value itself at N = 1."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="mamba2-130m")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-spectral", dest="spectral", action="store_false",
                    help="skip the power-iteration / min-singular / capped-step measurements")
    ap.add_argument("--no-fp32", dest="fp32", action="store_false", help="skip the fp32-path measurement")
    ap.add_argument("--mode", choices=["replicas", "sharded"], default="replicas",
                    help="replicas: every rank steps its own model (weak scaling, the default); sharded: one "
                         "model's step split over the ranks by matrix ownership (strong scaling)")
    ap.add_argument("--no-long-run", dest="long_run", action="store_false",
                    help="skip the >= 1 s steady-state repeat after the timed region")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    groups = WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, groups, rank)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from spectral_optimizer_state_b200 import Muon

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    if args.mode == "sharded":
        run_sharded(args, groups, world, rank, local, device)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    # cpu baseline first (rank 0, N = 1), before any pools or threads touch the GPU
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, spent = oracle_sample(groups)
        cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample,
               "seconds": round(spent, 2), "blas": blas_vendor(),
               "one_thread_seconds_per_matrix": {groups[0][0]: round(oracle_one_thread_seconds(groups), 3)}}

    mu = Muon(local)
    mu.set_coeffs([QUINTIC] * K_ITERS)
    Ws, Ms, Gsets, Ghost = make_inputs(groups, device, pinned_host=True)
    stream = torch.cuda.current_stream()

    # one plan per gradient set, checked and marshalled once (a training loop whose gradient
    # buffers stay in place does the same)
    step_plans = [mu.step_plan([(Ws[g], Gsets[s][g], Ms[g]) for g in range(len(groups))], **HP)
                  for s in range(GRAD_SETS)]

    def step(i):
        step_plans[i % GRAD_SETS](stream=stream)

    for i in range(args.warmup):
        step(i)
    st, flags = mu.status()
    assert st == 0, f"device status {st}"

    peaks, peak_src = load_peaks()
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")  # during the timed region

    mu.profile_read(reset=True)
    mu.profile_enable(True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    mu.profile_enable(False)
    prof = mu.profile_read(reset=True)
    st, flags = mu.status()
    assert st == 0, f"device status {st}"
    ms = max_over_ranks(t0.elapsed_time(t1), world, device)
    gpu_id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
    steady = steady_state_run(step, stream, mu, gpu_id, ms / args.steps, groups, peaks) if args.long_run else None

    # e2e through the host-gradient entry point (pinned host G in, norms + flags out)
    e2e_steps = max(3, min(args.e2e_steps, args.steps))
    for i in range(2):
        mu.step_groups_host([(Ws[g], Ghost[g], Ms[g]) for g in range(len(groups))], stream=stream, **HP)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        mu.step_groups_host([(Ws[g], Ghost[g], Ms[g]) for g in range(len(groups))], stream=stream, **HP)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)

    # AdamW over the parameters Muon does not take (the rest of Mamba-2 130M)
    adamw = None
    if args.workload == "mamba2-130m":
        from spectral_optimizer_state_b200 import AdamWGroup
        from synthetic import mamba2_130m_other_params
        others = mamba2_130m_other_params()
        aw = [torch.randn(int(np.prod(sh)), device=device).to(torch.bfloat16) * 0.02 for _, sh in others]
        ag = [torch.randn(w.numel(), device=device).to(torch.bfloat16) for w in aw]
        am = [torch.zeros(w.numel(), device=device) for w in aw]
        av = [torch.zeros(w.numel(), device=device) for w in aw]
        adam = AdamWGroup(aw, ag, am, av)  # checked and marshalled once, like an optimizer holding its state
        for i in range(3):
            adam.step(i + 1, stream=stream)
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        reps = 20
        a0.record(stream)
        for i in range(reps):
            adam.step(i + 4, stream=stream)
        a1.record(stream)
        torch.cuda.synchronize()
        a_ms = a0.elapsed_time(a1) / reps
        numel = sum(w.numel() for w in aw)
        gbs = 22 * numel / (a_ms / 1e3) / 1e9
        adamw = {"bound": "hbm", "params": numel, "ms_per_step": a_ms, "achieved_gbs": gbs,
                 "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"], "bytes_per_element": 22,
                 "tensors": len(aw), "launches_per_step": len(adam._calls),
                 "note": "AdamW over the non-Muon parameters of Mamba-2 130M, bf16 (AdamWGroup)"}
        del aw, ag, am, av

    spectral = measure_spectral(mu, Ws, Gsets[0], Ms, groups, stream, peaks) if args.spectral else None
    fp32 = None
    if args.fp32 and args.workload == "mamba2-130m":
        fp32 = measure_fp32(mu, groups, device, stream, peaks)

    n_mats = sum(L for _, L, _, _ in groups)
    steps_per_s = world * args.steps / (ms / 1e3)
    gemm_launches = sum(prof[k][0] for k in GEMM_KINDS)
    gemm_ms = sum(prof[k][1] for k in GEMM_KINDS)
    flops_timed = ns_flops(groups) * args.steps
    achieved_tf = flops_timed / (gemm_ms / 1e3) / 1e12
    burst, sustained = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    # a kernel timed inside a long loop of steps runs in the power-capped regime the
    # sustained peak was measured in; a short timed region is compared with the burst peak
    long_run = ms >= 1000.0
    peak = sustained if long_run else burst
    peak_kind = (f"{peak_src} bf16 sustained (cuBLAS loop under the power cap; timed region "
                 f"{ms / 1e3:.2f} s)" if long_run else f"{peak_src} bf16 burst (cuBLAS 8192^3)")
    traffic = recorded_traffic(args.workload)
    mom_launches, mom_ms = prof["momentum"]
    app_launches, app_ms = prof["apply"]
    app_gbs = apply_bytes(groups) * args.steps / (app_ms / 1e3) / 1e9 if app_ms > 0 else None
    mom_gbs = momentum_bytes(groups) * args.steps / (mom_ms / 1e3) / 1e9 if mom_ms > 0 else None
    h2d = sum(L * R * C * 2 for _, L, R, C in groups)
    d2h = n_mats * 8
    roof_ms = roofline_step_ms(groups, peak, peaks["hbm_gbs"])
    roof_steps = 1000.0 / roof_ms

    line = {
        "metric": METRIC, "value": steps_per_s, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(args),
        "matrices_per_s": steps_per_s * n_mats,
        "step_roofline": {"ms": roof_ms, "steps_per_s": world * roof_steps, "matrices_per_s": world * roof_steps * n_mats,
                          "tensor_peak_tflops": peak, "hbm_peak_gbs": peaks["hbm_gbs"],
                          "ns_flops": ns_flops(groups), "elementwise_bytes": step_bytes_algorithmic(groups),
                          "basis": "NS algorithmic flops at the tensor peak + 16 B/element at the HBM peak"},
        "steps_per_s_frac": steps_per_s / (world * roof_steps),
        "matrices_per_s_frac": steps_per_s / (world * roof_steps),
        "ns_tflops": achieved_tf,
        "ns_frac_of_bf16_peak": {"burst": achieved_tf / burst, "sustained": achieved_tf / sustained,
                                 "source": peak_src},
        "ns_dense_equivalent_tflops": ns_dense_flops(groups) * args.steps / (gemm_ms / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": "ns_gemm_kernel", "achieved": achieved_tf, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved_tf / peak, "peak_kind": peak_kind,
                     "traffic": traffic,
                     "flops_per_launch": flops_timed / max(gemm_launches, 1),
                     "avg_launch_ms": gemm_ms / max(gemm_launches, 1), "launches": gemm_launches},
        "momentum_kernel": {"bound": "hbm", "achieved_gbs": mom_gbs, "peak_gbs": peaks["hbm_gbs"],
                            "frac": (mom_gbs / peaks["hbm_gbs"]) if mom_gbs else None,
                            "bytes_per_element": 12, "launches": mom_launches},
        "apply_kernel": {"bound": "hbm", "achieved_gbs": app_gbs, "peak_gbs": peaks["hbm_gbs"],
                         "frac": (app_gbs / peaks["hbm_gbs"]) if app_gbs else None,
                         "bytes_per_element": 6, "launches": app_launches},
        "kernel_ms_per_step": {k: v[1] / args.steps for k, v in prof.items()},
        "adamw_kernel": adamw,
        "spectral": spectral,
        "fp32_path": fp32,
        "steady_state": steady,
        "cpu_baseline": cpu,
        "clocks": clk,
        "e2e": {"value": world * e2e_steps / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "entry": "muon_step_groups_host (pinned host G -> device, norms + flags -> host)",
                "bound": "the host-to-device upload of every gradient each step (W and M stay resident)"},
        "gpu_launches": sum(v[0] for v in prof.values()),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    mu.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
