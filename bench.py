"""Benchmark: block-sparse attention with the LiteAttention skip chain on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-e2e] [--no-cpu-baseline] [--no-configs]
    python bench.py --suite     (every workload's path, one JSON line each)

Default workload: the Wan2.1-14B-like 720p LiteAttention step (B=1, H=40,
d=128, 21 x 45 x 80 grid = 75,600 tokens, block 128, eps = 10): each bench
step is one denoising step's attention call, sa_sparse_attn_fwd with an
all-kept mask, skip_in = the previous step's skip_out, and a fresh skip_out
(the whole hot path of this workload; the skip test is fused in the kernel).
Each step's Q/K/V are that denoising step's drifted inputs (x <- 0.98 x +
0.2 xi), drawn on the device before the timed region; 3 x 774 MB per step is
far larger than L2, so no flush is needed between steps.

Printed metric: executed TFLOP/s of the attention forward (4 * d * sum over
visited (q-block, k-block) pairs of valid rows x valid columns), with ms per
call, density and the dense-equivalent rate alongside.  With N > 1 GPUs each
rank runs its own copy of the workload (heads are independent; weak scaling,
no collective on the data path) and the value is total FLOPs / max-over-ranks
time.

The same JSON line carries, under "configs" (single-GPU runs), the other
workloads' paths, each device-timed with its roofline fraction and an oracle
sample on the host (with the GPU-vs-oracle mask bit counts): the 480p
tau-mask path, the 720p radial path, the 480p PSA pyramid path, and a
labelled eps = 2 run of the 75.6K-token chain whose steps consume the skip
bits of the step before (the time per step against the executed tiles).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse attn ms/call, executed TFLOP/s & % B200 BF16 tensor peak at 75.6K tok"
# DRAM bytes (read + write) of one attention launch at 75,600 tokens x 40 heads,
# from an ncu capture of the 4-head case (239.5 MB read + 61.4 MB written,
# scaled by 40/4 heads).  Valid for the kernel version that capture measured;
# set to None whenever the kernel changes.  The source edits since that capture
# removed only code that never ran (a polynomial branch whose condition was
# false at compile time, an unused barrier helper), so the executed kernel is
# the one measured.
ATTN_DRAM_BYTES_PER_LAUNCH = 3.0087e9
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"sa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.dev)], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def replica_seed(base_seed, rank):
    """Seed of a rank's drift noise: every replica runs its own copy of the workload."""
    return base_seed + 1 + 1000 * rank


def replica_chain(wl, rank, nsteps, device, H=None):
    """The denoising inputs of one replica: the workload's step-0 draw (the same
    on every rank) and nsteps - 1 drift steps whose noise comes from the
    rank's own seed, so the replicas run different chains."""
    from block_sparse_attention_flash_b200 import inputs

    q0, k0, v0 = inputs.rff_qkv(wl, H=H, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(replica_seed(wl.seed, rank))
    qkv = [(q0, k0, v0)]
    for _ in range(1, nsteps):
        q, k, v = qkv[-1]
        qkv.append((inputs.drift(q, g), inputs.drift(k, g), inputs.drift(v, g)))
    return qkv


def reduce_over_ranks(total_ms, work, world, device):
    """(max over ranks of the timed region, sum over ranks of the work done).

    Every rank calls this with its own numbers; the whole-job value is the
    summed work over the slowest rank's time."""
    if world == 1:
        return float(total_ms), float(work)
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    w = torch.tensor([float(work)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(w, op=torch.distributed.ReduceOp.SUM)
    return float(t.item()), float(w.item())


def whole_job_tflops(work_all, ms_max):
    return work_all / (ms_max * 1e-3) / 1e12


def workload_config(wl, world):
    """The `config` object of both arms' JSON lines."""
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "grid": [wl.T, wl.Hh, wl.Ww], "d": wl.d,
            "block": wl.block, "eps": wl.eps, "mask": "all kept + LiteAttention skip chain",
            "l2": "inputs larger than L2 (3 x 774 MB per step)", "parallelism": f"replicas x{world}"}


def executed_flops(skip_in, N, block, d, mask=None):
    """4 * d * sum over visited (i, j) of valid rows_i * valid cols_j."""
    nb = -(-N // block)
    rows = torch.full((nb,), float(block), device=skip_in.device, dtype=torch.float64)
    rows[-1] = N - (nb - 1) * block
    vis = (1 - skip_in.to(torch.float64))
    if mask is not None:
        vis = vis * (mask != 0).to(torch.float64)
    per_bh = torch.einsum("i,bhij,j->bh", rows, vis, rows)
    return float(4.0 * d * per_bh.sum().item())


# ----------------------------------------------------------------- our arm ---

def run_ours(args, rank, world, local):
    from block_sparse_attention_flash_b200 import inputs, ops, build

    wl = inputs.WORKLOADS[args.workload]
    if wl.kind != "lite":
        raise SystemExit("bench.py times the LiteAttention chain workload")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    build.build()
    ops.lib()
    B, H, N, d, block, eps = wl.B, wl.H, wl.N, wl.d, wl.block, wl.eps
    nb = wl.nblocks
    nsteps = args.warmup + args.steps

    # Per-step inputs, drawn on the device before timing (the chain's drift).
    qkv = replica_chain(wl, rank, nsteps, dev)
    q0, k0, v0 = qkv[0]
    skips = [torch.zeros(B, H, nb, nb, dtype=torch.uint8, device=dev) for _ in range(nsteps + 1)]
    out = torch.empty_like(q0)
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nsteps)]

    def step(s):
        q, k, v = qkv[s]
        ev[s][0].record(stream)
        ops.sa_sparse_attn_fwd(q, k, v, block, mask=None, skip_in=skips[s], skip_out=skips[s + 1], eps=eps,
                               out=out, stream=stream)
        ev[s][1].record(stream)

    for s in range(args.warmup):
        step(s)
    ops.sa_get_device_status(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(args.warmup, nsteps):
        step(s)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    ops.sa_get_device_status(stream)
    total_ms = t0.elapsed_time(t1)
    kern_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(args.warmup, nsteps)]
    flops = [executed_flops(skips[s], N, block, d) for s in range(args.warmup, nsteps)]
    total_ms_max, flops_all = reduce_over_ranks(total_ms, sum(flops), world, dev)

    # end-to-end through the public API with host buffers, over the same drifted steps
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(ops, qkv, args.warmup, block, eps, nb, dev, stream, world)

    # the other workloads' paths and the eps = 2 chain (rank 0 of a single-GPU run)
    configs = None
    if rank == 0 and world == 1 and not args.no_configs:
        configs = {"lite_eps2_chain": lite_eps2_chain(ops, qkv, wl, dev, stream, statistics.median(kern_ms),
                                                      args.cpu_seconds_config)}
        del qkv
        torch.cuda.empty_cache()
        configs.update(run_configs(args, ops, dev, stream))
    else:
        del qkv

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        q, k, v = (t[:, :1].cpu() for t in (q0, k0, v0))
        cpu = cpu_sample(q, k, v, block, eps, args.cpu_seconds)

    if rank != 0:
        return None
    line = assemble_line(wl, world, args.steps, args.warmup, total_ms_max, flops_all, kern_ms, flops)
    line.update({"clocks": clk, "e2e": e2e, "cpu_baseline": cpu, "configs": configs})
    return line


def assemble_line(wl, world, steps, warmup, total_ms_max, flops_all, kern_ms, flops):
    """The JSON line of the device-timed run (rank 0): the whole-job value is
    the work summed over ranks divided by the slowest rank's timed region;
    the per-call figures and the roofline are rank 0's own launches."""
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    dense = 4.0 * d * N * N * B * H
    peaks, src = load_peaks()
    achieved = sum(flops) / (sum(kern_ms) * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    skip_rate = 1.0 - sum(flops) / (dense * len(flops))
    return {
        "metric": METRIC,
        "value": round(whole_job_tflops(flops_all, total_ms_max), 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(total_ms_max / steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded random-Fourier-feature locality generator + denoising drift, drawn on device)",
        "config": workload_config(wl, world),
        "ms_per_call": round(statistics.median(kern_ms), 3),
        "density": round(1.0 - skip_rate, 6),
        "executed_tflops": round(achieved, 2),
        "dense_equiv_tflops": round(dense / (statistics.median(kern_ms) * 1e-3) / 1e12, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_source": f"{src} bf16_tflops_sustained",
                     "frac_of_burst": round(achieved / float(peaks["bf16_tflops"]), 4),
                     "traffic": ATTN_DRAM_BYTES_PER_LAUNCH, "traffic_unit": "bytes per launch",
                     "algorithmic_bytes": 4 * B * H * N * d * 2},
        "gpu_launches": steps,
    }


E2E_HEADS_PER_CHUNK = 1   # measured: 1 head 95.9-96.6 ms per step, 2 heads 97.2-97.7 (same process), 4 heads 100.5, 8 heads 105


def run_e2e(ops, qkv, first, block, eps, nb, dev, stream, world):
    """Same metric through the public C-ABI call with host buffers
    (sa_sparse_attn_fwd_host), over the same drifted denoising steps as the
    device-timed value (steps first .. end of qkv) with the skip mask carried:
    every step copies that step's Q/K/V in from pinned host memory and O back
    out, inside the timed region; the library overlaps the copies of one chunk
    of heads with the attention of another.  One untimed warm-up call first."""
    steps = len(qkv) - first
    B, H, N, d = qkv[0][0].shape
    def pinned(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    host = [tuple(pinned(t) for t in qkv[s]) for s in range(first - 1, len(qkv))]
    ho = torch.empty_like(host[0][0]).pin_memory()
    ws = torch.empty(ops.sa_sparse_attn_fwd_host_workspace(N, d, min(E2E_HEADS_PER_CHUNK, H)), dtype=torch.uint8,
                     device=dev)
    skips = [torch.zeros(B, H, nb, nb, dtype=torch.uint8, device=dev) for _ in range(steps + 2)]

    def one(i):
        hq, hk, hv = host[i]
        ops.sa_sparse_attn_fwd_host(hq, hk, hv, block, out=ho, skip_in=skips[i], skip_out=skips[i + 1], eps=eps,
                                    heads_per_chunk=E2E_HEADS_PER_CHUNK, workspace=ws, stream=stream)

    one(0)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(1, steps + 1):
        one(i)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ops.sa_get_device_status(stream)
    ms = a.elapsed_time(b)
    ms, flops = reduce_over_ranks(ms, sum(executed_flops(skips[i], N, block, d) for i in range(1, steps + 1)),
                                  world, dev)
    n = qkv[0][0].numel()
    return {"value": round(whole_job_tflops(flops, ms), 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": 3 * n * 2, "d2h_bytes_per_step": n * 2,
            "ms_per_step": round(ms / steps, 3), "steps": steps,
            "inputs": "the same drifted denoising steps as the device-timed value, skip mask carried",
            "api": f"sa_sparse_attn_fwd_host, {E2E_HEADS_PER_CHUNK} heads per chunk"}


# ------------------------------------------------ the other workloads' paths ---

CONFIG_REPS = 10
LITE_DIAG_EPS = 2.0
LITE_DIAG_STEPS = 6


def lite_eps2_chain(ops, qkv, wl, dev, stream, ms_eps10, cpu_seconds):
    """Diagnostic, labelled: the same 75.6K-token chain at eps = 2 (the
    workload's eps = 10 skips nothing on this generator).  Step s consumes the
    skip bits of step s - 1, so its executed tiles fall; the time per step
    should fall with them (skipped tiles are neither loaded, multiplied nor
    exponentiated).  The oracle sample recomputes step 0 for q-blocks of
    head 0 and checks their skip rows."""
    B, H, N, d, block = wl.B, wl.H, wl.N, wl.d, wl.block
    nb = wl.nblocks
    n = min(LITE_DIAG_STEPS, len(qkv))
    skips = [torch.zeros(B, H, nb, nb, dtype=torch.uint8, device=dev) for _ in range(n + 1)]
    out = torch.empty_like(qkv[0][0])
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for s in range(n):                      # untimed pass: the chain's skip masks
        q, k, v = qkv[s]
        ops.sa_sparse_attn_fwd(q, k, v, block, skip_in=skips[s], skip_out=skips[s + 1], eps=LITE_DIAG_EPS, out=out,
                               stream=stream)
    torch.cuda.synchronize(dev)
    ms = []
    for rep in range(3):                    # timed: each step on its own skip_in (skip_out to a scratch mask)
        scratch = torch.empty_like(skips[0])
        for s in range(n):
            q, k, v = qkv[s]
            ev[s][0].record(stream)
            ops.sa_sparse_attn_fwd(q, k, v, block, skip_in=skips[s], skip_out=scratch, eps=LITE_DIAG_EPS, out=out,
                                   stream=stream)
            ev[s][1].record(stream)
        torch.cuda.synchronize(dev)
        ms.append([ev[s][0].elapsed_time(ev[s][1]) for s in range(n)])
    ops.sa_get_device_status(stream)
    dense = 4.0 * d * N * N * B * H
    per_step = []
    for s in range(n):
        t = statistics.median(m[s] for m in ms)
        fl = executed_flops(skips[s], N, block, d)
        per_step.append({"step": s, "ms": round(t, 3), "density": round(fl / dense, 4),
                         "executed_tflops": round(fl / t / 1e9, 1), "time_vs_eps10": round(t / ms_eps10, 4)})
    cpu = None
    if cpu_seconds > 0:
        q, k, v = (t[:, :1].cpu() for t in qkv[0])
        cpu = cpu_sample(q, k, v, block, LITE_DIAG_EPS, cpu_seconds, gpu_skip=skips[1][:, :1].cpu().numpy())
    return {"what": f"diagnostic: eps = {LITE_DIAG_EPS:g} instead of the workload's {wl.eps:g}, same inputs",
            "eps": LITE_DIAG_EPS, "ms_eps10": round(ms_eps10, 3), "steps": per_step, "cpu_baseline": cpu}


def run_configs(args, ops, dev, stream):
    """The three other workloads' hot paths, one entry each (device-timed,
    CUDA-event medians of CONFIG_REPS calls after 3 warm-ups)."""
    from block_sparse_attention_flash_b200 import inputs

    peaks, src = load_peaks()
    out = {}
    for name in ("wan13b_480p_tau", "hunyuan_720p_radial", "psa_480p_pyramid"):
        wl = inputs.WORKLOADS[name]
        q, k, v = inputs.rff_qkv(wl, device=dev)
        if wl.kind == "tau":
            out[name] = config_tau(ops, wl, q, k, v, dev, stream, peaks, src, args.cpu_seconds_config)
        elif wl.kind == "radial":
            out[name] = config_radial(ops, wl, q, k, v, dev, stream, peaks, src, args.cpu_seconds_config)
        else:
            out[name] = config_psa(ops, wl, q, k, v, dev, stream, peaks, src, args.cpu_seconds_config)
        ops.sa_get_device_status(stream)
        del q, k, v
        torch.cuda.empty_cache()
    return out


def _attn_entry(wl, ms, flops, peaks, src, algorithmic_flops=None):
    dense = 4.0 * wl.d * wl.N * wl.N * wl.B * wl.H
    alg = flops if algorithmic_flops is None else algorithmic_flops
    burst, sust = float(peaks["bf16_tflops"]), float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    tf = alg / ms / 1e9
    return {"ms_per_call": round(ms, 3), "density": round(alg / dense, 5), "executed_tflops": round(tf, 1),
            "dense_equiv_tflops": round(dense / ms / 1e9, 1),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": burst, "unit": "TFLOP/s",
                         "frac": round(tf / burst, 4), "frac_of_sustained": round(tf / sust, 4),
                         "peak_source": f"{src} bf16_tflops (burst: a kernel timed alone)"}}


def _hbm_entry(ms, nbytes, peaks, src):
    gbs = nbytes / ms / 1e6
    return {"ms_per_call": round(ms, 4), "roofline": {"bound": "hbm", "achieved": round(gbs, 1),
                                                      "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                                                      "frac": round(gbs / float(peaks["hbm_gbs"]), 4),
                                                      "algorithmic_bytes": nbytes, "peak_source": f"{src} hbm_gbs"}}


def config_tau(ops, wl, q, k, v, dev, stream, peaks, src, cpu_seconds):
    B, H, N, d = q.shape
    nb = wl.nblocks
    ws = torch.empty(ops.sa_build_mask_workspace(B, H, N, d, wl.block), dtype=torch.uint8, device=dev)
    m = torch.empty(B, H, nb, nb, dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    ms_m = _time(lambda: ops.sa_build_mask(q, k, wl.block, "tau", tau=wl.tau, mask_out=m, workspace=ws),
                 CONFIG_REPS, stream, SHORT_CALL_BATCH)
    ms_a = _time(lambda: ops.sa_sparse_attn_fwd(q, k, v, wl.block, mask=m, out=o), CONFIG_REPS, stream)
    flops = executed_flops(torch.zeros_like(m), N, wl.block, d, mask=m)
    mask_bytes = 2 * B * H * N * d * 2 + B * H * nb * nb
    entry = {"path": "sa_build_mask (tau) + sa_sparse_attn_fwd", "attention": _attn_entry(wl, ms_a, flops, peaks, src),
             "mask_builder": _hbm_entry(ms_m, mask_bytes, peaks, src)}
    # backward over the same mask (dQ, dK, dV from dO, O, LSE): algorithmic work is 5 GEMMs per
    # kept element (S, dP, dV, dK, dQ); the kernels execute 7 (S and dP again in the dQ pass)
    lse = torch.empty(B, H, N, device=dev)
    ops.sa_sparse_attn_fwd(q, k, v, wl.block, mask=m, out=o, lse=lse)
    gen = torch.Generator(device=dev).manual_seed(wl.seed + 11)
    dout = torch.randn(q.shape, generator=gen, device=dev).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bws = torch.empty(ops.sa_sparse_attn_bwd_workspace(B, H, N), dtype=torch.uint8, device=dev)
    ms_b = _time(lambda: ops.sa_sparse_attn_bwd(q, k, v, o, dout, lse, wl.block, mask=m, dq=dq, dk=dk, dv=dv,
                                                workspace=bws), CONFIG_REPS, stream)
    burst = float(peaks["bf16_tflops"])
    alg_tf = 2.5 * flops / ms_b / 1e9
    entry["backward"] = {"path": "sa_sparse_attn_bwd", "ms_per_call": round(ms_b, 3),
                         "algorithmic_tflops": round(alg_tf, 1),
                         "executed_tflops_7gemm": round(3.5 * flops / ms_b / 1e9, 1),
                         "roofline": {"bound": "tensor", "achieved": round(alg_tf, 1), "peak": burst,
                                      "unit": "TFLOP/s", "frac": round(alg_tf / burst, 4),
                                      "peak_source": f"{src} bf16_tflops (burst: a kernel timed alone)"}}
    del dout, dq, dk, dv, bws, lse
    # token permutation of Q, K, V: per-head PARO axis orders and 3 x 5 x 4 VMoBA cells
    orders = (torch.arange(H, device=dev) % 6).to(torch.uint8)
    pout = [torch.empty_like(q) for _ in range(3)]
    ms_p = _time(lambda: ops.sa_token_permute([q, k, v], wl.T, wl.Hh, wl.Ww, head_order=orders, cells=(3, 5, 4),
                                              out=pout), CONFIG_REPS, stream, SHORT_CALL_BATCH)
    entry["permute_qkv"] = dict(path="sa_token_permute", **_hbm_entry(ms_p, 2 * 3 * B * H * N * d * 2, peaks, src))
    del pout
    if cpu_seconds > 0:
        entry["cpu_baseline"] = cpu_config_sample(wl, q, k, v, m, cpu_seconds, "tau")
    return entry


def config_radial(ops, wl, q, k, v, dev, stream, peaks, src, cpu_seconds):
    B, H, N, d = q.shape
    nb = wl.nblocks
    rm = ops.sa_radial_mask(wl.T, wl.Hh, wl.Ww, wl.block)
    o = torch.empty_like(q)
    ms_r = _time(lambda: ops.sa_radial_mask(wl.T, wl.Hh, wl.Ww, wl.block, out=rm), CONFIG_REPS, stream,
                 SHORT_CALL_BATCH)
    ms_a = _time(lambda: ops.sa_sparse_attn_fwd(q, k, v, wl.block, mask=rm, out=o), CONFIG_REPS, stream)
    m4 = rm.view(1, 1, nb, nb).expand(B, H, nb, nb)
    flops = executed_flops(torch.zeros(B, H, nb, nb, dtype=torch.uint8, device=dev), N, wl.block, d, mask=m4)
    entry = {"path": "sa_radial_mask + sa_sparse_attn_fwd", "attention": _attn_entry(wl, ms_a, flops, peaks, src),
             "radial_mask": _hbm_entry(ms_r, nb * nb, peaks, src)}
    if cpu_seconds > 0:
        entry["cpu_baseline"] = cpu_config_sample(wl, q, k, v, rm, cpu_seconds, "radial")
    return entry


def pyramid_flops(lv, N, block, d):
    """Algorithmic pyramid work: 4 d x valid rows x pooled keys of each (i, j) at its level."""
    B, H, nb, _ = lv.shape
    rows = torch.full((nb,), float(block), device=lv.device, dtype=torch.float64)
    rows[-1] = N - (nb - 1) * block
    cols = torch.zeros(B, H, nb, nb, dtype=torch.float64, device=lv.device)
    for lvl in range(4):
        cnt = torch.full((nb,), float(block >> lvl), device=lv.device, dtype=torch.float64)
        cnt[-1] = -(-int(rows[-1].item()) // (1 << lvl))
        cols += (lv == lvl + 1).to(torch.float64) * cnt.view(1, 1, 1, nb)
    return float(4.0 * d * torch.einsum("i,bhij->", rows, cols).item())


def config_psa(ops, wl, q, k, v, dev, stream, peaks, src, cpu_seconds):
    B, H, N, d = q.shape
    nb = wl.nblocks
    ws = torch.empty(ops.sa_build_mask_workspace(B, H, N, d, wl.block), dtype=torch.uint8, device=dev)
    lv = torch.empty(B, H, nb, nb, dtype=torch.uint8, device=dev)
    kp, vp = ops.sa_pyramid_pool(k, v, wl.block)
    o = torch.empty_like(q)
    ms_l = _time(lambda: ops.sa_build_mask(q, k, wl.block, "levels", level_frac=wl.level_frac, mask_out=lv,
                                           workspace=ws), CONFIG_REPS, stream, SHORT_CALL_BATCH)
    ms_p = _time(lambda: ops.sa_pyramid_pool(k, v, wl.block, k_pool=kp, v_pool=vp), CONFIG_REPS, stream,
                 SHORT_CALL_BATCH)
    ms_a = _time(lambda: ops.sa_pyramid_attn_fwd(q, k, v, wl.block, lv, kp, vp, out=o), CONFIG_REPS, stream)
    flops = pyramid_flops(lv, N, wl.block, d)
    kv_bytes = 2 * B * H * N * d * 2
    entry = {"path": "sa_build_mask (levels) + sa_pyramid_pool + sa_pyramid_attn_fwd",
             "attention": _attn_entry(wl, ms_a, flops, peaks, src),
             "level_map": _hbm_entry(ms_l, kv_bytes + B * H * nb * nb, peaks, src),
             "pool": _hbm_entry(ms_p, kv_bytes + kv_bytes * 7 // 8, peaks, src)}
    if cpu_seconds > 0:
        entry["cpu_baseline"] = cpu_config_sample(wl, q, k, v, lv, cpu_seconds, "levels")
    return entry


# -------------------------------------------------------------- suite mode ---

SHORT_CALL_BATCH = 10   # calls per timed batch for the sub-millisecond paths


def _time(fn, reps, stream, batch=1):
    """Median ms per call of `fn` (CUDA events on `stream`), after 3 warm-ups.

    With batch > 1 each timed sample is `batch` calls issued back to back and
    divided by `batch`: for paths of about 0.1 ms the host-side argument
    marshalling of a single call (tens of microseconds, during which the GPU
    would sit idle inside the timed region) overlaps the previous call's
    kernels instead of being counted as device time."""
    for _ in range(3):
        fn()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(batch):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / batch)
    return statistics.median(ts)


def run_suite(args):
    """Every workload's hot path on one GPU: one JSON line per workload."""
    from block_sparse_attention_flash_b200 import inputs, ops, build

    build.build()
    ops.lib()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks, src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    tens = float(peaks["bf16_tflops"])
    out = []

    def attn_line(wl, name, ms, flops, extra):
        dense = 4.0 * wl.d * wl.N * wl.N * wl.B * wl.H
        d = {"workload": name, "N": wl.N, "H": wl.H, "d": wl.d, "block": wl.block, "ms_per_call": round(ms, 3),
             "density": round(flops / dense, 5), "executed_tflops": round(flops / ms / 1e9, 1),
             "dense_equiv_tflops": round(dense / ms / 1e9, 1),
             "frac_of_bf16_burst": round(flops / ms / 1e9 / tens, 4), "peak_source": src}
        d.update(extra)
        return d

    for name in ("wan13b_480p_tau", "hunyuan_720p_radial", "wan14b_720p_lite", "psa_480p_pyramid"):
        wl = inputs.WORKLOADS[name]
        q, k, v = inputs.rff_qkv(wl, device=dev)
        nb = wl.nblocks
        B, H, N, d = q.shape
        o = torch.empty_like(q)
        qk_bytes = 2 * B * H * N * d * 2
        if wl.kind == "tau":
            ws = torch.empty(ops.sa_build_mask_workspace(B, H, N, d, wl.block), dtype=torch.uint8, device=dev)
            m = torch.empty(B, H, nb, nb, dtype=torch.uint8, device=dev)
            ms_m = _time(lambda: ops.sa_build_mask(q, k, wl.block, "tau", tau=wl.tau, mask_out=m, workspace=ws),
                         args.suite_reps, stream, SHORT_CALL_BATCH)
            ms_a = _time(lambda: ops.sa_sparse_attn_fwd(q, k, v, wl.block, mask=m, out=o), args.suite_reps, stream)
            flops = executed_flops(torch.zeros_like(m), N, wl.block, d, mask=m)
            out.append(attn_line(wl, name, ms_a, flops, {
                "mask_ms": round(ms_m, 4), "mask_gbs": round(qk_bytes / ms_m / 1e6, 1),
                "mask_frac_of_hbm": round(qk_bytes / ms_m / 1e6 / hbm, 4)}))
            # backward pass over the same mask (dQ, dK, dV from dO, O, LSE)
            lse = torch.empty(B, H, N, device=dev)
            ops.sa_sparse_attn_fwd(q, k, v, wl.block, mask=m, out=o, lse=lse)
            gen = torch.Generator(device=dev).manual_seed(wl.seed + 11)
            dout = torch.randn(q.shape, generator=gen, device=dev).to(torch.bfloat16)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            bws = torch.empty(ops.sa_sparse_attn_bwd_workspace(B, H, N), dtype=torch.uint8, device=dev)
            ms_b = _time(lambda: ops.sa_sparse_attn_bwd(q, k, v, o, dout, lse, wl.block, mask=m, dq=dq, dk=dk, dv=dv,
                                                        workspace=bws), args.suite_reps, stream)
            # algorithmic backward work: 5 GEMMs (dV, dP, dS K, dS^T Q and the recomputed S) per kept
            # element; the kernels execute 7 (S and dP are recomputed in the dQ pass)
            out.append(attn_line(wl, name + "_backward", ms_b, 2.5 * flops, {
                "executed_tflops_7gemm": round(3.5 * flops / ms_b / 1e9, 1)}))
            # token permutation of Q, K, V: per-head PARO axis orders, 3 x 5 x 4 cells
            orders = (torch.arange(H, device=dev) % 6).to(torch.uint8)
            pout = [torch.empty_like(q) for _ in range(3)]
            ms_p = _time(lambda: ops.sa_token_permute([q, k, v], wl.T, wl.Hh, wl.Ww, head_order=orders, cells=(3, 5, 4),
                                                      out=pout), args.suite_reps, stream, SHORT_CALL_BATCH)
            pbytes = 2 * 3 * B * H * N * d * 2
            out.append({"workload": name + "_permute_qkv", "N": N, "H": H, "d": d, "ms_per_call": round(ms_p, 4),
                        "gbs": round(pbytes / ms_p / 1e6, 1), "frac_of_hbm": round(pbytes / ms_p / 1e6 / hbm, 4),
                        "peak_source": src})
        elif wl.kind == "radial":
            rm = ops.sa_radial_mask(wl.T, wl.Hh, wl.Ww, wl.block)
            ms_r = _time(lambda: ops.sa_radial_mask(wl.T, wl.Hh, wl.Ww, wl.block, out=rm), args.suite_reps, stream,
                         SHORT_CALL_BATCH)
            ms_a = _time(lambda: ops.sa_sparse_attn_fwd(q, k, v, wl.block, mask=rm, out=o), args.suite_reps, stream)
            m4 = rm.view(1, 1, nb, nb).expand(B, H, nb, nb)
            flops = executed_flops(torch.zeros(B, H, nb, nb, dtype=torch.uint8, device=dev), N, wl.block, d,
                                   mask=m4)
            out.append(attn_line(wl, name, ms_a, flops, {"radial_mask_ms": round(ms_r, 4)}))
        elif wl.kind == "lite":
            skip_a = torch.zeros(B, H, nb, nb, dtype=torch.uint8, device=dev)
            skip_b = torch.zeros_like(skip_a)
            ms_a = _time(lambda: ops.sa_sparse_attn_fwd(q, k, v, wl.block, skip_in=skip_a, skip_out=skip_b,
                                                        eps=wl.eps, out=o), args.suite_reps, stream)
            flops = executed_flops(skip_a, N, wl.block, d)
            skipped = int(skip_b.sum())
            ms_r = _time(lambda: ops.sa_sparse_attn_fwd(q, k, v, wl.block, skip_in=skip_a, skip_out=skip_b,
                                                        eps=wl.eps, out=o, order="radial"), args.suite_reps, stream)
            # diagnostic, clearly not the workload's eps: the share of (q-block, k-block)
            # pairs that the first step marks for skipping, per visit order and eps
            diag = {}
            for order in ("ascending", "radial"):
                for e in (2.0, 3.0, wl.eps):
                    ops.sa_sparse_attn_fwd(q, k, v, wl.block, skip_in=skip_a, skip_out=skip_b, eps=e, out=o,
                                           order=order)
                    diag[f"{order}_eps{e:g}"] = round(int(skip_b.sum()) / skip_b.numel(), 5)
            out.append(attn_line(wl, name, ms_a, flops, {"eps": wl.eps, "skipped_next_step": skipped,
                                                         "radial_order_ms": round(ms_r, 3),
                                                         "skip_share_diagnostic": diag}))
        else:
            kp, vp = ops.sa_pyramid_pool(k, v, wl.block)
            ms_p = _time(lambda: ops.sa_pyramid_pool(k, v, wl.block, k_pool=kp, v_pool=vp), args.suite_reps, stream,
                         SHORT_CALL_BATCH)
            lv = ops.sa_build_mask(q, k, wl.block, "levels", level_frac=wl.level_frac)
            ms_a = _time(lambda: ops.sa_pyramid_attn_fwd(q, k, v, wl.block, lv, kp, vp, out=o), args.suite_reps,
                         stream)
            flops = pyramid_flops(lv, N, wl.block, d)
            pool_bytes = qk_bytes + qk_bytes * 7 // 8
            out.append(attn_line(wl, name, ms_a, flops, {
                "pool_ms": round(ms_p, 4), "pool_gbs": round(pool_bytes / ms_p / 1e6, 1),
                "pool_frac_of_hbm": round(pool_bytes / ms_p / 1e6 / hbm, 4)}))
        ops.sa_get_device_status()
        del q, k, v, o
        torch.cuda.empty_cache()
    for line in out:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ oracle timing ---

def _threads():
    from threadpoolctl import threadpool_info
    return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])


def _bit_check(got, want, flags=None):
    """Counts of a GPU-vs-oracle mask comparison (flags: the oracle's margin flags)."""
    import numpy as np
    bad = np.asarray(got) != np.asarray(want)
    out = {"bits": int(bad.size), "mismatches": int(bad.sum())}
    if flags is not None:
        f = np.asarray(flags, dtype=bool)
        out.update({"flagged": int(f.sum()), "flagged_mismatches": int((bad & f).sum()),
                    "unflagged_mismatches": int((bad & ~f).sum())})
    return out


def cpu_sample(q, k, v, block, eps, seconds, gpu_skip=None):
    """Time the fp64 oracle's lite_step on q-blocks of head 0, step 0, for about
    `seconds` of host time; report its executed TFLOP/s.  With gpu_skip (the
    GPU's skip_out of that step for head 0) the oracle's skip rows of the
    sampled q-blocks are compared with it (bit counts, margin-flag aware)."""
    import numpy as np
    import oracle

    N, d = q.shape[2], q.shape[3]
    nb = -(-N // block)
    order = list(range(0, nb, max(1, nb // 64)))
    done, flops = 0, 0.0
    got, want, flags = [], [], []
    t0 = time.perf_counter()
    for i in order:
        ref = oracle.lite_step(q, k, v, block, None, None, eps, qblocks=[(0, 0, i)])
        rows = min(block, N - i * block)
        flops += 4.0 * d * rows * N
        done += 1
        if gpu_skip is not None:
            _, _, srow, mrow = ref[(0, 0, i)]
            got.append(gpu_skip[0, 0, i]), want.append(srow), flags.append(oracle.skip_flags(mrow))
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    out = {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
           "sample": f"{done} q-blocks of head 0 at denoising step 0 (all {N} keys each), {dt:.1f} s"}
    if gpu_skip is not None:
        out["skip_check"] = _bit_check(np.stack(got), np.stack(want), np.stack(flags))
    return out


def cpu_config_sample(wl, q, k, v, gpu_mask, seconds, kind):
    """The oracle on head 0 of one workload: its mask builder (timed, and its
    mask compared with the GPU's, margin-flag aware), then its attention on
    its own mask for q-blocks spread over the sequence, for about `seconds`;
    the value is executed TFLOP/s of the attention (algorithmic work)."""
    import numpy as np
    import oracle

    qh, kh, vh = (t[:, :1].cpu() for t in (q, k, v))
    N, d, block = wl.N, wl.d, wl.block
    nb = wl.nblocks
    t0 = time.perf_counter()
    if kind == "tau":
        ref, flags, _ = oracle.tau_mask(qh, kh, block, wl.tau, return_info=True)
    elif kind == "levels":
        ref, flags, _ = oracle.level_map(qh, kh, block, wl.level_frac, return_info=True)
    else:
        ref, flags = oracle.radial_mask(wl.T, wl.Hh, wl.Ww, block)[None, None], None
    t_mask = time.perf_counter() - t0
    g = gpu_mask.cpu().numpy()
    g = g[:1, :1] if g.ndim == 4 else g[None, None]
    check = _bit_check(g, ref, flags)
    valid = np.full(nb, block, dtype=np.int64)
    valid[-1] = N - (nb - 1) * block
    order = list(range(0, nb, max(1, nb // 64)))
    done, flops = 0, 0.0
    t0 = time.perf_counter()
    for i in order:
        if kind == "levels":
            oracle.pyramid_attention(qh, kh, vh, block, ref, qblocks=[(0, 0, i)])
            cols = sum(-(-int(valid[j]) // (1 << (int(ref[0, 0, i, j]) - 1))) for j in range(nb) if ref[0, 0, i, j])
        else:
            oracle.masked_attention(qh, kh, vh, block, ref, qblocks=[(0, 0, i)])
            cols = int(valid[ref[0, 0, i] != 0].sum())
        flops += 4.0 * d * int(valid[i]) * cols
        done += 1
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"mask builder on head 0 ({t_mask:.1f} s), then attention on the oracle's mask for {done} "
                      f"q-blocks of head 0 ({dt:.1f} s)",
            "mask_check": check}


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step a bounded sample of the workload."""
    from block_sparse_attention_flash_b200 import inputs

    if rank != 0:
        return None
    wl = inputs.WORKLOADS[args.workload]
    q, k, v = inputs.rff_qkv(wl, H=1)
    per_step = max(1.0, args.ref_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_sample(q, k, v, wl.block, wl.eps, per_step)
    vals = []
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_sample(q, k, v, wl.block, wl.eps, per_step)
        vals.append(last["value"])
    dt = time.perf_counter() - t0
    value = statistics.mean(vals)
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / max(1, args.steps), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded random-Fourier-feature locality generator)", "impl": "reference",
            "config": workload_config(wl, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan14b_720p_lite")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' entries")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--cpu-seconds-config", type=float, default=5.0,
                    help="oracle seconds per entry of `configs` (0: no oracle sample there)")
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    ap.add_argument("--suite", action="store_true", help="time every workload's hot path (one line each)")
    ap.add_argument("--suite-reps", type=int, default=10)
    args = ap.parse_args()
    if args.suite:
        run_suite(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_env()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=torch.device("cuda", local))
        line = run_ours(args, rank, world, local)
        if world > 1:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
