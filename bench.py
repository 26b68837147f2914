"""Benchmark of the fused Gaussian-mixture EM step on B200.

A step is one EM iteration (log-sum-exp sweep, statistics sweep, M-step) over the
whole resident X.  Default workload: N = 100,000,000, D = 128, K = 1024, diagonal
model, fp32 X (51.2 GB resident in HBM, far larger than L2), the Table-1 generator
of synth/ with seed = rank.  Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload table1-1e8|table1-1e6|c1] [--prec auto|fp32|fp16x3]

Multi-GPU (torchrun, one process per GPU): the ranks fit ONE mixture to the union
of their row shards, each rank holding the full per-rank size (weak scaling).  A
step is fgmm_em_partial on every shard, one NCCL all-gather of the statistics
vectors (K (1 + 2D) + 1 doubles), a rank-ordered sum and fgmm_em_finish on every
rank; the timing is reduced as the max over ranks, and one step over W ranks counts
as W units of the per-GPU metric.
--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only), its rows sharded over one worker process per host core,
and scales it to the metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "table1-1e8": dict(gen="table1", N=100_000_000, D=128, K=1024),
    "table1-1e6": dict(gen="table1", N=1_000_000, D=128, K=1024),
    "table1-1e5": dict(gen="table1", N=100_000, D=128, K=1024),
    "c1": dict(gen="c1", N=10_000, D=16, K=16),
    "ivf-1e7": dict(gen="ivf", N=10_000_000, D=128, K=4096),
    "border-1e6": dict(gen="border", N=1_000_000, D=960, K=256),
}
METRIC = "EM iters/s at N=100M,K=1024,D=128 fp32"


def workload_name(w):
    return f"{w['gen']} N={w['N']} D={w['D']} K={w['K']} diag fp32"


# ------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 7:
                continue
            try:
                sm.append(float(p[0]))
                mx.append(float(p[1]))
            except ValueError:
                continue
            for nm, v in zip(names, p[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(dev: int) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


# ------------------------------------------------------------------------------- peaks
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}, "fallback"


def kernel_source_hash() -> str:
    """Hash of the source text of the two tensor-core sweep kernels (the part of
    fgmm_tc.cu from the sweep-1 section to the end of the sweep-2 section) and of the
    PTX wrappers they use: recorded ncu traffic is reported only while these match."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ivf_quantizer_b200", "csrc")
    with open(os.path.join(csrc, "fgmm_tc.cu")) as fh:
        text = fh.read()
    a = text.find("// ------------------------------------------------------------------ sweep 1")
    b = text.find("// ------------------------------------------------------------------ bounded-wait")
    h.update(text[a:b].encode())
    with open(os.path.join(csrc, "sm100_ptx.cuh"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, prec: str):
    """Per-launch DRAM bytes of `kernel` from a committed ncu summary, or None when
    the summary was taken on other kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    e = rec.get(f"{prec}/{kernel}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


# ------------------------------------------------------------------------------- CPU oracle
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_worker_init():
    # one BLAS thread per worker process: the pool already has one process per core
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # pragma: no cover
        pass


def _oracle_shard(args):
    """Worker: the oracle's statistics of one row shard (runs in a spawned process)."""
    X, w, mu, var = args
    from oracle import gmm_oracle as O
    return O.shard_statistics(X, w, mu, var)


class OraclePool:
    """The fp64 oracle as it stands, on every core of the host: one EM step over a
    sample of rows is the oracle's shard_statistics on row shards in a pool of worker
    processes (one per core, started with spawn), summed in shard order, then its
    m_step_from_statistics.  Workers are started (and import NumPy) before any timing."""

    ROWS = 2048   # rows per shard

    def __init__(self, procs=None):
        import multiprocessing as mp
        self.procs = max(1, procs or host_cores())
        self.pool = mp.get_context("spawn").Pool(self.procs, initializer=_oracle_worker_init)
        self.pool.map(_oracle_shard, [(np.zeros((1, 1)), np.ones(1), np.zeros((1, 1)),
                                       np.ones((1, 1)))] * self.procs)

    def step_time(self, w, sample_n: int, seed: int = 0) -> float:
        import synth
        from oracle import gmm_oracle as O
        X = synth.generate(w["gen"], sample_n, seed=seed)
        wt, mu, var = synth.init_params(X, w["K"], seed=seed)
        Xn = X.double().numpy()
        wt, mu, var = wt.double().numpy(), mu.double().numpy(), var.double().numpy()
        jobs = [(Xn[a:a + self.ROWS], wt, mu, var) for a in range(0, sample_n, self.ROWS)]
        t0 = time.perf_counter()
        parts = self.pool.map(_oracle_shard, jobs, chunksize=1)
        st = np.zeros_like(parts[0])
        for p in parts:
            st += p
        O.m_step_from_statistics(st, wt, mu, var)
        return time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()


def oracle_sample_size(w, procs: int, target_s=15.0):
    # the oracle's cost is ~ N*K*D fp64 element operations, ~6.5 ns each per core
    per_point = w["K"] * w["D"] * 6.5e-9
    n = int(max(64, min(w["N"], procs * target_s / per_point)))
    n = max(w["K"], n)
    if n > OraclePool.ROWS:
        n = -(-n // OraclePool.ROWS) * OraclePool.ROWS
    return min(n, w["N"])


def cpu_baseline_line(w, dt: float, n_s: int, procs: int) -> dict:
    N = w["N"]
    return {"value": 1.0 / (dt * N / n_s), "unit": "iters/s", "cores": procs, "kind": "oracle",
            "cpu_model": cpu_model(), "extrapolated": n_s < N,
            "sample": f"one fp64 oracle EM step on {n_s} of {N} points (K={w['K']}, D={w['D']}), "
                      f"rows sharded over {procs} worker processes, {dt:.1f} s, "
                      f"scaled by N/{n_s}"}


# ------------------------------------------------------------------------------- main
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="table1-1e8", choices=sorted(WORKLOADS))
    ap.add_argument("--prec", default="auto", choices=["auto", "fp32", "fp16x3", "fp16"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-block-skip", action="store_true",
                    help="dense statistics sweep on the tensor cores (fgmm_set_block_skip 0)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--mode", default="em", choices=["em", "kmeans", "assign"],
                    help="kmeans: time Lloyd iterations of the warm start; assign: time the "
                         "top-2 soft assignment (r > 0.1) after the EM steps")
    return ap.parse_args()


def run_reference(args, w):  # noqa: C901
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    pool = OraclePool()
    n_s = oracle_sample_size(w, pool.procs,
                             target_s=max(2.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        pool.step_time(w, min(n_s, pool.procs * OraclePool.ROWS))
    times = []
    for _ in range(args.steps):
        dt = pool.step_time(w, n_s)
        times.append(dt * w["N"] / n_s)
    pool.close()
    t_step = sum(times) / len(times)
    value = 1.0 / t_step
    cpu = cpu_baseline_line(w, t_step * n_s / w["N"], n_s, pool.procs)
    metric = METRIC if args.workload == "table1-1e8" else f"EM iters/s ({args.workload})"
    line = {"impl": "reference", "metric": metric, "value": value, "unit": "iters/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(w)},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": "iters/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_kmeans(args, w):
    """Lloyd iterations of the k-means warm start on the same workload (rank 0 only)."""
    import torch

    import ivf_quantizer_b200 as q
    import synth
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    N, D, K = w["N"], w["D"], w["K"]
    X = torch.empty(N, D, device="cuda", dtype=torch.float32)
    synth.generate(w["gen"], N, seed=0, device="cuda", out=X)
    g = q.GMM(K, D)
    gen = torch.Generator(device="cuda").manual_seed(0)
    C = X[torch.randperm(N, device="cuda", generator=gen)[:K]].contiguous()
    inertia = torch.zeros(1, dtype=torch.float64, device="cuda")
    for _ in range(args.warmup):
        g.kmeans_step(X, C, inertia=inertia)
    torch.cuda.synchronize()
    g.check_status()
    sampler = ClockSampler(gpu_id_for(0))
    sampler.start()
    time.sleep(0.3)
    g.profile(True)
    g.profile_read(reset=True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        g.kmeans_step(X, C, inertia=inertia)
    b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    kern = g.profile_read(reset=True)["kernels"].get("km_assign", {"active": 1, "active_ms": 0})
    g.profile(False)
    ms = a.elapsed_time(b)
    peaks, _ = measured_peaks()
    clk = float(peaks.get("sm_max_mhz", 1965.0))
    n_chunks = -(-N // q.CHUNK_POINTS)
    ops = 3.0 * (N / n_chunks) * K * D            # subtract, square, add per (point, centroid, dim)
    avg = kern["active_ms"] / max(1, kern["active"])
    peak = 148 * 128 * clk * 1e6 / 1e12             # one fp32 op per lane per clock (no FMA)
    line = {"metric": f"k-means Lloyd iters/s ({args.workload})", "value": args.steps / (ms / 1e3),
            "unit": "iters/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "dtype": "f32",
            "data": "synthetic", "config": {"workload": workload_name(w), "mode": "kmeans"},
            "roofline": {"bound": "alu", "kernel": "km_assign", "unit": "Tops/s",
                         "achieved": ops / (avg / 1e3) / 1e12, "peak": peak,
                         "frac": ops / (avg / 1e3) / 1e12 / peak, "avg_launch_ms": avg,
                         "peak_note": f"148 SMs x 128 lanes x {clk:.0f} MHz, one fp32 op each"},
            "inertia_last": float(inertia.item()), "clocks": clocks}
    print(json.dumps(line), flush=True)
    g.close()
    return 0


def run_assign(args, w):
    """fgmm_soft_assign (top_m = 2, r_threshold = 0.1, the IVF multi-assignment) timed on
    the workload after `warmup` EM steps (rank 0 only).  One step = one assignment of
    all N points: the tensor-core sweep marks each point's candidate component blocks,
    the CUDA-core kernel evaluates those exactly."""
    import torch

    import ivf_quantizer_b200 as q
    import synth
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    N, D, K = w["N"], w["D"], w["K"]
    X = torch.empty(N, D, device="cuda", dtype=torch.float32)
    synth.generate(w["gen"], N, seed=0, device="cuda", out=X)
    wt, mu, var = synth.init_params(X, K, seed=0)
    g = q.GMM(K, D)
    wd, md, vd = g.new_params(wt, mu, var)
    for _ in range(args.warmup):
        g.step(X, wd, md, vd)
    ids = torch.empty(N, 2, dtype=torch.int32, device="cuda")
    resp = torch.empty(N, 2, dtype=torch.float32, device="cuda")
    g.soft_assign(X, wd, md, vd, top_m=2, r_threshold=0.1, ids=ids, resp=resp)
    torch.cuda.synchronize()
    g.check_status()
    sampler = ClockSampler(gpu_id_for(0))
    sampler.start()
    time.sleep(0.3)
    g.profile(True)
    g.profile_read(reset=True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        g.soft_assign(X, wd, md, vd, top_m=2, r_threshold=0.1, ids=ids, resp=resp)
    b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    kern = g.profile_read(reset=True)["kernels"]
    g.profile(False)
    ms = a.elapsed_time(b) / args.steps
    peaks, peak_src = measured_peaks()
    multi = float((ids[:, 1] >= 0).float().mean().item())
    n_chunks = -(-N // q.CHUNK_POINTS)
    by_kernel = {k: round(v["ms"] / args.steps, 3) for k, v in
                 sorted(kern.items(), key=lambda kv: -kv[1]["ms"])}
    line = {"metric": f"soft assignments/s ({args.workload}, top_m=2, r>0.1)",
            "value": N / (ms / 1e3), "unit": "points/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "f32",
            "data": "synthetic", "config": {"workload": workload_name(w), "mode": "assign"},
            "step_ms_by_kernel": by_kernel, "second_assignment_fraction": multi,
            "clocks": clocks}
    if "tc_lse" in kern:
        lse = kern["tc_lse"]
        avg = lse["ms"] / max(1, lse["launches"])
        flops = 4.0 * D * K * (N / n_chunks)          # the filter sweep: 4 D per point-component
        peak = float(peaks["bf16_tflops_sustained"])
        line["roofline"] = {"bound": "tensor", "kernel": "tc_lse", "unit": "TFLOP/s",
                            "achieved": flops / (avg / 1e3) / 1e12, "peak": peak,
                            "frac": flops / (avg / 1e3) / 1e12 / peak, "avg_launch_ms": avg,
                            "peak_source": peak_src,
                            "peak_note": "fp16 dense = bf16 dense (measured, sustained); "
                                         "algorithmic 4*D flops per point-component"}
        line["path"] = "tensor-core filter + exact CUDA-core evaluation of the marked blocks"
    else:
        clk = float(peaks.get("sm_max_mhz", 1965.0))
        flops = 3.0 * N * K * D
        peak = 148 * 128 * 2 * clk * 1e6 / 1e12
        line["roofline"] = {"bound": "alu", "kernel": "soft_assign", "unit": "TFLOP/s",
                            "achieved": flops / (ms / 1e3) / 1e12, "peak": peak,
                            "frac": flops / (ms / 1e3) / 1e12 / peak}
        line["path"] = "CUDA cores, every component"
    print(json.dumps(line), flush=True)
    g.close()
    return 0


def main():
    args = parse()
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.mode == "kmeans":
        return run_kmeans(args, w)
    if args.mode == "assign":
        return run_assign(args, w)

    import torch
    import torch.distributed as dist

    import ivf_quantizer_b200 as q
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    N, D, K = w["N"], w["D"], w["K"]
    prec = {"auto": q.PREC_AUTO, "fp32": q.PREC_FP32, "fp16x3": q.PREC_FP16X3,
            "fp16": q.PREC_FP16}[args.prec]
    X = torch.empty(N, D, device=dev, dtype=torch.float32)
    synth.generate(w["gen"], N, seed=rank, device=dev, out=X)
    # every rank starts from rank 0's initial parameters: the ranks fit ONE mixture to
    # the union of their shards (one statistics exchange per step)
    wt, mu, var = synth.init_params(X, K, seed=0)
    g = q.GMM(K, D)
    try:
        g.set_precision(prec)
    except q.FgmmError:
        g.set_precision(q.PREC_FP32)
    prec_set = {q.PREC_FP32: "fp32", q.PREC_FP16X3: "fp16x3", q.PREC_AUTO: "auto",
                q.PREC_FP16: "fp16"}[g.precision]
    g.set_block_skip(not args.no_block_skip)
    wd, md, vd = g.new_params(wt, mu, var)
    if world > 1:
        for t in (wd, md, vd):
            dist.broadcast(t, src=0)
    ll = torch.zeros(1, dtype=torch.float64, device=dev)
    from ivf_quantizer_b200 import dist as shard

    def em_step(Xs, w_, m_, v_):
        if world > 1:
            shard.sharded_step(g, Xs, w_, m_, v_, loglik=ll)
        else:
            g.step(Xs, w_, m_, v_, loglik=ll)

    for _ in range(args.warmup):
        em_step(X, wd, md, vd)
    torch.cuda.synchronize()
    g.check_status()
    barrier()

    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    time.sleep(0.3)
    g.profile(True)
    g.profile_read(reset=True)
    stream = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    t0.record(stream)
    for _ in range(args.steps):
        em_step(X, wd, md, vd)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    prof = g.profile_read(reset=True)
    g.profile(False)
    g.check_status()
    ms = t0.elapsed_time(t1)
    ms_t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    iters_per_s = world * args.steps / (ms_max / 1e3)

    # ---- roofline of the dominant kernel (per launch, live CUDA-event durations)
    # Under AUTO a step enqueues both paths' kernels and the other path's return at
    # their gate; only the launches that did work ("active") enter the per-launch time.
    peaks, peak_src = measured_peaks()
    kern = prof["kernels"]
    sweeps = {"tc_lse": "sweep1", "tc_stats": "sweep2", "lse_simt": "sweep1",
              "stats_simt": "sweep2"}
    dom = max(sweeps, key=lambda k: kern.get(k, {}).get("active_ms", 0.0))
    kd = kern.get(dom, {"active": 0, "active_ms": 0.0})
    launches = kd["active"]
    avg_ms = kd["active_ms"] / max(1, launches)
    n_chunks = -(-N // q.CHUNK_POINTS)
    pts_per_launch = N / n_chunks                       # one launch = one chunk of points
    flops_per_launch = 4.0 * D * K * pts_per_launch     # each sweep: 4*D flops per (point, comp)
    achieved = flops_per_launch / (avg_ms / 1e3) / 1e12 if launches else 0.0
    prec_used = ("fp16" if prec_set == "fp16" else "fp16x3") if dom.startswith("tc_") else "fp32"
    if prec_used == "fp32":
        clk = float(peaks.get("sm_max_mhz", 1965.0))
        peak = 148 * 128 * 2 * clk * 1e6 / 1e12
        roof = {"bound": "alu", "unit": "TFLOP/s", "peak_note":
                f"fp32 FMA: 148 SMs x 128 lanes x 2 x {clk:.0f} MHz"}
    else:
        peak = float(peaks["bf16_tflops_sustained"])
        roof = {"bound": "tensor", "unit": "TFLOP/s", "peak_note":
                f"fp16 dense peak = bf16 dense, {peak_src}, sustained; algorithmic flops "
                f"(4*D per point-component per sweep); the split products "
                f"({3 if prec_used == 'fp16x3' else 1} per term) and the recompute are not "
                f"counted"}
    traffic = recorded_traffic(dom, prec_used)
    roof.update({"kernel": dom, "achieved": achieved, "peak": peak,
                 "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                 "launches": launches, "avg_launch_ms": avg_ms,
                 "flops_per_launch": flops_per_launch,
                 "share_of_step": kd["active_ms"] / max(1e-9, ms)})
    # where a step's time goes: active time per kernel per step, and how many passes
    # over the data each path made per step (an AUTO redo shows as > 1)
    breakdown = {k: round(v["active_ms"] / args.steps, 3) for k, v in
                 sorted(kern.items(), key=lambda kv: -kv[1]["active_ms"]) if v["active"]}
    passes = {"tensor": kern.get("tc_stats", {}).get("active", 0) / (args.steps * n_chunks),
              "cuda_core": kern.get("stats_simt", {}).get("active", 0) / (args.steps * n_chunks)}

    # ---- end to end through the public API from pinned host memory
    # All ranks agree first on whether the pinned copy of X could be made, so that they
    # all take the same collective steps below.
    e2e = None
    if not args.no_e2e:
        err = None
        try:
            Xh = torch.empty(N, D, dtype=torch.float32, pin_memory=True)
            Xh.copy_(X)
        except Exception as ex:  # pinned allocation of X may fail on small hosts
            Xh, err = None, str(ex)[:200]
        ok = torch.tensor([0 if err else 1], dtype=torch.int32, device=dev)
        if world > 1:
            dist.all_reduce(ok, op=dist.ReduceOp.MIN)
        if int(ok.item()) == 1:
            # continue from the warmed-up parameters: the same steady-state step as above,
            # with X streamed from pinned host memory by the library (fgmm_em_step_host:
            # every pass of the step copies X chunk by chunk, overlapping the sweeps)
            wd2, md2, vd2 = wd.clone(), md.clone(), vd.clone()
            llh = torch.zeros(1, dtype=torch.float64, pin_memory=True)

            def e2e_step():
                em_step(Xh, wd2, md2, vd2)
                llh.copy_(ll, non_blocking=True)
                torch.cuda.current_stream().synchronize()
                return float(llh.item())

            e2e_step()
            barrier()
            g.profile(True)
            g.profile_read(reset=True)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(args.e2e_steps):
                e2e_step()
            b.record()
            torch.cuda.synchronize()
            ek = g.profile_read(reset=True)["kernels"]
            g.profile(False)
            e_passes = (ek.get("tc_stats", {}).get("active", 0) +
                        ek.get("stats_simt", {}).get("active", 0)) / (args.e2e_steps * n_chunks)
            e_ms = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
            if world > 1:
                dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
            e2e = {"value": world * args.e2e_steps / (float(e_ms.item()) / 1e3), "unit": "iters/s",
                   "h2d_bytes_per_step": int(round(N * D * 4 * e_passes)),
                   "d2h_bytes_per_step": 8, "steps": args.e2e_steps,
                   "how": "X in pinned host memory, streamed by fgmm_em_step_host in 2^20-point "
                          "chunks overlapping the sweeps; bytes = N x D x 4 per pass over X",
                   "passes_per_step": e_passes}
        else:
            e2e = {"value": None, "unit": "iters/s", "error": err or "pinned copy failed on a rank"}
        del Xh

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        pool = OraclePool()
        n_s = oracle_sample_size(w, pool.procs)
        dt = pool.step_time(w, n_s)
        pool.close()
        cpu = cpu_baseline_line(w, dt, n_s, pool.procs)

    if rank == 0:
        line = {
            "metric": METRIC if args.workload == "table1-1e8" else f"EM iters/s ({args.workload})",
            "value": iters_per_s, "unit": "iters/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": workload_name(w), "precision": prec_used,
                       "precision_setting": prec_set, "block_skip": g.block_skip,
                       "l2": f"inputs larger than L2 (X = {N * D * 4 / 1e9:.1f} GB per GPU)"
                       if N * D * 4 > 126e6 else "inputs smaller than L2",
                       "parallelism": (f"dp{world}: row shards of one mixture fit, one all-gather "
                                       f"of the {g.stats_len}-double statistics vector per step"
                                       if world > 1 else "single GPU")},
            "evals_per_s": iters_per_s * N * K,
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "step_ms_by_kernel": breakdown, "passes_per_step": passes,
            "gpu_launches": int(prof["launches"]),
            "workspace_bytes": g.workspace_bytes,
            "clocks": clocks,
            "loglik_last": float(ll.item()),
        }
        print(json.dumps(line), flush=True)
    g.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
