"""Throughput of the streaming log-domain Sinkhorn hot path on B200.

One step = one full pass of the hot path over one synthetic problem: fs_potentials
(the fixed-count alternating iterations), fs_grad_x, fs_marginal_residual and fs_cost,
each called through the C ABI exactly as a user calls it. The metric is pair
evaluations per second, N*M*iters / step time (each iteration runs two N*M passes).

Default workload: the clustered unit-cube problem, N = M = 2^20, d = 3, 1000 Gaussians
(std 0.01), eps = (N^(-1/3))^2 = 2^(-40/3), 20 iterations (the FlashSinkhorn 2 scale
rule "blur = mean interparticle distance"), float32.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c5] [--impl reference]

Under torchrun (N > 1) each rank solves its own independently seeded instance of the
same workload (replicas; weak scaling); value = all ranks' pair evaluations / the
slowest rank's time. `--impl reference` times the float64 CPU oracle on a bounded sample
of the same workload on this host's cores (rank 0 only).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "pair-evals/s (N·M·iters/s) log-domain Sinkhorn; % of ex2/FMA roofline"
UNIT = "pair-evals/s"
CONFIG_INDEX = {"c1": 0, "c2": 1, "c3": 2, "c4": 3, "c5": 4}
# MUFU ex2 throughput per SM per clock on sm_100 (16 results/clk/SM, CUDA throughput table).
EX2_PER_CLK_PER_SM = 16
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="c5", choices=sorted(CONFIG_INDEX))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--n", type=int, default=None,
                    help="clustered (c5) or mixture (c4) workload: use n = m points (c5: eps by "
                         "the same spacing rule; c4: the same eps), e.g. a small case to profile")
    ap.add_argument("--d", type=int, default=None,
                    help="50k-point mixture workload (c4) only: use d coordinates, eps = d / 64")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the measurements after the timed region (the unscreened pass "
                         "and the solve variants)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU seconds of the oracle sample")
    return ap.parse_args()


def workload(cfg: str, rank: int, n_override=None, d_override=None):
    from streaming_sinkhorn_b200 import workloads
    import dataclasses
    if cfg == "c4" and (d_override is not None or n_override is not None):
        # the same recipe at another width or size; eps grows with d so that kappa |x - y|^2
        # keeps the scale it has at d = 64, eps = 1
        d = 64 if d_override is None else d_override
        n = 50000 if n_override is None else n_override
        w = workloads.mixture_pair(n=n, d=d, k=10, mean_scale=2.0, std=1.0,
                                   seed=3 + 1000 * rank, eps=d / 64.0, n_iters=100)
        size = "50k" if n == 50000 else str(n)
        return dataclasses.replace(w, name=f"mix_{size}_d{d}")
    if d_override is not None:
        raise SystemExit("--d applies to the 50k-point mixture workload (c4) only")
    if n_override is not None:
        if cfg != "c5":
            raise SystemExit("--n applies to the clustered (c5) and mixture (c4) workloads only")
        w = workloads.clustered_cube(n=n_override, seed=4 + 1000 * rank, n_iters=20)
        return dataclasses.replace(w, name=f"clustered_cube_n{n_override}")
    # rank r > 0 runs an independently seeded replica of the same recipe
    return workloads.config(CONFIG_INDEX[cfg], seed_offset=1000 * rank)


# ---------------------------------------------------------------- clocks ----------

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fs_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- roofline ---------

def kernel_source_digest() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "streaming_sinkhorn_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(cfg: str):
    """Per-launch DRAM bytes of the LSE pass from a committed ncu summary, if it was
    measured on the current kernel sources (profiles/lse_pass_traffic.txt)."""
    path = os.path.join(ROOT, "profiles", "lse_pass_traffic.txt")
    if not os.path.exists(path):
        return None
    rec = {}
    for line in open(path):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.split("=", 1)
            rec[k.strip()] = v.strip()
    if rec.get("kernel_source_digest") != kernel_source_digest() or rec.get("config") != cfg:
        return None
    try:
        return float(rec["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            return json.load(open(path))
        except ValueError:
            return {}
    return {}


# ---------------------------------------------------------------- oracle sample ----

def oracle_sample(w, target_s: float):
    """Times the float64 oracle's f-update over a sample of rows against all M columns.

    Returns (pair-evals/s in the metric's unit, threads, description). One iteration is
    two N*M passes, so pairs/s of one pass / 2 is N*M*iters/s.
    """
    import oracle
    oracle.build()
    g0 = np.zeros(w.m, dtype=np.float64)
    rng = np.random.default_rng(0)
    # calibrate on enough rows to keep every oracle thread busy
    k0 = min(w.n, max(64, 8 * oracle.threads()))
    rows = rng.choice(w.n, size=k0, replace=False)
    t0 = time.perf_counter()
    oracle.lse_update(w.x, w.y, w.b, g0, w.eps, rows=rows)
    per_row = (time.perf_counter() - t0) / len(rows)
    k = int(max(1, min(w.n, target_s / max(per_row, 1e-9))))
    rows = rng.choice(w.n, size=k, replace=False)
    t0 = time.perf_counter()
    oracle.lse_update(w.x, w.y, w.b, g0, w.eps, rows=rows)
    dt = time.perf_counter() - t0
    pairs = float(k) * w.m
    value = pairs / dt / 2.0
    desc = (f"float64 oracle f-update (two-pass LSE, direct-difference cost) over {k} sampled "
            f"rows x all {w.m} columns of {w.name} ({pairs:.3e} pair evaluations, {dt:.1f} s); "
            f"scaled to N*M*iters/s as pair-evals/s / 2")
    return value, oracle.threads(), desc, dt


# ---------------------------------------------------------------- ranks ------------

def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time; every rank returns it (a MAX all-reduce, or ms alone)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(pairs_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the pairs all ranks processed per step over the slowest time."""
    return pairs_per_rank_step * world / (ms_per_step / 1e3)


# ---------------------------------------------------------------- native arm -------

def run_native(args, rank, world, local_rank):
    import torch
    import streaming_sinkhorn_b200 as fs

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    w = workload(args.config, rank, args.n, args.d)
    dev = torch.device("cuda", local_rank)
    x = torch.from_numpy(w.x).to(dev)
    y = torch.from_numpy(w.y).to(dev)
    a = torch.from_numpy(w.a).to(dev)
    b = torch.from_numpy(w.b).to(dev)
    f = torch.empty(w.n, dtype=torch.float32, device=dev)
    g = torch.empty(w.m, dtype=torch.float32, device=dev)
    gx = torch.empty((w.n, w.d), dtype=torch.float32, device=dev)
    ws = torch.empty(fs.workspace_bytes(w.n, w.m, w.d, dev), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        # one Morton sort per step, as for clouds that change from step to step; the three
        # later calls of the step reuse its order through the workspace
        fs.workspace_invalidate(ws)
        fs.potentials(x, y, a, b, eps=w.eps, n_iters=w.n_iters, out=(f, g), workspace=ws)
        fs.grad_x(x, y, g, a, b, eps=w.eps, out=gx, workspace=ws)
        res = fs.marginal_residual(x, y, f, g, a, b, eps=w.eps, workspace=ws)
        c = fs.cost(x, y, f, g, a, b, eps=w.eps, workspace=ws)
        return res, c

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()

    clocks = ClockSampler(local_rank)
    clocks.start()
    fs.timing_enable(True)
    fs.timing_reset()
    launches0 = fs.launch_count()
    barrier()
    total_ms = 0.0
    for _ in range(args.steps):
        flush.zero_()  # L2 flush between timed steps, outside the step's events
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        res, c = step()
        e1.record(stream)
        e1.synchronize()
        total_ms += e0.elapsed_time(e1)
    barrier()
    launches = fs.launch_count() - launches0
    timing = fs.timing_get()
    fs.timing_enable(False)
    clk = clocks.stop()
    ms_per_step = max_over_ranks(total_ms / args.steps, dist, dev)
    pairs_per_step = float(w.n) * w.m * w.n_iters
    value = job_value(pairs_per_step, world, ms_per_step)

    # roofline of the dominant kernel: the potential-update pass
    lse = timing["lse_pass"]
    per_launch_ms = lse["total_ms"] / max(lse["launches"], 1)
    # exponentials actually issued (after block screening; padding included); the tensor-core
    # path does not screen and reports none, so its nominal pair count stands
    executed = lse["evaluated"] if lse["evaluated"] > 0 else lse["pairs"]
    per_launch_pairs = executed / max(lse["launches"], 1)
    achieved = per_launch_pairs / (per_launch_ms / 1e3)  # ex2 / s
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    max_mhz = clk.get("sm_max_mhz") or measured_peaks().get("sm_max_mhz") or 1965.0
    peak = sms * EX2_PER_CLK_PER_SM * max_mhz * 1e6
    roofline = {"bound": "alu", "achieved": achieved / 1e12, "peak": peak / 1e12,
                "unit": "Tex2/s", "frac": achieved / peak,
                "traffic": recorded_traffic(args.config),
                "kernel": "lse_pass_kernel (potential update)",
                "peak_basis": f"{sms} SMs x {EX2_PER_CLK_PER_SM} ex2/clk x {max_mhz:.0f} MHz",
                "frac_at_observed_clock": (achieved / (sms * EX2_PER_CLK_PER_SM * clk["sm_mhz"] * 1e6)
                                           if clk.get("sm_mhz") else None),
                "launches_timed": lse["launches"], "ms_per_launch": per_launch_ms,
                "executed_ex2_per_launch": per_launch_pairs,
                "nominal_pairs_per_launch": lse["pairs"] / max(lse["launches"], 1),
                "screened_fraction": (1.0 - executed / lse["pairs"]) if lse["pairs"] else 0.0}
    if lse["evaluated"] > 0 and roofline["screened_fraction"] > 0.5:
        roofline["note"] = ("frac is the rate of the exponentials the screened pass issues: "
                            "block screening and, for d <= 3, the 16-point group skip leave "
                            "it only the pairs near each row's maximum, so each kept tile "
                            "also carries its copy, centring and group tests; dense_pass "
                            "gives the same kernel's rate on all N*M pairs")

    # The same pass with screening off, outside the timed region: one solve iteration (an
    # f pass and a g pass over all N x M pairs) on the same inputs, so the kernel's roofline
    # is also shown on dense work.
    if not args.no_extras:
        fs.screening_enable(False)
        fd, gd = torch.empty_like(f), torch.empty_like(g)
        fs.potentials(x, y, a, b, eps=w.eps, n_iters=1, out=(fd, gd), workspace=ws)
        torch.cuda.synchronize(dev)
        fs.timing_enable(True)
        fs.timing_reset()
        fs.potentials(x, y, a, b, eps=w.eps, n_iters=1, out=(fd, gd), workspace=ws)
        torch.cuda.synchronize(dev)
        td = fs.timing_get()["lse_pass"]
        fs.timing_enable(False)
        fs.screening_enable(True)
        d_ms = td["total_ms"] / max(td["launches"], 1)
        d_exec = (td["evaluated"] if td["evaluated"] > 0 else td["pairs"]) / max(td["launches"], 1)
        roofline["dense_pass"] = {
            "what": "potential pass with screening off (fs_screening_enable(0)), 2 launches",
            "ms_per_launch": d_ms, "executed_ex2_per_launch": d_exec,
            "achieved": d_exec / (d_ms / 1e3) / 1e12, "frac": d_exec / (d_ms / 1e3) / peak}

    # The general solve on the same inputs, outside the timed region: the symmetric
    # (Jacobi) schedule for the same iteration count, and the alternating schedule stopped
    # by the marginal check.
    solve_extras = None
    if not args.no_extras:
        solve_extras = {}
        for name, kw in (("symmetric_fixed", dict(n_iters=w.n_iters, variant="symmetric",
                                                  alpha=0.5)),
                         ("alternating_marginal_stop",
                          dict(stop_mode="marginal", stop_tol=0.12 * float(w.a.max()),
                               stop_check_every=5, stop_max_iter=200)),
                         ("multiscale_marginal_stop",
                          dict(stop_mode="marginal", stop_tol=0.12 * float(w.a.max()),
                               stop_check_every=5, stop_max_iter=200, multiscale=True))):
            kw = dict(kw)
            ms = kw.pop("multiscale", False)
            if ms and w.d > 16:
                continue

            def run():
                if ms:
                    ff, gg, r = fs.solve_multiscale(x, y, a, b, eps=w.eps,
                                                    lift_tol=kw["stop_tol"], **kw)
                    r = dict(r["fine"], coarse_rounds=r["rounds"], lift_viol=r["lift_viol"])
                    return r
                return fs.solve(x, y, a, b, eps=w.eps, out=(f, g), workspace=ws, **kw)[2]

            run()
            torch.cuda.synchronize(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            rep = run()
            e1.record(stream)
            e1.synchronize()
            ms_t = e0.elapsed_time(e1)
            solve_extras[name] = {
                "options": {k: v for k, v in kw.items()}, "ms": ms_t,
                "iters_run": rep["iters_run"], "converged": rep["converged"],
                "final_viol": None if rep["final_viol"] != rep["final_viol"] else rep["final_viol"],
                "pair_evals_per_s": float(w.n) * w.m * rep["iters_run"] / (ms_t / 1e3)}
            for k in ("coarse_rounds", "lift_viol"):
                if k in rep:
                    solve_extras[name][k] = rep[k]
        # a transport-matrix product (P Y, d channels) and a Hessian-vector product at the
        # potentials just solved
        if True:
            from streaming_sinkhorn_b200 import _lib
            p_ = _lib.fs_problem(x.data_ptr(), y.data_ptr(), a.data_ptr(), b.data_ptr(), w.n, w.m,
                                 w.d, w.eps)
            import ctypes
            twork = torch.empty(int(_lib.load().fs_transport_workspace_bytes(ctypes.byref(p_))),
                                dtype=torch.uint8, device=dev)
            v = torch.randn((w.n, w.d), generator=torch.Generator().manual_seed(5)).to(dev)
            for name, call in (
                    ("debiased_divergence_with_grads", lambda: (None, {"value": float(
                        fs.sinkhorn_divergence(x, y, a, b, eps=w.eps, n_iters=w.n_iters,
                                               grads=True)[0])})),
                    ("transport_apply_PY", lambda: (fs.transport_apply(
                        x, y, f, g, y, a, b, eps=w.eps, workspace=twork), None)),
                    ("hvp", lambda: fs.hvp(x, y, g, v, a, b, eps=w.eps, cg_max_iter=50,
                                           cg_tol=1e-4, workspace=twork))):
                call()
                torch.cuda.synchronize(dev)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                _, rep = call()
                e1.record(stream)
                e1.synchronize()
                solve_extras[name] = {"ms": e0.elapsed_time(e1)}
                if rep is not None:
                    solve_extras[name].update(rep)

    # Work the kernels actually did: pairs evaluated per step by every pass of the step (after
    # screening; the tensor-core path does not screen, so there it is the nominal count),
    # and the metric rate the unscreened pass sustains.
    evaluated = 0.0
    for k in ("lse_pass", "grad_pass", "marg_pass"):
        t = timing[k]
        evaluated += t["evaluated"] if t["evaluated"] > 0 else t["pairs"]
    executed = {
        "pairs_evaluated_per_step": evaluated / args.steps,
        "executed_pair_evals_per_s": evaluated / args.steps / (ms_per_step / 1e3),
        "what": "pairs the kernels evaluated per step (all passes: 2 x iters potential passes, "
                "gradient, marginal and plan-mass passes) over the step time"}
    if "dense_pass" in roofline:
        dp = roofline["dense_pass"]
        # one iteration = two N x M passes; N*M*iters/s of the pass run unscreened
        executed["dense_metric_rate"] = float(w.n) * w.m / (dp["ms_per_launch"] / 1e3) / 2.0
        executed["dense_metric_rate_what"] = ("N*M*iters/s of the potential pass with screening "
                                              "off (N*M pairs per launch, two per iteration)")

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "n": w.n, "m": w.m, "d": w.d, "eps": w.eps,
                   "iters": w.n_iters, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "step": "fs_potentials + fs_grad_x + fs_marginal_residual + fs_cost (one Morton sort per step, reused by the later calls)",
                   "l2": "flushed between timed steps (256 MiB write); inputs "
                         f"{((w.n + w.m) * (w.d + 1) * 4) / 1e6:.0f} MB",
                   "screening": "on: value counts all N*M*iters pairs; roofline.executed_ex2 "
                                "counts the exponentials the kernels issued"},
        "gpu_launches": int(launches),
        "executed": executed,
        "roofline": roofline,
        "clocks": clk,
        "kernel_timing": timing,
        "solve_variants": solve_extras,
        "check": {"residual": [float(v) for v in res.cpu().numpy()], "cost": float(c.item())},
    }

    if not args.no_e2e:
        result["e2e"] = run_e2e(args, w, dev, world, dist)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc, _ = oracle_sample(w, args.cpu_seconds)
        result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                  "sample": desc}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_e2e(args, w, dev, world, dist):
    """Same metric through fs_solve_host: host inputs copied in and results copied out
    inside every timed step. Each step drops the workspace's sort record first, so it sorts
    once as the device-timed step does, and runs in the same mode (per-kernel timing on, so
    no CUDA graph replay); the same loop with timing off (graph replay of the iterations)
    is reported beside it."""
    import torch
    import streaming_sinkhorn_b200 as fs
    pin = lambda v: torch.from_numpy(v).pin_memory()  # noqa: E731
    xh, yh, ah, bh = pin(w.x), pin(w.y), pin(w.a), pin(w.b)
    out = {"f": torch.empty(w.n, dtype=torch.float32).pin_memory(),
           "g": torch.empty(w.m, dtype=torch.float32).pin_memory(),
           "grad_x": torch.empty((w.n, w.d), dtype=torch.float32).pin_memory(),
           "cost": torch.empty(1, dtype=torch.float64).pin_memory(),
           "residual": torch.empty(4, dtype=torch.float64).pin_memory()}
    import ctypes
    from streaming_sinkhorn_b200 import _lib
    p = _lib.fs_problem(xh.data_ptr(), yh.data_ptr(), ah.data_ptr(), bh.data_ptr(), w.n, w.m, w.d,
                        w.eps)
    nbytes = int(_lib.load().fs_solve_host_workspace_bytes(ctypes.byref(p)))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    steps = args.e2e_steps if args.e2e_steps is not None else args.steps
    stream = torch.cuda.current_stream(dev)

    def one():
        fs.workspace_invalidate(ws)
        fs.solve_host(xh, yh, ah, bh, eps=w.eps, n_iters=w.n_iters, device=dev, workspace=ws,
                      out=out)

    def timed(per_kernel_timing: bool) -> float:
        fs.timing_enable(per_kernel_timing)
        one()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            one()
        e1.record(stream)
        e1.synchronize()
        fs.timing_enable(False)
        return max_over_ranks(e0.elapsed_time(e1) / steps, dist, dev)

    ms = timed(True)
    ms_graphs = timed(False)
    h2d = (w.n * w.d + w.m * w.d + w.n + w.m) * 4
    d2h = (w.n + w.m + w.n * w.d) * 4 + 5 * 8
    pairs = float(w.n) * w.m * w.n_iters
    return {"value": job_value(pairs, world, ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": steps, "api": "fs_solve_host (pinned host buffers)",
            "mode": "per-kernel timing on, no graph replay, one sort per step (as the device leg)",
            "graph_replay": {"value": job_value(pairs, world, ms_graphs), "ms_per_step": ms_graphs,
                             "mode": "timing off: iterations 2.. replayed as one CUDA graph"}}


# ---------------------------------------------------------------- reference arm ----

def run_reference(args, rank, world):
    if rank != 0:
        return
    w = workload(args.config, 0, args.n, args.d)
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, min(per_step, 3.0))
    vals, secs = [], 0.0
    desc, cores = "", 1
    for _ in range(args.steps):
        v, cores, desc, dt = oracle_sample(w, per_step)
        vals.append(v)
        secs += dt
    value = float(np.mean(vals))
    pairs_per_step = float(w.n) * w.m * w.n_iters
    ms_per_step = pairs_per_step / value * 1e3
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "n": w.n, "m": w.m, "d": w.d, "eps": w.eps,
                   "iters": w.n_iters, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc + "; each step one such sample"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        world = int(os.environ["WORLD_SIZE"])
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1 and "RANK" not in os.environ:
        raise SystemExit("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    from streaming_sinkhorn_b200 import build
    if not os.path.exists(build.LIB):
        build.build()
    run_native(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
