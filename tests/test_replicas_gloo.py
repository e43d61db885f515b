"""The N > 1 path of bench.py on the CPU: two gloo ranks agree on the slowest rank's time
and on the whole-job value, each rank draws its own seeded replica of the workload, and the
reference arm runs on rank 0 only. No GPU is used."""
import os
import socket
import subprocess
import sys

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 7.5 * rank
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.job_value(1e6, world, ms)
        q.put((rank, local_ms, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max(g[1] for g in got)
    assert all(g[2] == slowest for g in got)
    # 1e6 pairs per rank per step, 2 ranks, 17.5 ms -> 2e6 / 0.0175 s
    assert all(abs(g[3] - 2e6 / 0.0175) < 1e-3 for g in got)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
    assert bench.job_value(4e6, 1, 2.0) == 2e9


def test_each_rank_draws_its_own_replica():
    for cfg in ("c1", "c2", "c3", "c5"):
        if cfg == "c5":
            w0 = bench.workload("c5", 0, 4096)
            w1 = bench.workload("c5", 1, 4096)
        else:
            w0, w1 = bench.workload(cfg, 0), bench.workload(cfg, 1)
        assert w0.x.shape == w1.x.shape and w0.y.shape == w1.y.shape and w0.eps == w1.eps
        assert not np.array_equal(w0.x, w1.x)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_workload_overrides_keep_the_recipes():
    """--n and --d build the named recipes at other sizes (small cases to profile): the
    clustered cube keeps its spacing rule for eps, the mixture keeps eps = d / 64."""
    w = bench.workload("c5", 0, 4096, None)
    assert (w.n, w.m, w.d) == (4096, 4096, 3) and abs(w.eps - 4096.0 ** (-2.0 / 3.0)) < 1e-12
    w0 = bench.workload("c4", 0, 16384, None)
    assert (w0.n, w0.m, w0.d) == (16384, 16384, 64) and w0.eps == 1.0 and w0.n_iters == 100
    w = bench.workload("c4", 0, None, 512)
    assert (w.n, w.m, w.d) == (50000, 50000, 512) and w.eps == 8.0
    r1 = bench.workload("c4", 1, 16384, None)  # rank 1: its own replica of the same recipe
    assert r1.x.shape == w0.x.shape and not np.array_equal(r1.x, w0.x)
