"""Host logic of bench.py's N > 1 path on CPU: world-size-2 gloo ranks run
the same barrier-bracketed timed region, the reported time is the max over
ranks, and only rank 0 prints (weak scaling: each rank quantises its own
layer, no data-path collective)."""

import json
import os
import socket
import subprocess
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _WallTimer:
    def sync(self):
        pass

    def start(self):
        self.t0 = time.perf_counter()

    def stop(self):
        self.t1 = time.perf_counter()

    def elapsed_ms(self):
        return (self.t1 - self.t0) * 1e3


def _rank_main(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist("gloo", world)
    calls = []

    def step():  # rank 1 is slower: the reported time must be its time
        calls.append(1)
        time.sleep(0.02 if rank == 1 else 0.002)

    ms = bench.timed_steps(step, 5, dist, _WallTimer())
    dist.destroy_process_group()
    q.put((rank, ms, len(calls)))


def test_timed_region_takes_max_over_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, n0), (r1, ms1, n1) = res
    assert n0 == n1 == 5                      # every rank ran exactly the timed steps
    assert ms0 == ms1                         # both report the same (max) value
    assert ms0 >= 20.0                        # ... which is the slow rank's time per step


def test_reference_arm_runs_on_rank0_only(tmp_path):
    """Under torchrun with N > 1 the oracle arm runs on rank 0; other ranks
    exit 0 without work and print nothing."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_bench_rejects_short_warmup():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "1"],
                         capture_output=True, text=True, timeout=120)
    assert out.returncode != 0 and "warmup" in (out.stderr + out.stdout)
