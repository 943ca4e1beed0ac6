"""Multi-rank host logic of bench.py, on CPU with the gloo backend (world size 2).

The benchmark runs one replica of the workload per rank; the job's time is the slowest
rank's and its throughput counts every rank's work. These tests run that reduction across
two real processes, and check that the reference arm (the oracle on the host) does its work
and prints on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, result_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(times[rank], dist, "cpu")
        rate = bench.job_rate(world, 3.0e12, 5, mx, 1e12)
        with open(os.path.join(result_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max_ms": mx, "rate": rate}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_world2(tmp_path):
    times = [12.5, 40.0]  # rank 1 is the slow one
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r in res:
        assert r["max_ms"] == 40.0  # every rank sees the slowest rank's time
        # 2 ranks x 3e12 FLOP x 5 steps in 40 ms = 750 TFLOP/s for the whole job
        assert r["rate"] == pytest.approx(750.0)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.25) == 7.25
    assert bench.job_rate(1, 2.0e9, 4, 8.0, 1e9) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_exit_silently():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0
    assert out.stdout.strip() == ""


def test_visible_pairs_brute_force():
    """The attended (query, key) pair count against enumeration on small shapes."""
    import bench
    for Nq, Nk, causal, window in [(5, 5, True, 0), (3, 9, True, 0), (9, 9, True, 4),
                                   (4, 11, True, 3), (6, 7, False, 0), (1, 1, True, 1)]:
        off = Nk - Nq
        n = 0
        for i in range(Nq):
            for j in range(Nk):
                hi = i + off if causal else Nk - 1
                lo = hi - window + 1 if window > 0 else 0
                n += lo <= j <= hi
        assert bench.visible_pairs(Nq, Nk, causal, window) == n
