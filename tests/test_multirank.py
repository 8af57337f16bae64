"""The N > 1 host path of bench.py on CPU: two gloo ranks (one process each, as torchrun would
start them).  Each rank times its own replica; the job's time is the max over ranks and the
job's throughput counts every rank's blocks.  Also checks that the reference arm runs on rank 0
only."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, results):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r "took" 0.5 + r seconds: the job took the slowest rank's time
        t = bench.max_over_ranks(0.5 + rank, torch.device("cpu"), world)
        v = bench.job_throughput(40, 5, world, t)
        # the reference arm does its work and prints on rank 0 only
        class A:  # minimal argparse stand-in; rank != 0 returns before touching it
            pass
        ref = bench.run_reference(A(), rank, world) if rank != 0 else "rank0"
        dist.barrier()
        results[rank] = (t, v, ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_job_throughput():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(results)
    assert set(res) == {0, 1}
    for r in range(world):
        t, v, _ = res[r]
        assert t == pytest.approx(1.5)                 # max of 0.5 and 1.5 on both ranks
        assert v == pytest.approx(40 * 5 * 2 / 1.5)    # all ranks' layer-blocks / job time
    assert res[1][2] is None                           # rank 1: no reference work, no line


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.25, torch.device("cpu"), 1) == 0.25
    assert bench.job_throughput(40, 5, 1, 2.0) == pytest.approx(100.0)


def test_gpus_mismatch_with_launcher_fails_loudly():
    """A launcher that started fewer ranks than --gpus asks for must not time one GPU."""
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    import subprocess
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2"],
                         env=env, capture_output=True, text=True, timeout=120)
    assert res.returncode == 2 and "--gpus 2" in res.stderr


def test_gpus_without_launcher_starts_one_rank_per_gpu(monkeypatch):
    """--gpus N with no launcher re-runs the script under torch.distributed.run with N ranks
    on 127.0.0.1."""
    sys.path.insert(0, ROOT)
    import bench
    seen = {}
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: (seen.setdefault("cmd", cmd), 0)[1])
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "2"])

    class A:
        gpus = 4
    assert bench._launch_ranks(A()) == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "2"]


def test_job_throughput_counts_streams_not_ranks_for_a_head_split():
    sys.path.insert(0, ROOT)
    import bench
    # 4 ranks sharing one stream (heads split) vs 4 independent streams
    assert bench.job_throughput(40, 5, 1, 2.0) == pytest.approx(100.0)
    assert bench.job_throughput(40, 5, 4, 2.0) == pytest.approx(400.0)
