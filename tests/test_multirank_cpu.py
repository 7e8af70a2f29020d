"""bench.py's multi-rank host logic at world size 2 on gloo, without a GPU.

`bench.py --gpus N` runs one process per GPU. Each rank runs its own full
workload with no data exchange. Ranks meet only at barriers and at the
max-over-ranks of the step time. These tests bring up two CPU ranks on
127.0.0.1 and check the following:
- every rank gets the slowest rank's time;
- a clock rejection seen on one rank reaches every rank, so all time the step
  again together;
- the whole-job rate counts every rank's tokens;
- the reference arm's other ranks exit at once, with no process group.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    w, r, _ = bench.dist_setup()
    try:
        backend = torch.distributed.get_backend()
        slow = bench.max_over_ranks(10.0 + 5.0 * rank, w)   # rank 1 is the slow one
        bench.barrier(w)
        again = (bench.any_rank(rank == 1, w), bench.any_rank(False, w))
        q.put((r, w, backend, slow, bench.job_rate(w, 131072, slow), again))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time(monkeypatch):
    import torch.multiprocessing as mp
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "")   # children: host ranks only
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert [p.exitcode for p in procs] == [0, 0]
    got = sorted(q.get(timeout=10) for _ in range(2))
    for r, (rank, world, backend, slow, rate, again) in enumerate(got):
        assert (rank, world, backend) == (r, 2, "gloo")
        assert slow == 15.0                          # max over ranks, on every rank
        assert rate == pytest.approx(2 * 131072 / 15e-3)
        assert again == (True, False)                # rank 1's flag reaches rank 0


def test_job_rate_is_whole_job_throughput():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_rate(1, 131072, 300.0) == pytest.approx(131072 / 0.3)
    assert bench.job_rate(8, 64, 0.5) == pytest.approx(8 * 64 / 0.5e-3)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    env.pop("MASTER_ADDR", None)
    env.pop("MASTER_PORT", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
