"""The bench's multi-rank logic on CPU: two gloo ranks, replicas only.

With N ranks every rank decodes its own replicas (there is no data exchange
on the path); the reported value is the units of all ranks divided by the
slowest rank's time, and only rank 0 prints.  The reduction is the one the
bench uses, here over gloo instead of NCCL.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (r + 1) * 10 ms for its steps and 100 + r ms end to end
        got = bench.max_over_ranks([(rank + 1) * 10.0, 100.0 + rank], world, "cpu")
        rate = bench.whole_job_rate(50, world, got[0])
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rate in res:
        assert got == [20.0, 101.0]  # the slowest rank's times
        assert rate == pytest.approx(2 * 50 / 0.020)  # both ranks' units / slowest time


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
    assert bench.whole_job_rate(10, 1, 1000.0) == pytest.approx(10.0)


@pytest.mark.parametrize("config,unit", [("tiny", "decodes/s"), ("deltanet", "updates/s")])
@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_zero_only(rank, config, unit):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", config,
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300,
                       cwd=root)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank != 0:
        assert lines == []
    else:
        d = json.loads(lines[-1])
        assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
