"""The N > 1 host logic of bench.py on CPU: two gloo ranks, as torchrun would start them.

bench.py runs one independent replica per GPU (the path has no exchange between
sequences); the only collectives are the barriers and the maximum over ranks of the
timed region.  These tests run that aggregation with world_size 2 over gloo on
127.0.0.1, and check that the reference arm does no work on ranks other than 0.
"""

import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_ms, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        got = bench.replica_aggregate(local_ms[rank], 1000, world, "cpu")
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_the_slowest_rank():
    world, port = 2, _free_port()
    local_ms = [10.0, 25.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    for r in range(world):
        max_ms, value = res[r]
        assert max_ms == 25.0                        # every rank sees the slowest rank's time
        assert value == 1000 * world / 25e-3         # tokens of all ranks / that time


def test_reference_arm_does_no_work_off_rank_zero(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"workload": "llama2_7b_bf16", "steps": 3, "warmup": 3, "gpus": 2})()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
