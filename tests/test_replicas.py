"""The host logic of the multi-GPU benchmark path on CPU: replicas reduce
their timings and status with one MAX all-reduce (gloo, world size 2 here;
NCCL on GPUs), and the job's rate counts every replica's units over the
slowest replica's time."""
import importlib.util
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("hgd_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, vals, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        res = _bench().replica_reduce(vals[rank], "cpu")
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_replica_reduce_takes_the_slowest_rank_and_any_error():
    import torch.multiprocessing as mp
    world = 2
    # (device ms, end-to-end s, status): rank 1 is slower on the device, rank 0
    # end to end, and rank 1 reports an error
    vals = [[812.5, 2.25, 0], [907.0, 1.5, 5]]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, vals, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert got[r] == [907.0, 2.25, 5.0]


def test_aggregate_rate_counts_every_replica():
    b = _bench()
    # 4 replicas, 128 tokens each, slowest replica took 0.5 s
    assert b.aggregate_rate(4, 128, 0.5) == pytest.approx(1024.0)
    assert b.aggregate_rate(1, 128, 0.128) == pytest.approx(1000.0)
