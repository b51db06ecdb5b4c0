"""The multi-rank bench path on CPU: two gloo ranks (no GPU).

bench.py runs one replica per GPU with no data-path collective; the only
cross-rank steps are the barriers around the timed region and the max over
ranks of the timed milliseconds.  These tests run those helpers in two spawned
processes over gloo on 127.0.0.1."""
import argparse
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # rank r took 10 (r + 1) ms for 5 steps of 4096 tokens
        value, ms_max = bench.aggregate_throughput(4096 * 5, 10.0 * (rank + 1), world)
        # the reference arm: every rank but 0 returns at once, without work
        ref = None
        if rank != 0:
            args = argparse.Namespace(preset="olmoe", tokens=4096, steps=1, warmup=3, gpus=world)
            ref = bench.run_reference(args)
        bench.barrier(world)
        q.put((rank, value, ms_max, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, value, ms_max, ref in res:
        assert ms_max == pytest.approx(20.0)
        # both ranks' tokens over the slower rank's time
        assert value == pytest.approx(2 * 4096 * 5 / 0.020)
        assert ref is None
