"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

The benchmark runs one independent replica per GPU; its only cross-rank steps
are the barriers around the timed region and the max over ranks of the
elapsed time.  Both are exercised here with the gloo backend, without a GPU.
"""
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


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(True, None)
        elapsed = 10.0 + 5.0 * rank          # ranks see different times
        got = bench.max_over_ranks(elapsed, True, None)
        bench.barrier(True, None)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_with_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, False) == 3.5
    bench.barrier(False)
    ws, rank, local = bench.dist_setup()
    assert ws >= 1 and rank >= 0 and local >= 0
