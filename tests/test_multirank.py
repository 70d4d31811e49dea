"""The N > 1 benchmark path on CPU: two gloo ranks (127.0.0.1).

The decode step shards by sequence with no data-path collective; the only
cross-rank operation is the timing aggregation (max over ranks).  These tests
run that aggregation and the rank handling of the reference arm under a real
two-process group, without a GPU.
"""
import os
import socket
import sys
from types import SimpleNamespace

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    import bench
    import workloads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench._dist()
        # per-rank "timings"; every rank must see the slowest
        got = bench.max_over_ranks(10.0 + 5.0 * r, "cpu")
        # the reference arm does its work on rank 0 only; other ranks return at once
        args = SimpleNamespace(steps=1, warmup=0)
        ref = bench.run_reference(args, workloads.get("tiny")) if r != 0 else "skipped"
        out[r] = (ws, r, local, got, ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_over_ranks_and_reference_rank_handling():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert res[0][:3] == (2, 0, 0) and res[1][:3] == (2, 1, 1)
    assert res[0][3] == 15.0 and res[1][3] == 15.0
    assert res[1][4] is None


def test_single_process_max_over_ranks_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
