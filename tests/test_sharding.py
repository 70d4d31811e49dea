"""Host logic of the prefill split by query rows (sharding.py), on CPU.

The balanced ranges are checked against a brute-force sum of the per-row
cost; the cache exchange runs under a real two-process gloo group
(127.0.0.1) on CPU tensors, the same collective NCCL runs on the GPUs.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from long_context_indexing_lightning_b200 import sharding  # noqa: E402


@pytest.mark.parametrize("n_q,world,pos0,topk", [(300, 2, 0, 16), (1000, 4, 0, 64), (777, 3, 1234, 64),
                                                 (5, 8, 0, 4), (0, 2, 0, 16), (65536, 8, 0, 2048)])
def test_balanced_ranges_cover_and_balance(n_q, world, pos0, topk):
    ranges = sharding.balanced_row_ranges(n_q, world, pos0=pos0, topk=topk)
    assert len(ranges) == world
    assert ranges[0][0] == 0 and ranges[-1][1] == n_q
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    assert all(r0 <= r1 for r0, r1 in ranges)
    cost = [sharding.row_cost(pos0 + t, topk) for t in range(n_q)]
    total = sum(cost)
    assert sharding._cum_cost(n_q, pos0, topk, sharding.ATTN_ROW_COST) == pytest.approx(total, rel=1e-12)
    cmax = max(cost) if cost else 0.0
    for r0, r1 in ranges:
        assert abs(sum(cost[r0:r1]) - total / world) <= cmax * (1 + 1e-9)


def test_balanced_ranges_give_early_ranks_more_rows():
    # causal cost grows with position: the first rank takes the most rows
    ranges = sharding.balanced_row_ranges(65536, 4, topk=2048)
    sizes = [r1 - r0 for r0, r1 in ranges]
    assert sizes == sorted(sizes, reverse=True) and sizes[0] > sizes[-1]


@pytest.mark.parametrize("n_new,world", [(10, 3), (9, 3), (1, 4), (0, 2), (65536, 8)])
def test_append_shares_partition_the_new_tokens(n_new, world):
    shares = [sharding.append_share(n_new, world, r) for r in range(world)]
    got = [i for a, b in shares for i in range(a, b)]
    assert got == list(range(n_new))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fill(rank, B, S, W, dtype):
    g = torch.Generator().manual_seed(100 + rank)  # every rank holds different stale rows
    return torch.randn(B, S, W, generator=g).to(dtype)


def _worker(rank, world, port, cfg, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    from long_context_indexing_lightning_b200 import sharding as sh
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, S, W, b, row0, n_new = cfg
        cache = _fill(rank, B, S, W, torch.bfloat16)
        scale = _fill(rank, B, S, 1, torch.float32)[..., 0].contiguous()
        before = cache.clone()
        a0, a1 = sh.append_share(n_new, world, rank)
        # this rank's share of the new rows: a value that names the row
        for i in range(a0, a1):
            cache[b, row0 + i] = float(row0 + i)
            scale[b, row0 + i] = 0.5 * (row0 + i)
        sh.gather_cache_rows(cache, b, row0, n_new)
        sh.gather_cache_rows(scale, b, row0, n_new)
        new = cache[b, row0:row0 + n_new].float()
        ok_new = bool((new == torch.arange(row0, row0 + n_new).float()[:, None]).all())
        ok_scale = bool((scale[b, row0:row0 + n_new] == 0.5 * torch.arange(row0, row0 + n_new).float()).all())
        c = -(-n_new // world)
        keep = torch.ones(B, S, dtype=torch.bool)
        keep[b, row0:row0 + world * c] = False
        ok_rest = bool((cache[keep] == before[keep]).all())
        out[rank] = (ok_new, ok_scale, ok_rest)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cfg", [(2, 64, 8, 1, 5, 21), (1, 40, 8, 0, 0, 40)])
def test_two_gloo_ranks_gather_the_new_cache_rows(cfg):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, cfg, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert res == {0: (True, True, True), 1: (True, True, True)}


def test_gather_range_must_fit_the_cache():
    import torch.distributed as dist

    orig = dist.get_world_size, dist.get_rank
    dist.get_world_size, dist.get_rank = (lambda group=None: 4), (lambda group=None: 0)
    try:
        with pytest.raises(ValueError):
            sharding.gather_cache_rows(torch.zeros(1, 10, 2), 0, 3, 5)  # 4 chunks of 2 rows from row 3 > 10
    finally:
        dist.get_world_size, dist.get_rank = orig


def _worker_dropout(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import time
    import torch.distributed as dist
    from long_context_indexing_lightning_b200 import sharding as sh
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        # this rank leaves between steps, before the exchange, without a word
        os._exit(0)
    cache = torch.zeros(1, 32, 4, dtype=torch.bfloat16)
    t0 = time.monotonic()
    try:
        sh.gather_cache_rows(cache, 0, 0, 32)
        out[rank] = ("no error", time.monotonic() - t0)
    except Exception as e:  # the survivor learns of it from the collective
        out[rank] = (type(e).__name__, time.monotonic() - t0)


def test_a_rank_that_leaves_before_the_exchange_fails_the_collective():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker_dropout, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
        res = dict(out)
    assert 0 in res, "the surviving rank did not report"
    kind, secs = res[0]
    assert kind != "no error" and secs < 60, res
