"""Host logic of the N-GPU benchmark path on CPU: two gloo ranks check the max-over-ranks
timing reduction and the per-rank seeds (each rank draws its own independent batch; the
work shards across ranks with no collective on the data path)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, ws = bench.rank_env()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, ws)
        w = workloads.WORKLOADS["tiny"]
        seed = bench.rank_seed(w, r)
        x = workloads.make_inputs(w, seed=seed).q
        # every rank holds a different batch
        gathered = [torch.zeros_like(x.float()) for _ in range(ws)]
        dist.all_gather(gathered, x.float())
        distinct = not torch.equal(gathered[0], gathered[1])
        q.put((r, lr, ws, ms, seed, distinct))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in results] == [0, 1]
    assert all(r[2] == 2 for r in results)
    assert all(r[3] == 15.0 for r in results)          # max over ranks, seen by every rank
    assert results[0][4] != results[1][4]              # per-rank seeds differ
    assert all(r[5] for r in results)                  # and so do the batches


def test_single_rank_defaults(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (0, 0, 1)
    assert bench.max_over_ranks(3.5, 1) == 3.5
