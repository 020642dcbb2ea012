"""The multi-GPU paths on the CPU with gloo ranks: replicas, each timing its
own layer (the job's step time is the slowest rank's and the throughput
counts every rank's tokens: weak scaling, no data-path collective); and the
collective of a head-sharded layer, driven through the C function pointer
the library calls."""
from __future__ import annotations

import os
import socket

import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slower one
    ms = bench.max_over_ranks(local_ms, world, "cpu")
    tokens_per_rank = 136_900
    q.put((rank, ms, world * tokens_per_rank / (ms / 1e3), bench.dist_env()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value, env in out:
        assert ms == 15.0                              # the slower rank's time, on every rank
        assert abs(value - 2 * 136_900 / 0.015) < 1e-6
        assert env == (rank, 2, 0)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5


def _exchange_rank(rank: int, world: int, port: int, q):
    import torch
    import torch.distributed as dist

    from token_merging_view_b200 import binding as B
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ex = B.TorchExchange()
    ws = torch.zeros(1024, dtype=torch.uint8)          # stands in for a workspace
    ex.workspace = ws
    hist = ws[256:256 + 4 * 96].view(torch.int32)      # a histogram
    hist.copy_(torch.arange(96, dtype=torch.int32) * (rank + 1))
    cnt = ws[8:16].view(torch.int64)
    cnt.fill_(1000 + rank)
    fn = ex.c.allreduce_sum                               # the pointer the library would call
    st = [fn(hist.data_ptr(), 96, 4, None, None), fn(cnt.data_ptr(), 1, 8, None, None)]
    bad = [fn(ws.data_ptr() + 1020, 2, 4, None, None),    # runs past the workspace
           fn(ws.data_ptr() + 2, 1, 4, None, None),       # misaligned
           fn(None, 1, 4, None, None)]
    q.put((rank, st, bad, hist.tolist(), int(cnt.item()), ex.calls))
    dist.barrier()
    dist.destroy_process_group()


def test_torch_exchange_sums_workspace_buffers_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, st, bad, hist, cnt, calls in out:
        assert st == [0, 0] and bad == [1, 1, 1] and calls == 2
        assert hist == [3 * i for i in range(96)]
        assert cnt == 2001
