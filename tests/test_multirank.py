"""The multi-GPU path on the CPU: two gloo ranks, each timing its own layer;
the job's step time is the slowest rank's and the throughput counts every
rank's tokens (weak scaling, no data-path collective)."""
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
