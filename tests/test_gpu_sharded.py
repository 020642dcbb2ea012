"""A head-sharded layer on one GPU.  The shards run as host threads, each
with its own plan, workspace and stream, and an in-process collective sums
their buffers: stream-ordered (events), no kernel waits on another.  The
shards' outlier masks, outlier counts, slots and per-head exports equal the
unsharded layer's exactly (the global top-d% of key design 3 is one
selection over all heads, ties by flat index), and their outputs equal it
up to the summation order of attention items split along the keys."""
from __future__ import annotations

import threading

import numpy as np
import pytest
import torch

import oracle.httm_oracle as O
from tests import paritylib as PL
from token_merging_view_b200 import binding as B
from token_merging_view_b200.workloads import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

MID = Workload("mid_8f", T=8, grid=37, h=4, d=64, fp32=False, n_s=128, n_t=3, q_stride=4, kv_stride=4,
               q_pct=70, kv_pct=50, out_pct=10, seed=11, noise_sigma=0.3, max_shift=2)


class ThreadCollective:
    """Sums a buffer over shards that run as threads of this process: every
    shard records an event on its stream and waits (host barrier) for the
    others; shard 0 adds the buffers on a stream of its own after all those
    events and writes the sum back to each; every shard's stream then waits
    for that addition."""

    def __init__(self, shards: int):
        self.barrier = threading.Barrier(shards, timeout=120)
        self.slots = [None] * shards
        self.done = None
        self.stream = torch.cuda.Stream()

    def member(self, rank: int) -> "_Member":
        return _Member(self, rank)


class _Member:
    def __init__(self, col: ThreadCollective, rank: int):
        self.col, self.rank = col, rank
        self.workspace = None
        self.calls = 0
        self._fn = B.EXCHANGE_FN(self._sum)
        self.c = B.httm_exchange(self._fn, None)

    def _sum(self, buf, count, elem_bytes, stream, user) -> int:
        col = self.col
        try:
            view = B.exchange_view(self.workspace, buf, count, elem_bytes)
            s = torch.cuda.ExternalStream(stream) if stream else torch.cuda.default_stream()
            ev = torch.cuda.Event()
            ev.record(s)
            col.slots[self.rank] = (view, ev)
            col.barrier.wait()
            if self.rank == 0:
                rs = col.stream
                for _, e in col.slots:
                    rs.wait_event(e)
                with torch.cuda.stream(rs):
                    total = torch.stack([v for v, _ in col.slots]).sum(0, dtype=view.dtype)
                    for v, _ in col.slots:
                        v.copy_(total)
                done = torch.cuda.Event()
                done.record(rs)
                col.done = done
            col.barrier.wait()
            s.wait_event(col.done)
            col.barrier.wait()
            self.calls += 1
            return 0
        except Exception:
            col.barrier.abort()
            return 1


def run_sharded(w: Workload, shards: int, Q, K, V):
    hl = w.h // shards
    col = ThreadCollective(shards)
    jobs = []
    for r in range(shards):
        plan = B.httm_plan(B.LayerConfig.from_workload(w, h=hl)).shard(r, shards)
        sl = slice(r * hl, (r + 1) * hl)
        jobs.append(dict(plan=plan, q=Q[sl].contiguous(), k=K[sl].contiguous(), v=V[sl].contiguous(),
                         ws=plan.new_workspace(), dbg=B.debug_buffers(plan), stream=torch.cuda.Stream(),
                         member=col.member(r)))
    torch.cuda.synchronize()

    def work(j):
        try:
            j["out"] = B.httm_forward_sharded(j["plan"], j["q"], j["k"], j["v"], j["member"], workspace=j["ws"],
                                              dbg=j["dbg"], stream=j["stream"])
            j["status"] = B.httm_get_device_status(j["plan"], j["ws"], stream=j["stream"])
        except Exception as e:   # reported below
            j["error"] = e

    threads = [threading.Thread(target=work, args=(j,)) for j in jobs]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    torch.cuda.synchronize()
    for j in jobs:
        assert "error" not in j, j.get("error")
        assert j["status"] == 0 and j["member"].calls == 5
    return jobs


def check_against_unsharded(w: Workload, shards: int, Q, K, V):
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    out, dbg, ws, status = PL.run(plan, Q, K, V)
    assert status == 0
    n_out = B.workspace_view(plan, ws, "n_out").cpu().numpy()
    jobs = run_sharded(w, shards, Q, K, V)
    hl = w.h // shards
    for r, j in enumerate(jobs):
        sl = slice(r * hl, (r + 1) * hl)
        d = PL.cpu(j["dbg"])
        for key in ("outlier", "q_slot", "k_slot", "dev", "q_best", "k_best", "q_merged", "k_merged"):
            assert np.array_equal(d[key], dbg[key][sl]), key
        assert np.array_equal(B.workspace_view(j["plan"], j["ws"], "n_out").cpu().numpy(), n_out[sl])
        a, b = j["out"].float(), out[sl].float()
        assert (a - b).abs().max().item() <= 2e-2 * max(1.0, b.abs().max().item())
    return dbg, jobs


@pytest.mark.parametrize("w,shards", [(WORKLOADS["vggt_30f"], 2), (MID, 4), (MID, 2)],
                         ids=["vggt_30f_2", "mid_4", "mid_2"])
def test_sharded_layer_equals_unsharded(w, shards):
    Q, K, V = PL.inputs(w)
    check_against_unsharded(w, shards, Q, K, V)


@pytest.mark.parametrize("shards", [2, 4])
def test_sharded_big_groups_equal_unsharded(shards):
    """Groups of more than 32 members (each shard lists its own heads' and
    sums them with the CTA-wide kernels): the same masks, slots and
    exports as the unsharded layer."""
    Q, K, V = PL.inputs(MID)
    PL.plant_big_groups(MID, Q, K, V)
    dbg, _ = check_against_unsharded(MID, shards, Q, K, V)
    counts = np.stack([np.bincount(row, minlength=MID.N) for row in dbg["q_slot"]])
    assert (counts > 32).sum() >= 20


def test_sharded_ties_are_taken_in_flat_index_order():
    """Q all zero: every eligible query deviates by 0, so the whole budget
    (40 % of h N here) is one tie, taken in flat-index order: every eligible
    query of heads 0 and 1, part of head 2's and none of head 3's -- quotas
    that cross two shard boundaries (one head per shard)."""
    w = MID.with_(T=3, out_pct=40)
    Q, K, V = PL.inputs(w)
    Q = torch.zeros_like(Q)
    dbg, _ = check_against_unsharded(w, 4, Q, K, V)
    res = O.forward_plan(PL.oracle_cfg(w), *(PL.to64(t) for t in (Q, K, V)))
    mask = dbg["outlier"].astype(bool)
    assert np.array_equal(mask, res.mask)
    per_head = mask.sum(axis=1)
    k = 40 * w.h * w.N // 100
    e = int(per_head[0])   # zero queries give every head the same plan, so the same eligible count
    assert per_head.tolist() == [e, e, k - 2 * e, 0] and 0 < k - 2 * e < e


def test_sharded_tiny_fp32_matches_oracle_mask():
    w = WORKLOADS["tiny_4f_8x8"]
    Q, K, V = PL.inputs(w)
    res = O.forward_plan(PL.oracle_cfg(w), *(PL.to64(t) for t in (Q, K, V)))
    jobs = run_sharded(w, 2, Q, K, V)
    mask = np.concatenate([PL.cpu(j["dbg"])["outlier"] for j in jobs]).astype(bool)
    assert np.array_equal(mask, res.mask)
