"""LiteVGGT's destination rule inside HTTM's temporal blocks (HTTM_PARTITION)
on the CUDA path, through the C ABI, against the fp64 oracles: the token
classes the device computes from a score against
oracle.litevggt_partition's (bit-exact), the per-head matching against that
oracle's plans (a destination mismatch excused only inside the 1e-4 tie
margin of the oracle's own cosines), the merged flags exactly (they follow
from the classes), the plan's sizes, and the layer's output at every token
whose final query slot holds the oracle's members (the HTTM oracle run on
the partition oracle's plans)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle.httm_oracle as O
import oracle.litevggt_partition as L
from tests import paritylib as PL
from token_merging_view_b200 import binding as B
from token_merging_view_b200.inputs import make_score
from token_merging_view_b200.workloads import PARTITION, WORKLOADS, Workload

pytestmark = pytest.mark.gpu

PLAN_FIELDS = ("q_best", "q_score", "q_merged", "k_best", "k_score", "k_merged", "q_slot")

# 8 frames of the 37 x 37 grid, 4 heads, blocks of 128 patches x 3 frames
# (partial regions, a partial temporal group; the first group holds frame 1)
MIDP = Workload("mid_8f_partition", T=8, grid=37, h=4, d=64, fp32=False, n_s=128, n_t=3, q_stride=4, kv_stride=4,
                q_pct=70, kv_pct=50, out_pct=10, seed=11, noise_sigma=0.3, max_shift=2, mode=PARTITION)


def _check(w: Workload, ga_pct: int, slots_per_head: int = 1 << 30):
    Q, K, V = PL.inputs(w)
    score = make_score(T=w.T, grid=w.grid, seed=w.seed + 7).float().contiguous().to("cuda")
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    roles_g = B.httm_plan_partition(plan, score, ga_pct).cpu().numpy()
    roles_o = L.partition_roles(score.double().cpu().numpy(), w.grid, ga_pct)
    assert np.array_equal(roles_g, roles_o)
    q, k, v = (PL.to64(t) for t in (Q, K, V))
    cfg = PL.oracle_cfg(w)
    blocks = O.block_list(cfg)
    qp = L.plan_tensor_partition(q, blocks, roles_o)
    kp = L.plan_tensor_partition(k, blocks, roles_o)
    assert plan.info.q_slots == qp.n_slots and plan.info.kv_slots == kp.n_slots
    res = O.forward_plan(cfg, q, k, v, q_plan=qp, k_plan=kp)
    out, dbg, ws, status = PL.run(plan, Q, K, V, fields=PLAN_FIELDS)
    assert status == 0
    ex = PL.compare_best(q, qp, dbg["q_best"], dbg["q_score"]) + PL.compare_best(k, kp, dbg["k_best"], dbg["k_score"])
    assert ex <= 1e-3 * w.h * w.N
    assert np.array_equal(dbg["q_merged"].astype(bool), qp.merged)
    assert np.array_equal(dbg["k_merged"].astype(bool), kp.merged)
    ok = PL.shared_slot_tokens(res.restore.slot_final, dbg["q_slot"])
    assert ok.mean() >= 0.99, ok.mean()
    mx, rl2, _ = PL.sample_slot_error(res, out, cfg, slots_per_head, seed=1, token_ok=ok)
    assert mx <= PL.OUT_MAX_ABS and rl2 <= PL.OUT_REL_L2, (mx, rl2)
    return roles_g, ex


@pytest.mark.parametrize("ga_pct", [10, 0, 35])
def test_partition_layer_matches_oracle(ga_pct):
    roles, _ = _check(MIDP, ga_pct)
    assert (roles == L.ROLE_GA).sum() == MIDP.T * L.ga_count(MIDP.P, ga_pct)


def test_partition_all_ga_is_dense_attention():
    """Every token geometry-aware: nothing merges, the layer is plain
    attention (the oracle's no-merging special case)."""
    w = MIDP.with_(T=2, h=2)
    roles, _ = _check(w, 100)
    assert np.all(roles == L.ROLE_GA)


def test_partition_resizes_and_rejects():
    w = MIDP.with_(T=2, h=2)
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    Q, K, V = PL.inputs(w)
    with pytest.raises(B.HttmError) as e:           # not partitioned yet
        B.httm_forward(plan, Q, K, V, workspace=plan.new_workspace())
    assert e.value.status == 1
    s1 = make_score(T=w.T, grid=w.grid, seed=1).float().contiguous().to("cuda")
    B.httm_plan_partition(plan, s1, 10)
    a = plan.info.q_slots
    B.httm_plan_partition(plan, s1, 50)             # a new partition of the same plan
    assert plan.info.q_slots > a                    # more GA tokens, fewer merges, more slots
    out = B.httm_forward(plan, Q, K, V, workspace=plan.new_workspace())
    assert out.shape == Q.shape


@pytest.mark.slow
def test_partition_vggt_30f_layer():
    """The 30-frame layer (16 heads, 41,070 tokens; blocks of up to ~1050
    destinations, above the stride rule's 960) with 10 % GA tokens."""
    _check(WORKLOADS["vggt_30f"].with_(mode=PARTITION), 10, slots_per_head=4096)
