"""Cross-layer reuse of the merge indices (httm_forward_reuse) vs the oracle.

The LiteVGGT note (key design 3, cross-layer cached merging) computes the
merge indices on one layer and reuses them on the following ones.  The
oracle side is forward_plan() on the next layer's Q/K/V with the first
layer's plans passed in.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.httm_oracle as O
from tests import paritylib as PL
from token_merging_view_b200 import binding as B
from token_merging_view_b200.workloads import DENSE, Workload

pytestmark = pytest.mark.gpu

MID = Workload("mid_8f", T=8, grid=37, h=4, d=64, fp32=False, n_s=128, n_t=3, q_stride=4, kv_stride=4,
               q_pct=70, kv_pct=50, out_pct=10, seed=11, noise_sigma=0.3, max_shift=2)


def _next_layer(w: Workload, X: tuple, seed: int) -> tuple:
    """Inputs of a following layer: the same tokens drifted towards another
    draw of the same generator (token similarity mostly kept)."""
    Y = PL.inputs(w.with_(seed=seed))
    return tuple((0.8 * a.float() + 0.6 * b.float()).to(a.dtype).contiguous() for a, b in zip(X, Y))


def _setup(w: Workload):
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    cfg = PL.oracle_cfg(w)
    X1 = PL.inputs(w)
    return plan, cfg, X1


def _check_layer(w, plan, cfg, ws, out, X, res_plan):
    """``out`` = the reused layer's output on inputs X, with the member lists
    of ``res_plan`` (an oracle result whose plans were injected)."""
    q, k, v = (PL.to64(t) for t in X)
    res = O.forward_plan(cfg, q, k, v, q_plan=res_plan.q_plan, k_plan=res_plan.k_plan)
    kt = B.workspace_view(plan, ws, "k")[: w.h * plan.info.kv_slots]
    vt = B.workspace_view(plan, ws, "v")[: w.h * plan.info.kv_slots]
    assert PL.bf16_ulps(kt, res.k_means.reshape(-1, w.d)) <= 1
    assert PL.bf16_ulps(vt, res.v_means.reshape(-1, w.d)) <= 1
    # the same layer with the plans passed in gives the same bits, and its
    # debug exports give the outlier mask and deviations of the reused call
    dbg = B.debug_buffers(plan)
    out_p = B.httm_forward_with_plan(plan, *X, PL.oracle_plan_tensors(res_plan, mask=False), dbg,
                                     workspace=plan.new_workspace())
    assert torch.equal(out, out_p)
    dbg = PL.cpu(dbg)
    assert np.all(np.abs(dbg["dev"] - res.dev) <= 1e-4 * np.maximum(1.0, res.dev))
    # the mask may differ from the oracle's only on deviation near-ties; the
    # output is then checked against the oracle run on that mask
    assert PL.compare_mask(res, dbg["outlier"]) <= 2
    res = O.forward_plan(cfg, q, k, v, q_plan=res_plan.q_plan, k_plan=res_plan.k_plan,
                         mask=dbg["outlier"].astype(bool))
    assert np.array_equal(B.workspace_view(plan, ws, "n_out").cpu().numpy(), res.restore.n_out)
    mx, rl2 = PL.sample_out_error(res, PL.to64(out), cfg, 1 << 30)
    assert mx <= PL.OUT_MAX_ABS and rl2 <= PL.OUT_REL_L2, (mx, rl2)


def test_reuse_matches_oracle_on_injected_plan():
    w = MID
    plan, cfg, X1 = _setup(w)
    res1 = O.forward_plan(cfg, *(PL.to64(t) for t in X1))
    ws = plan.new_workspace()
    # layer 1 on the oracle's plan writes the member lists the next layers reuse
    B.httm_forward_with_plan(plan, *X1, PL.oracle_plan_tensors(res1, mask=False), workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    X = X1
    for layer, seed in enumerate((101, 102)):
        X = _next_layer(w, X, seed)
        out = B.httm_forward_reuse(plan, *X, workspace=ws)
        assert B.httm_get_device_status(plan, ws) == 0, layer
        _check_layer(w, plan, cfg, ws, out, X, res1)


def test_reuse_equals_forward_with_the_same_plan():
    """Reusing the layer's own plan gives the bits httm_forward_with_plan
    gives when that plan is passed in explicitly."""
    w = MID
    plan, cfg, X1 = _setup(w)
    dbg = B.debug_buffers(plan)
    ws = plan.new_workspace()
    B.httm_forward_debug(plan, *X1, dbg, workspace=ws)
    full = plan.launches()
    X2 = _next_layer(w, X1, 7)
    out_r = B.httm_forward_reuse(plan, *X2, workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    assert plan.launches() < full
    inj = {k: dbg[k] for k in ("q_best", "q_merged", "k_best", "k_merged")}
    out_p = B.httm_forward_with_plan(plan, *X2, inj, workspace=plan.new_workspace())
    assert torch.equal(out_r, out_p)


def test_reuse_keeps_the_big_group_lists():
    """Groups of more than 32 members are summed by kernels of their own
    from lists the planning writes; a reusing call plans nothing and takes
    them from the workspace with the member lists.  Its output equals that
    of the same plan passed in (which plans, and lists, afresh)."""
    w = MID
    plan, cfg, X1 = _setup(w)
    PL.plant_big_groups(w, *X1)
    dbg = B.debug_buffers(plan)
    ws = plan.new_workspace()
    B.httm_forward_debug(plan, *X1, dbg, workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    counts = np.stack([np.bincount(row, minlength=w.N) for row in dbg["q_slot"].cpu().numpy()])
    assert (counts > 32).sum() >= 20
    X2 = _next_layer(w, X1, 9)
    out_r = B.httm_forward_reuse(plan, *X2, workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    inj = {k: dbg[k] for k in ("q_best", "q_merged", "k_best", "k_merged")}
    out_p = B.httm_forward_with_plan(plan, *X2, inj, workspace=plan.new_workspace())
    assert torch.equal(out_r, out_p)


def test_reuse_without_member_lists_sets_status():
    w = MID.with_(T=3, h=2)
    plan, cfg, X1 = _setup(w)
    # a workspace no forward of this plan has written
    ws = torch.zeros(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    B.httm_forward_reuse(plan, *X1, workspace=ws)
    assert B.httm_get_device_status(plan, ws) & B.HTTM_DEV_BAD_PLAN
    # member lists of another plan (same sizes) do not count
    other = B.httm_plan(B.LayerConfig.from_workload(w))
    B.httm_forward(other, *X1, workspace=ws)
    assert B.httm_get_device_status(other, ws) == 0
    B.httm_forward_reuse(plan, *X1, workspace=ws)
    assert B.httm_get_device_status(plan, ws) & B.HTTM_DEV_BAD_PLAN
    # nor do those of a call whose planning failed
    B.httm_forward(plan, *X1, workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    res = O.forward_plan(cfg, *(PL.to64(t) for t in X1))
    bad = PL.oracle_plan_tensors(res, mask=False)
    bad["q_merged"] = torch.zeros_like(bad["q_merged"])
    B.httm_forward_with_plan(plan, *X1, bad, workspace=ws)
    assert B.httm_get_device_status(plan, ws) & B.HTTM_DEV_BAD_PLAN
    B.httm_forward_reuse(plan, *X1, workspace=ws)
    assert B.httm_get_device_status(plan, ws) & B.HTTM_DEV_BAD_PLAN
    # a good forward makes reuse valid again
    B.httm_forward(plan, *X1, workspace=ws)
    B.httm_forward_reuse(plan, *X1, workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0


def test_reuse_host_errors():
    w = MID.with_(T=2, h=2)
    X = PL.inputs(w)
    dense = B.httm_plan(B.LayerConfig.from_workload(w.with_(mode=DENSE)))
    with pytest.raises(B.HttmError) as e:
        B.httm_forward_reuse(dense, *X, workspace=dense.new_workspace())
    assert e.value.status == 1                                   # HTTM_ERR_ARG
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    with pytest.raises(ValueError):
        B.httm_forward_reuse(plan, *X)
