"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.httm_oracle as O
from tests import paritylib as PL
from token_merging_view_b200 import binding as B
from token_merging_view_b200.workloads import CONTIGUOUS, DENSE, HEAD_UNIFORM, WORKLOADS, Workload

pytestmark = pytest.mark.gpu

# 8 frames of the 37 x 37 grid, 4 heads: blocks of 384 / 267 / 256 / 178
# tokens (partial regions and a partial temporal group), several 128-row tiles
# with ragged tails.
MID = Workload("mid_8f", T=8, grid=37, h=4, d=64, fp32=False, n_s=128, n_t=3, q_stride=4, kv_stride=4,
               q_pct=70, kv_pct=50, out_pct=10, seed=11, noise_sigma=0.3, max_shift=2)
TINY = WORKLOADS["tiny_4f_8x8"]


def _case(w: Workload, transform=None, **kw):
    w = w.with_(**kw) if kw else w
    Q, K, V = PL.inputs(w)
    if transform is not None:
        transform(w, Q, K, V)
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    cfg = PL.oracle_cfg(w)
    return w, plan, cfg, (Q, K, V), tuple(PL.to64(t) for t in (Q, K, V))


PLAN_FIELDS = ("q_best", "q_score", "q_merged", "k_best", "k_score", "k_merged", "q_slot")
MERGE_FIELDS = ("q_means", "k_means", "v_means", "dev", "outlier")
RESTORE_FIELDS = ("q_restored", "q_slot", "outlier")


def _full_check(w: Workload, slots_per_head: int = 1 << 30, max_excused_frac: float = 1e-3, transform=None,
                inspect=None):
    w, plan, cfg, (Q, K, V), (q, k, v) = _case(w, transform)
    res = O.forward_plan(cfg, q, k, v)
    if inspect is not None:
        inspect(res)
    # 1. the layer's own plan, and its own end-to-end output
    out, dbg, ws, status = PL.run(plan, Q, K, V, fields=PLAN_FIELDS)
    assert status == 0
    blocks = O.block_list(cfg)
    ex = PL.compare_best(q, res.q_plan, dbg["q_best"], dbg["q_score"])
    ex += PL.compare_best(k, res.k_plan, dbg["k_best"], dbg["k_score"])
    ex += PL.compare_merged(blocks, cfg.q_stride, cfg.q_pct, res.q_plan, dbg["q_merged"])
    ex += PL.compare_merged(blocks, cfg.kv_stride, cfg.kv_pct, res.k_plan, dbg["k_merged"])
    assert ex <= max_excused_frac * w.h * w.N
    # the output of every token whose final query slot holds the same members
    # as the oracle's (all of them unless an excused near-tie moved a few)
    ok = PL.shared_slot_tokens(res.restore.slot_final, dbg["q_slot"])
    assert ok.mean() >= 0.99, ok.mean()
    own = PL.sample_slot_error(res, out, cfg, slots_per_head, seed=1, token_ok=ok)
    assert own[0] <= PL.OUT_MAX_ABS and own[1] <= PL.OUT_REL_L2, own
    del out, dbg, ws
    # 2. merging, deviation and the filter on the oracle's plan (mask computed)
    inj = PL.oracle_plan_tensors(res, mask=False)
    _, dbg2, ws2, status = PL.run(plan, Q, K, V, injected=inj, fields=MERGE_FIELDS)
    assert status == 0
    assert PL.rel_rows(dbg2["q_means"], res.q_means).max() < PL.FEAT_REL
    assert PL.rel_rows(dbg2["k_means"], res.k_means).max() < PL.FEAT_REL
    assert PL.rel_rows(dbg2["v_means"], res.v_means).max() < PL.FEAT_REL
    kt = B.workspace_view(plan, ws2, "k")[: w.h * plan.info.kv_slots]
    vt = B.workspace_view(plan, ws2, "v")[: w.h * plan.info.kv_slots]
    if not w.fp32:
        assert PL.bf16_ulps(kt, res.k_means.reshape(-1, w.d)) <= 1
        assert PL.bf16_ulps(vt, res.v_means.reshape(-1, w.d)) <= 1
    assert np.all(np.abs(dbg2["dev"] - res.dev) <= 1e-4 * np.maximum(1.0, res.dev))
    n_mask_ex = PL.compare_mask(res, dbg2["outlier"])
    assert n_mask_ex <= max(2, max_excused_frac * w.h * w.N)
    del dbg2, ws2, kt, vt
    # 3. the whole layer on the oracle's plan and mask
    inj["outlier"] = PL.oracle_plan_tensors(res)["outlier"]
    out3, dbg3, ws3, status = PL.run(plan, Q, K, V, injected=inj, fields=RESTORE_FIELDS)
    assert status == 0
    live = res.restore.live
    assert PL.rel_rows(dbg3["q_restored"][live], res.restore.means[live]).max() < PL.FEAT_REL
    assert np.array_equal(B.workspace_view(plan, ws3, "n_out").cpu().numpy(), res.restore.n_out)
    assert np.array_equal(dbg3["q_slot"], res.restore.slot_final)
    assert np.array_equal(dbg3["outlier"].astype(bool), res.mask)
    mx, rl2, _ = PL.sample_slot_error(res, out3, cfg, slots_per_head)
    assert mx <= PL.OUT_MAX_ABS and rl2 <= PL.OUT_REL_L2, (mx, rl2)
    return ex, n_mask_ex, own[:2]


def test_tiny_fp32_layer_exact_plan():
    ex, mex, _ = _full_check(TINY, max_excused_frac=0.0)
    assert ex == 0 and mex == 0


def test_mid_layer():
    _full_check(MID)


def test_mid_layer_contiguous_blocks():
    _full_check(MID.with_(mode=CONTIGUOUS, contig_block=384))


def test_mid_layer_head_uniform():
    _full_check(MID.with_(mode=HEAD_UNIFORM))


@pytest.mark.parametrize("kw", [dict(out_pct=0), dict(out_pct=100), dict(q_pct=0, kv_pct=0),
                                dict(T=1, n_t=1), dict(q_stride=8, q_pct=85), dict(n_s=100, n_t=2)])
def test_mid_layer_edge_cases(kw):
    _full_check(MID.with_(**kw))


def test_vggt_30f_layer():
    """The 30-frame layer (41,070 tokens, 16 heads): every query slot of every
    head, on the oracle's plan and on the layer's own."""
    _full_check(WORKLOADS["vggt_30f"])


@pytest.mark.slow
def test_vggt_30f_contiguous_3840_blocks():
    """Contiguous un-reordered blocks of 3840 tokens at the 30-frame layer
    (HTTM note, key design 2, Fig. 8a): ten full blocks of 960 destinations
    and a partial last block of 2670 tokens."""
    _full_check(WORKLOADS["vggt_30f"].with_(mode=CONTIGUOUS, contig_block=3840), slots_per_head=4096)


@pytest.mark.slow
def test_vggt_100f_layer_sampled():
    _full_check(WORKLOADS["vggt_100f"], slots_per_head=4096)


@pytest.mark.slow
def test_vggt_500f_layer_sampled():
    """The 500-frame layer (684,500 tokens, queries with destinations every
    8th token and 85% merged) in the launch configuration bench.py times."""
    _full_check(WORKLOADS["vggt_500f"], slots_per_head=4096)


@pytest.mark.slow
def test_vggt_1000f_layer_sampled():
    """The 1000-frame layer (1,369,000 tokens; head-wise temporal, Q r = 70 %,
    outlier d = 10 %), the longest sequence the pages time: the whole plan of
    every block and head against the oracle's, and the output on 512 seeded
    query slots per head.  Its [h, N, d] element offsets reach 1.4e9, within
    a factor 1.6 of the int32 limit."""
    _full_check(WORKLOADS["vggt_1000f"], slots_per_head=512)


def test_reorder_matches_oracle():
    for w in (TINY, MID, MID.with_(mode=CONTIGUOUS, contig_block=500)):
        _, plan, cfg, (Q, _, _), (q, _, _) = _case(w)
        Xb = B.httm_reorder(plan, Q)
        want = O.reorder(q, O.block_list(cfg))
        assert np.array_equal(PL.to64(Xb), want)
        back = B.httm_reorder(plan, Xb, inverse=True)
        assert torch.equal(back, Q)


def test_dense_mode_and_unmerged_layer():
    w = MID.with_(T=2, h=2)
    _, plan, cfg, (Q, K, V), (q, k, v) = _case(w, mode=DENSE)
    out = B.httm_forward(plan, Q, K, V)
    want = O.forward(PL.oracle_cfg(w.with_(mode=DENSE)), q, k, v).out
    g = PL.to64(out)
    assert np.abs(g - want).max() <= PL.OUT_MAX_ABS
    assert np.linalg.norm(g - want) / np.linalg.norm(want) <= PL.OUT_REL_L2
    # r = 0: the merged layer reduces to dense attention
    _, plan0, _, _, _ = _case(w, q_pct=0, kv_pct=0)
    out0 = B.httm_forward(plan0, Q, K, V)
    g0 = PL.to64(out0)
    assert np.abs(g0 - want).max() <= PL.OUT_MAX_ABS


@pytest.mark.parametrize("kw", [dict(), dict(out_pct=100)], ids=["d10", "d100"])
def test_big_groups(kw):
    """Groups of more than 32 members (a destination that draws most of its
    block) take the CTA-wide sums of the gathers and the restore: every stage
    against the oracle, as in the other layers, with big groups in both plans
    and outliers among their members."""
    def check(res):
        qs, ks = PL.group_sizes(res.q_plan), PL.group_sizes(res.k_plan)
        assert (qs > 32).sum() >= 20 and (ks > 32).sum() >= 20, ((qs > 32).sum(), (ks > 32).sum())
        big = np.take_along_axis(qs, np.maximum(res.q_plan.best, 0), axis=1) > 32
        assert (res.mask & big).sum() > 0
    _full_check(MID.with_(**kw) if kw else MID, transform=PL.plant_big_groups, inspect=check)


def test_identical_and_zero_tokens():
    w = MID.with_(T=3, h=2)
    _, plan, cfg, (Q, K, V), _ = _case(w)
    Q = torch.zeros_like(Q)
    K = K[:, :1].expand_as(K).contiguous()          # every key identical
    q, k, v = (PL.to64(t) for t in (Q, K, V))
    res = O.forward_plan(cfg, q, k, v)
    out, dbg, ws, status = PL.run(plan, Q, K, V)
    assert status == 0
    assert np.array_equal(dbg["q_best"], res.q_plan.best) and np.array_equal(dbg["k_best"], res.k_plan.best)
    assert np.array_equal(dbg["q_merged"].astype(bool), res.q_plan.merged)
    assert np.array_equal(dbg["k_merged"].astype(bool), res.k_plan.merged)
    assert np.all(dbg["dev"] == 0.0)


@pytest.mark.slow
def test_identical_tokens_30f_layer():
    """The 30-frame layer with every query zero and every key of a head
    identical (V as drawn): every cosine ties, so each block's sources all
    take its first destination and the top-r merge takes its first r sources
    -- one group of about 2,000 members per block, head and tensor, the case
    the CTA-wide big-slot kernels are for.  Every query deviation is 0, so
    the outlier budget is one tie taken in flat-index order.  The query plan,
    the mask, the slots and the outlier counts equal the oracle's exactly
    (zero rows make its cosines and deviations exactly 0 too); the key plan
    equals the tie rules written out; every output row is the mean of the
    shortened values (every score ties)."""
    w = WORKLOADS["vggt_30f"]
    _, plan, cfg, (Q, K, V), _ = _case(w)
    Q = torch.zeros_like(Q)
    K = K[:, :1].expand_as(K).contiguous()
    q, k, v = (PL.to64(t) for t in (Q, K, V))
    res = O.forward_plan(cfg, q, k, v)
    out, dbg, ws, status = PL.run(plan, Q, K, V)
    assert status == 0
    # the key plan by the tie rules: every source to its block's first
    # destination; the first r sources (in-block order) merged
    blocks = O.block_list(cfg)
    best = np.full(w.N, -1, dtype=np.int64)
    merged = np.zeros(w.N, dtype=bool)
    members = []                                   # the key slots' members, every head alike
    for toks in blocks:
        d_i, s_i = O.split_dst_src(toks.shape[0], cfg.kv_stride)
        r = O.merge_count(toks.shape[0], cfg.kv_pct)
        best[toks[s_i]] = toks[0]
        merged[toks[s_i[:r]]] = True
        members.append(np.concatenate([toks[:1], toks[s_i[:r]]]))
        members += [toks[[i]] for i in d_i[1:]] + [toks[[i]] for i in s_i[r:]]
    assert max(m.shape[0] for m in members) > 1000
    assert np.array_equal(dbg["k_best"], np.broadcast_to(best, dbg["k_best"].shape))
    assert np.array_equal(dbg["k_merged"].astype(bool), np.broadcast_to(merged, dbg["k_merged"].shape))
    assert np.array_equal(dbg["q_best"], res.q_plan.best)
    assert np.array_equal(dbg["q_merged"].astype(bool), res.q_plan.merged)
    assert (PL.group_sizes(res.q_plan) > 1000).sum() >= w.h * 10
    assert np.all(dbg["dev"] == 0.0)
    assert np.array_equal(dbg["outlier"].astype(bool), res.mask)
    assert np.array_equal(dbg["q_slot"], res.restore.slot_final)
    assert np.array_equal(B.workspace_view(plan, ws, "n_out").cpu().numpy(), res.restore.n_out)
    # Q~ is zero, so every score is 0 and every output row is the mean of V~
    vt = np.stack([np.stack([v[hh, m].mean(axis=0) for m in members]) for hh in range(w.h)])
    want = vt.mean(axis=1)                         # [h, d]
    got = out.float().cpu().numpy()
    err = np.abs(got - want[:, None, :]).max()
    assert err <= PL.OUT_MAX_ABS, err


def test_deterministic():
    _, plan, _, (Q, K, V), _ = _case(MID)
    a, da, _, _ = PL.run(plan, Q, K, V)
    b, db, _, _ = PL.run(plan, Q, K, V)
    assert torch.equal(a, b)
    for key in da:
        assert np.array_equal(da[key], db[key], equal_nan=True), key


@pytest.mark.parametrize("w", [MID, TINY, WORKLOADS["vggt_30f"]], ids=lambda w: w.name)
def test_plain_and_debug_calls_agree(w):
    """httm_forward restores only the slots holding outliers; the debug call
    (which exports every slot's restored mean) walks all slots.  Same bits."""
    _, plan, _, (Q, K, V), _ = _case(w)
    a = B.httm_forward(plan, Q, K, V, workspace=plan.new_workspace())
    b, _, _, status = PL.run(plan, Q, K, V)
    assert status == 0
    assert torch.equal(a, b)


def test_output_independent_of_workspace_contents():
    """Rows of Q~ past a work item's end are never written; attention must
    not let them change the live rows (filled with zeros, then with large
    finite values)."""
    _, plan, _, (Q, K, V), _ = _case(MID)
    outs = []
    for fill in (0x00, 0x47):
        ws = torch.full((plan.workspace_bytes,), fill, dtype=torch.uint8, device="cuda")
        outs.append(B.httm_forward(plan, Q, K, V, workspace=ws))
        assert B.httm_get_device_status(plan, ws) == 0
    assert torch.equal(outs[0], outs[1])


def test_invalid_injected_plan_sets_status():
    w, plan, cfg, (Q, K, V), (q, k, v) = _case(MID.with_(T=3, h=2))
    res = O.forward_plan(cfg, q, k, v)
    inj = PL.oracle_plan_tensors(res, mask=False)
    inj["q_merged"] = torch.zeros_like(inj["q_merged"])        # wrong merge count in every block
    _, _, _, status = PL.run(plan, Q, K, V, injected=inj, debug=False)
    assert status & B.HTTM_DEV_BAD_PLAN
    inj = PL.oracle_plan_tensors(res, mask=False)
    inj["k_best"] = torch.where(inj["k_best"] >= 0, (inj["k_best"] + 1) % w.N, inj["k_best"])  # a non-dst target
    _, _, _, status = PL.run(plan, Q, K, V, injected=inj, debug=False)
    assert status & B.HTTM_DEV_BAD_PLAN
    # a clean call afterwards reports a clean status
    _, _, _, status = PL.run(plan, Q, K, V, debug=False)
    assert status == 0


def test_host_errors():
    _, plan, _, (Q, K, V), _ = _case(MID.with_(T=2, h=2))
    ws = plan.new_workspace()
    with pytest.raises(B.HttmError) as e:
        B.httm_forward(plan, Q, K, V, workspace=ws[: plan.workspace_bytes // 2])
    assert e.value.status == 4                                   # HTTM_ERR_WORKSPACE
    with pytest.raises(B.HttmError) as e:
        B.httm_forward(plan, Q, K, V, workspace=ws[1:])
    assert e.value.status == 5                                   # HTTM_ERR_ALIGN
    Qm = torch.empty(Q.numel() + 8, dtype=Q.dtype, device=Q.device)[1:1 + Q.numel()].view(Q.shape)
    with pytest.raises(B.HttmError) as e:
        B.httm_forward(plan, Qm, K, V, workspace=ws)
    assert e.value.status == 5


@pytest.mark.parametrize("T", [1, 2])
def test_short_key_ranges_split_parts(T):
    """Few key tiles per head: every work item of the last (here the only)
    wave runs as parts of one or two key tiles whose partial results are
    merged.  Repeated calls must agree bit for bit, and with the oracle on
    its own plan and mask (this case once exposed two barrier races)."""
    w = MID.with_(T=T, n_t=T)
    _, plan, cfg, (Q, K, V), (q, k, v) = _case(w)
    res = O.forward_plan(cfg, q, k, v)
    inj = PL.oracle_plan_tensors(res)
    outs = []
    for _ in range(4):
        out, _, _, status = PL.run(plan, Q, K, V, injected=inj, debug=False)
        assert status == 0
        outs.append(out)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    mx, rl2 = PL.sample_out_error(res, PL.to64(outs[0]), cfg, 1 << 30)
    assert mx <= PL.OUT_MAX_ABS and rl2 <= PL.OUT_REL_L2, (mx, rl2)


@pytest.mark.slow
def test_vggt_30f_head_uniform_plan():
    """The head-uniform plan at the 30-frame layer's shape (16 heads, blocks
    of 3840 / 2670 tokens) from the tensor-core matcher: the plan against the
    oracle's, and the output on the oracle's plan and mask."""
    _full_check(WORKLOADS["vggt_30f"].with_(mode=HEAD_UNIFORM), slots_per_head=4096)


@pytest.mark.parametrize("kw", [dict(d=16), dict(fp32=True, T=3, h=2)], ids=["bf16_d16", "fp32_d64"])
def test_mid_layer_cuda_core_paths(kw):
    """Shapes served by the CUDA-core matching and attention kernels (bf16
    with d_head = 16, fp32 with d_head = 64) against the oracle."""
    _full_check(MID.with_(**kw))


@pytest.mark.parametrize("w", [MID, MID.with_(mode=HEAD_UNIFORM)], ids=["headwise", "head_uniform"])
def test_wait_that_runs_out_sets_timeout_and_context_recovers(w):
    """Failure detection without a fault: with a zero wait budget the first
    device wait that is not already complete gives up, the status word says
    HTTM_DEV_TIMEOUT, the kernels free what they hold and exit; with the
    default budget restored the same plan gives the same bits as before."""
    _, plan, _, (Q, K, V), _ = _case(w)
    ref = B.httm_forward(plan, Q, K, V, workspace=plan.new_workspace())
    ws = plan.new_workspace()
    B.httm_set_wait_budget(plan, 0)
    B.httm_forward(plan, Q, K, V, workspace=ws)
    assert B.httm_get_device_status(plan, ws) & B.HTTM_DEV_TIMEOUT
    B.httm_set_wait_budget(plan, 2_000_000_000)
    again = B.httm_forward(plan, Q, K, V, workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    assert torch.equal(again, ref)


@pytest.mark.parametrize("w", [MID, WORKLOADS["vggt_30f"], MID.with_(mode=HEAD_UNIFORM)],
                         ids=["mid", "vggt_30f", "mid_head_uniform"])
def test_forward_records_into_a_cuda_graph(w):
    """A forward captured on a stream (its key branch forked onto the plan's
    own stream and joined back by events) replays to the eager call's bits,
    and re-plans from the data on each replay: new Q, K, V in the captured
    buffers give the eager output of the new inputs."""
    w, plan, _, (Q, K, V), _ = _case(w)
    ws = plan.new_workspace()
    eager = B.httm_forward(plan, Q, K, V, workspace=ws)       # first call binds the plan to the device
    torch.cuda.synchronize()
    ws_g = plan.new_workspace()
    out_g = torch.empty_like(Q)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        B.httm_forward(plan, Q, K, V, out=out_g, workspace=ws_g)
    g.replay()
    torch.cuda.synchronize()
    assert B.httm_get_device_status(plan, ws_g) == 0
    assert torch.equal(out_g, eager)
    Q2, K2, V2 = PL.inputs(w.with_(seed=w.seed + 1))
    Q.copy_(Q2), K.copy_(K2), V.copy_(V2)
    g.replay()
    eager2 = B.httm_forward(plan, Q2, K2, V2, workspace=ws)
    torch.cuda.synchronize()
    assert B.httm_get_device_status(plan, ws_g) == 0
    assert torch.equal(out_g, eager2)
    assert not torch.equal(eager2, eager)
    del g


@pytest.mark.parametrize("w", [MID, MID.with_(T=1, n_t=1), MID.with_(out_pct=100),
                               MID.with_(mode=CONTIGUOUS, contig_block=384), WORKLOADS["vggt_30f"]],
                         ids=["mid", "split_parts", "all_outliers", "contiguous", "vggt_30f"])
def test_fused_unmerge_is_bit_identical(w):
    """httm_set_fused_unmerge: the attention epilogue (and the merge of the
    last wave's split items) writes each output row straight to its tokens
    -- a slot's non-outlier members, or the outlier itself -- instead of O~
    plus an unmerge kernel.  Same bits as the default path, clean status,
    also when every eligible query is an outlier (drained slots)."""
    _, plan, _, (Q, K, V), _ = _case(w)
    ref = B.httm_forward(plan, Q, K, V, workspace=plan.new_workspace())
    B.httm_set_fused_unmerge(plan, True)
    ws = plan.new_workspace()
    got = B.httm_forward(plan, Q, K, V, out=torch.full_like(Q, float("nan")), workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    assert torch.equal(got, ref)
    B.httm_set_fused_unmerge(plan, False)
