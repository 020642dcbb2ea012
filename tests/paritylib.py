"""Helpers for comparing the CUDA path with the fp64 oracle.

Inputs come from the seeded generator and are handed to both sides as the
same bytes.  Nothing computed by the CUDA path is ever fed to the oracle:
where fp32 (GPU) and fp64 (oracle) may legitimately pick differently -- a
destination tied within rounding, a source at the top-r boundary, a query at
the outlier threshold -- the mismatch is excused only if the ORACLE's own
values put the two candidates within the stated margin (1e-4).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle.httm_oracle as O
from token_merging_view_b200 import binding as B
from token_merging_view_b200.inputs import make_qkv
from token_merging_view_b200.workloads import Workload

TIE = 1e-4           # near-tie margin of the plan comparison
FEAT_REL = 1e-3      # merged features (fp32 exports) vs fp64, per-vector relative L2
OUT_MAX_ABS = 2e-2   # attention output with the oracle's plan injected
OUT_REL_L2 = 1e-2


def oracle_cfg(w: Workload) -> O.OracleConfig:
    return O.OracleConfig(h=w.h, T=w.T, P=w.P, d=w.d, n_s=w.n_s, n_t=w.n_t, q_stride=w.q_stride,
                          kv_stride=w.kv_stride, q_pct=w.q_pct, kv_pct=w.kv_pct, out_pct=w.out_pct,
                          mode=w.mode, contig_block=w.contig_block)


def inputs(w: Workload, device="cuda"):
    dt = torch.float32 if w.fp32 else torch.bfloat16
    Q, K, V = make_qkv(T=w.T, grid=w.grid, h=w.h, d=w.d, seed=w.seed, noise_sigma=w.noise_sigma,
                       max_shift=w.max_shift, dtype=dt, device=device)
    return Q, K, V


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def cpu(x):
    return {k: v.cpu().numpy() for k, v in x.items()}


def oracle_plan_tensors(res: O.OracleResult, device="cuda", mask=True) -> dict:
    """The oracle's plan in the injection format of httm_forward_with_plan."""
    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a.astype(np.int32))).to(device)

    def u8(a):
        return torch.from_numpy(np.ascontiguousarray(a.astype(np.uint8))).to(device)
    d = dict(q_best=i32(res.q_plan.best), q_merged=u8(res.q_plan.merged),
             k_best=i32(res.k_plan.best), k_merged=u8(res.k_plan.merged))
    if mask:
        d["outlier"] = u8(res.mask)
    return d


def compare_best(X64: np.ndarray, plan: O.TensorPlan, g_best: np.ndarray, g_score: np.ndarray) -> int:
    """Destination choice per source.  Returns the number of excused mismatches;
    asserts on any other."""
    src = ~plan.is_dst
    mism = (g_best != plan.best) & src[None, :]
    excused = 0
    for hh, n in zip(*np.nonzero(mism)):
        t = int(g_best[hh, n])
        assert 0 <= t < X64.shape[1] and plan.is_dst[t], (hh, n, t)
        c = O.cosine_similarity(X64[hh, n][None], X64[hh, t][None])[0, 0]
        gap = plan.score[hh, n] - c
        assert gap < TIE, f"head {hh} token {n}: GPU dst {t} is {gap:.3g} below the best"
        excused += 1
    # a source whose block has no destination (possible under LiteVGGT's
    # partition) has no match: the oracle's score is nan, nothing to compare
    agree = src[None, :] & ~mism & ~np.isnan(plan.score)
    err = np.abs(g_score - plan.score)[agree]
    assert err.size == 0 or err.max() < 1e-5, f"score error {err.max():.3g}"
    return excused


def compare_merged(blocks, stride: int, pct: int, plan: O.TensorPlan, g_merged: np.ndarray) -> int:
    """Top-r membership; a mismatch is excused when the oracle's score of that
    source lies within TIE of its block's r-boundary."""
    excused = 0
    h = g_merged.shape[0]
    for toks in blocks:
        n_b = toks.shape[0]
        _, src_i = O.split_dst_src(n_b, stride)
        r_b = O.merge_count(n_b, pct)
        st = toks[src_i]
        for hh in range(h):
            g = g_merged[hh, st].astype(bool)
            o = plan.merged[hh, st]
            assert g.sum() == r_b
            bad = np.nonzero(g != o)[0]
            if bad.size == 0:
                continue
            sc = np.sort(plan.score[hh, st])[::-1]
            lo = sc[r_b] if r_b < sc.shape[0] else -np.inf
            hi = sc[r_b - 1] if r_b > 0 else np.inf
            for k in bad:
                s = plan.score[hh, st[k]]
                assert min(abs(s - lo), abs(s - hi)) < TIE, (hh, st[k], s, lo, hi)
                excused += 1
    return excused


def rel_rows(g: np.ndarray, o: np.ndarray) -> np.ndarray:
    num = np.linalg.norm(g - o, axis=-1)
    den = np.maximum(np.linalg.norm(o, axis=-1), 1e-3)
    return num / den


def compare_mask(res: O.OracleResult, g_mask: np.ndarray) -> int:
    o = res.mask
    bad = np.nonzero(g_mask.astype(bool) != o)
    if bad[0].size == 0:
        return 0
    dev = res.dev[res.eligible]
    k = int(o.sum())
    thr = np.sort(dev)[::-1][k - 1] if k > 0 else 0.0
    for hh, n in zip(*bad):
        assert abs(res.dev[hh, n] - thr) < TIE * max(1.0, thr), (hh, n, res.dev[hh, n], thr)
    return bad[0].size


def bf16_ulps(g: torch.Tensor, o: np.ndarray) -> int:
    """Max distance in bf16 units between g (bf16) and o rounded to bf16."""
    ob = torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16)
    gi = g.cpu().view(torch.int16).to(torch.int32)
    oi = ob.view(torch.int16).to(torch.int32)
    return int((gi - oi).abs().max()) if gi.numel() else 0


def sample_out_error(res: O.OracleResult, out_g: np.ndarray, cfg: O.OracleConfig, tokens_per_head: int,
                     seed: int = 0):
    """Oracle attention for a seeded sample of tokens per head (all tokens if
    the head is small); returns (max abs error, relative L2 error)."""
    rng = np.random.default_rng(seed)
    h, N, _ = out_g.shape
    errs, nums, dens = [], 0.0, 0.0
    for hh in range(h):
        toks = np.arange(N) if N <= tokens_per_head else np.sort(rng.choice(N, tokens_per_head, replace=False))
        slots = res.restore.slot_final[hh, toks]
        uniq, inv = np.unique(slots, return_inverse=True)
        qt = res.restore.q_tilde[hh][uniq]
        o = O.attention(qt, res.k_means[hh], res.v_means[hh], cfg.softmax_scale)[inv]
        g = out_g[hh, toks]
        errs.append(np.abs(g - o).max())
        nums += float(((g - o) ** 2).sum())
        dens += float((o ** 2).sum())
    return max(errs), np.sqrt(nums / dens)


def shared_slot_tokens(o_slot: np.ndarray, g_slot: np.ndarray) -> np.ndarray:
    """[h, N] bool: the tokens whose final query slot holds the same members
    on both sides (the oracle's slot map and the GPU's exported one).  A slot
    is identified by its members, not its number: (count, sum and minimum of
    the member indices) of the token's slot must agree.  A near-tie that the
    plan comparison excused moves a few tokens between slots (and renumbers
    later singletons or outlier ranks); only the tokens of those slots drop
    out, the output of every other token must match the oracle's."""
    h, N = o_slot.shape
    n = np.arange(N, dtype=np.int64)
    ok = np.zeros((h, N), dtype=bool)

    def sig(s):
        ns = int(s.max()) + 1
        cnt = np.bincount(s, minlength=ns)
        tot = np.bincount(s, weights=n.astype(np.float64), minlength=ns)   # exact below 2^53
        order = np.lexsort((n, s))
        first = np.full(ns, N, dtype=np.int64)
        ss = s[order]
        start = np.r_[True, ss[1:] != ss[:-1]]
        first[ss[start]] = n[order][start]
        return cnt[s], tot[s], first[s]

    for hh in range(h):
        a, b = sig(np.asarray(o_slot[hh], dtype=np.int64)), sig(np.asarray(g_slot[hh], dtype=np.int64))
        ok[hh] = (a[0] == b[0]) & (a[1] == b[1]) & (a[2] == b[2])
    return ok


def sample_slot_error(res: O.OracleResult, out_g, cfg: O.OracleConfig, slots_per_head: int, seed: int = 0,
                      token_ok: np.ndarray | None = None):
    """Oracle attention for a seeded sample of the live query slots of each
    head (all of them if the head has fewer), compared at every token whose
    output comes from a sampled slot, so the unmerge's fan-out is checked as
    well.  out_g: the GPU output, a torch tensor (any device) or an array,
    [h, N, d].  token_ok ([h, N] bool, optional) restricts the comparison to
    those tokens (and the sample to slots holding one).  Returns (max abs
    error, relative L2 error, slots compared)."""
    rng = np.random.default_rng(seed)
    h = res.restore.slot_final.shape[0]
    errs, nums, dens, n_slots = [], 0.0, 0.0, 0
    for hh in range(h):
        sf = res.restore.slot_final[hh]
        live = np.unique(sf if token_ok is None else sf[token_ok[hh]])   # drained slots are read by no token
        chosen = live if live.size <= slots_per_head else np.sort(rng.choice(live, slots_per_head, replace=False))
        toks = np.nonzero(np.isin(sf, chosen) & (True if token_ok is None else token_ok[hh]))[0]
        inv = np.searchsorted(chosen, sf[toks])
        o = O.attention(res.restore.q_tilde[hh][chosen], res.k_means[hh], res.v_means[hh], cfg.softmax_scale)[inv]
        if isinstance(out_g, torch.Tensor):
            g = out_g[hh][torch.from_numpy(toks).to(out_g.device)].double().cpu().numpy()
        else:
            g = np.asarray(out_g[hh, toks], dtype=np.float64)
        errs.append(np.abs(g - o).max())
        nums += float(((g - o) ** 2).sum())
        dens += float((o ** 2).sum())
        n_slots += chosen.size
    return max(errs), np.sqrt(nums / dens), n_slots


def run(plan: B.Plan, Q, K, V, injected=None, debug=True, fields=None):
    """One forward through the C ABI; `fields` limits the debug exports to
    those names (the others stay NULL), all of them by default."""
    dbg = B.debug_buffers(plan) if debug else None
    if dbg is not None and fields is not None:
        dbg = {k: v for k, v in dbg.items() if k in fields}
    ws = plan.new_workspace()
    if injected is not None:
        out = B.httm_forward_with_plan(plan, Q, K, V, injected, dbg, workspace=ws)
    elif debug:
        out = B.httm_forward_debug(plan, Q, K, V, dbg, workspace=ws)
    else:
        out = B.httm_forward(plan, Q, K, V, workspace=ws)
    status = B.httm_get_device_status(plan, ws)
    return out, (cpu(dbg) if debug else None), ws, status


def plant_big_groups(w: Workload, Q, K, V):
    """Near-copies of every block's first destination: about 60 % of each
    block's sources (the same tokens in Q and K, every head) become that
    destination's row plus Gaussian noise of a per-token size in [0.02, 1.2]
    (rows have unit-variance entries), so that the destination's group draws
    far more than 32 members and its noisiest members have the largest
    deviations of the layer (the outliers)."""
    cfg = oracle_cfg(w)
    assert cfg.q_stride == cfg.kv_stride
    g = torch.Generator().manual_seed(w.seed + 101)
    picks = []
    for toks in O.block_list(cfg):
        src = toks[np.arange(toks.shape[0]) % cfg.q_stride != 0]
        keep = torch.rand(src.shape[0], generator=g).numpy() < 0.6
        picks.append((int(toks[0]), torch.from_numpy(src[keep])))
    for X in (Q, K):
        Xc = X.float().cpu()
        for d0, pick in picks:
            eps = 0.02 + 1.18 * torch.rand(pick.shape[0], generator=g)
            noise = torch.randn(w.h, pick.shape[0], w.d, generator=g)
            Xc[:, pick] = Xc[:, d0][:, None, :] + eps[None, :, None] * noise
        X.copy_(Xc.to(X.dtype))


def group_sizes(plan: O.TensorPlan) -> np.ndarray:
    """Members per group (the destination itself included), per head."""
    out = []
    for hh in range(plan.best.shape[0]):
        dst = plan.best[hh][plan.merged[hh]]
        out.append(np.bincount(dst, minlength=plan.best.shape[1]) + plan.is_dst)
    return np.stack(out)
