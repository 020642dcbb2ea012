"""Pins of the LiteVGGT partition oracle (``oracle.litevggt_partition``),
CPU only: pure-Python brute force of the three token classes and of the
matching inside blocks, the invariants the LiteVGGT note states (GA share per
frame, the first frame anchors, one lowest-scoring destination per 2x2
cell), special cases that reduce to plain attention, and a planted mistake
that the checks must catch."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.httm_oracle as O
import oracle.litevggt_partition as L
from tests import bruteforce as BF
from token_merging_view_b200.inputs import make_qkv, make_score

ROLE = {"src": L.ROLE_SRC, "dst": L.ROLE_DST, "ga": L.ROLE_GA}


def _rand_score(rng, T, grid, levels):
    return rng.integers(0, levels, size=(T, grid * grid)).astype(np.float64)   # many ties


@pytest.mark.parametrize("seed", range(16))
def test_partition_vs_bruteforce(seed):
    rng = np.random.default_rng(seed)
    T, grid = int(rng.integers(1, 5)), int(rng.integers(1, 8))
    ga_pct = int(rng.choice([0, 10, 25, 60, 100]))
    score = _rand_score(rng, T, grid, int(rng.integers(1, 5)))
    got = L.partition_roles(score, grid, ga_pct)
    want = BF.partition_roles(score.tolist(), grid, ga_pct)
    assert got.tolist() == [[ROLE[r] for r in row] for row in want]


def _follows_the_note(score, roles, grid, ga_pct) -> bool:
    """The classes the note describes: per frame the ga_pct share of highest
    scores is GA; the first frame's other tokens are destinations; in later
    frames each 2x2 cell with a non-GA token has exactly one destination, its
    lowest-scoring non-GA token."""
    T, P = score.shape
    cell = L.cell_of_patch(grid)
    for t in range(T):
        ga = roles[t] == L.ROLE_GA
        if ga.sum() != L.ga_count(P, ga_pct) or (ga.any() and (~ga).any() and
                                                 score[t, ga].min() < score[t, ~ga].max()):
            return False
        if t == 0:
            if not np.all(roles[t][~ga] == L.ROLE_DST):
                return False
            continue
        for c in np.unique(cell):
            members = np.nonzero((cell == c) & ~ga)[0]
            if members.size == 0:
                continue
            dst = members[roles[t, members] == L.ROLE_DST]
            if dst.size != 1 or score[t, dst[0]] != score[t, members].min():
                return False
    return True


def test_partition_follows_the_note_on_a_vggt_frame_grid():
    grid, T, ga_pct = 37, 4, 10
    score = make_score(T=T, grid=grid, seed=3).double().numpy()
    roles = L.partition_roles(score, grid, ga_pct)
    assert L.ga_count(grid * grid, ga_pct) == 136
    assert ((grid + 1) // 2) ** 2 == 361          # 19 x 19 cells, the last row and column one patch wide
    assert _follows_the_note(score, roles, grid, ga_pct)


def _tiny_layer(T=3, grid=6, h=2, d=8, seed=7, ga_pct=10):
    Q, K, V = make_qkv(T=T, grid=grid, h=h, d=d, seed=seed, noise_sigma=0.3, max_shift=1, dtype=torch.float32)
    q, k, v = (t.double().numpy() for t in (Q, K, V))
    score = make_score(T=T, grid=grid, seed=seed + 1).double().numpy()
    cfg = O.OracleConfig(h=h, T=T, P=grid * grid, d=d, n_s=12, n_t=2, out_pct=10)
    return cfg, q, k, v, L.partition_roles(score, grid, ga_pct)


def test_matching_and_groups_vs_bruteforce():
    cfg, q, k, v, roles = _tiny_layer()
    blocks = O.block_list(cfg)
    flat = roles.reshape(-1)
    names = {L.ROLE_SRC: "src", L.ROLE_DST: "dst", L.ROLE_GA: "ga"}
    for X in (q, k):
        plan = L.plan_tensor_partition(X, blocks, roles)
        for hh in range(cfg.h):
            for toks in blocks:
                rows = [X[hh, n].tolist() for n in toks]
                want = BF.match_block_roles(rows, [names[int(flat[n])] for n in toks])
                got = {}
                for i, n in enumerate(toks):
                    got.setdefault(int(plan.slot[hh, n]), []).append(i)
                # slot order: destinations' groups first, then singletons, each ascending
                assert [sorted(got[s]) for s in sorted(got)] == [sorted(g) for g in want]
        assert np.all(plan.merged[:, flat == L.ROLE_SRC] | (plan.best[:, flat == L.ROLE_SRC] < 0))
        assert not plan.merged[:, flat != L.ROLE_SRC].any()


def test_merged_means_follow_the_partition():
    cfg, q, k, v, roles = _tiny_layer()
    blocks = O.block_list(cfg)
    flat = roles.reshape(-1)
    qp = L.plan_tensor_partition(q, blocks, roles)
    kp = L.plan_tensor_partition(k, blocks, roles)
    res = O.forward_plan(cfg, q, k, v, q_plan=qp, k_plan=kp)
    for hh in range(cfg.h):
        for s in range(kp.n_slots):
            members = np.nonzero(kp.slot[hh] == s)[0]
            np.testing.assert_allclose(res.v_means[hh, s], v[hh, members].mean(axis=0), rtol=0, atol=1e-12)
    # slots per head: in each block its destinations and GA tokens, plus its
    # sources when the block has no destination
    want = 0
    for toks in blocks:
        r = flat[toks]
        n_dst = int((r == L.ROLE_DST).sum())
        want += n_dst + int((r == L.ROLE_GA).sum()) + (0 if n_dst else int((r == L.ROLE_SRC).sum()))
    assert qp.n_slots == kp.n_slots == want


@pytest.mark.parametrize("case", ["all_ga", "first_frame_only"])
def test_no_merging_cases_equal_dense_attention(case):
    """Every token GA (ga = 100 %), or a single frame (all destinations):
    nothing merges, so the layer is plain attention."""
    T = 1 if case == "first_frame_only" else 3
    cfg, q, k, v, roles = _tiny_layer(T=T, ga_pct=100 if case == "all_ga" else 10)
    blocks = O.block_list(cfg)
    res = O.forward(cfg, q, k, v, q_plan=L.plan_tensor_partition(q, blocks, roles),
                    k_plan=L.plan_tensor_partition(k, blocks, roles))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), scale=cfg.softmax_scale).numpy()
    np.testing.assert_allclose(res.out, want, rtol=0, atol=1e-12)


def test_planted_cell_rule_mistake_is_caught():
    """A partition that anchors each cell on its HIGHEST-scoring non-GA
    token must fail both the brute force and the note's rule check."""
    rng = np.random.default_rng(0)
    grid, T, ga_pct = 6, 3, 10
    score = rng.standard_normal((T, grid * grid))
    good = L.partition_roles(score, grid, ga_pct)
    bad = good.copy()
    cell = L.cell_of_patch(grid)
    for t in range(1, T):
        for c in np.unique(cell):
            free = np.nonzero((cell == c) & (good[t] != L.ROLE_GA))[0]
            if free.size:
                bad[t, free] = L.ROLE_SRC
                bad[t, free[np.argmax(score[t, free])]] = L.ROLE_DST
    want = BF.partition_roles(score.tolist(), grid, ga_pct)
    assert good.tolist() == [[ROLE[r] for r in row] for row in want]
    assert _follows_the_note(score, good, grid, ga_pct)
    assert bad.tolist() != good.tolist()
    assert not _follows_the_note(score, bad, grid, ga_pct)
