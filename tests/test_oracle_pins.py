"""Pins of the fp64 oracle against things other than itself: brute force on
tiny inputs, closed forms, a library attention routine, the ratios the HTTM
note prints, and planted mistakes that the pins must catch.  CPU only."""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.httm_oracle as O
from tests import bruteforce as bf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# Blocks and reorder
# --------------------------------------------------------------------------

def _sizes(T, P, n_s, n_t):
    out = {}
    for b in O.temporal_blocks(T, P, n_s, n_t):
        out[b.shape[0]] = out.get(b.shape[0], 0) + 1
    return out


def check_block_sizes():
    # counts computed by hand from T = 30 G + rest, P = 1369 = 10 * 128 + 89
    assert _sizes(4, 64, 16, 4) == {64: 4}
    assert _sizes(30, 1369, 128, 30) == {3840: 10, 2670: 1}
    assert _sizes(100, 1369, 128, 30) == {3840: 30, 2670: 3, 1280: 10, 890: 1}
    assert _sizes(500, 1369, 128, 30) == {3840: 160, 2670: 16, 2560: 10, 1780: 1}
    assert _sizes(1000, 1369, 128, 30) == {3840: 330, 2670: 33, 1280: 10, 890: 1}


def test_block_sizes():
    check_block_sizes()


def check_blocks_vs_enumeration(T, P, n_s, n_t):
    enum = bf.blocks_by_enumeration(T, P, n_s, n_t)
    blocks = O.temporal_blocks(T, P, n_s, n_t)
    assert len(blocks) == len(enum)
    for b, toks in enumerate(blocks):
        assert toks.tolist() == enum[b]


@pytest.mark.parametrize("T,P,n_s,n_t", [(4, 64, 16, 4), (7, 50, 16, 3), (5, 37, 8, 2), (3, 1369, 128, 30)])
def test_blocks_vs_enumeration(T, P, n_s, n_t):
    check_blocks_vs_enumeration(T, P, n_s, n_t)


def test_reorder_inverse_identity():
    for (T, P, n_s, n_t) in [(4, 64, 16, 4), (7, 50, 16, 3), (100, 1369, 128, 30)]:
        blocks = O.temporal_blocks(T, P, n_s, n_t)
        perm = np.concatenate(blocks)
        assert np.array_equal(np.sort(perm), np.arange(T * P))  # a bijection
    X = _rng(1).standard_normal((3, 7 * 50, 4))
    blocks = O.temporal_blocks(7, 50, 16, 3)
    Xb = O.reorder(X, blocks)
    assert not np.array_equal(Xb, X)
    assert np.array_equal(O.inverse_reorder(Xb, blocks), X)


def test_contiguous_blocks():
    sizes = [b.shape[0] for b in O.contiguous_blocks(10_000, 3840)]
    assert sizes == [3840, 3840, 2320]
    last = O.contiguous_blocks(1_369_000, 3840)[-1]
    assert last.shape[0] == 1_369_000 % 3840 == 1960
    assert np.array_equal(np.concatenate(O.contiguous_blocks(10_000, 3840)), np.arange(10_000))


# --------------------------------------------------------------------------
# Matching and top-r
# --------------------------------------------------------------------------

def _plan_single_block(rows, stride, pct):
    X = np.asarray(rows, dtype=np.float64)[None]          # [1, n_b, d]
    blocks = [np.arange(X.shape[1])]
    return O.plan_tensor(X, blocks, stride, pct)


def check_match_vs_bruteforce(seed, n_b, d, stride, pct, ties=False):
    rng = _rng(seed)
    rows = rng.standard_normal((n_b, d))
    if ties:  # duplicate destinations and a zero row force ties
        rows[stride] = rows[0]
        rows[1] = 0.0
        rows[2] = rows[3]
    best, score, merged = bf.match_block(rows.tolist(), stride, pct)
    plan = _plan_single_block(rows, stride, pct)
    for s in best:
        assert plan.best[0, s] == best[s], (s, plan.best[0, s], best[s])
        assert abs(plan.score[0, s] - score[s]) < 1e-12
        assert bool(plan.merged[0, s]) == merged[s]
    # slots: the brute-force groups, in order, are the slots
    for k, members in enumerate(bf.groups(n_b, stride, best, merged)):
        for m in members:
            assert plan.slot[0, m] == k


@pytest.mark.parametrize("seed,n_b,d,stride,pct", [
    (0, 16, 5, 4, 50), (1, 24, 3, 4, 25), (2, 17, 6, 4, 70), (3, 40, 4, 8, 85), (4, 9, 2, 4, 60)])
def test_match_vs_bruteforce(seed, n_b, d, stride, pct):
    check_match_vs_bruteforce(seed, n_b, d, stride, pct)


def test_match_vs_bruteforce_ties():
    check_match_vs_bruteforce(5, 16, 4, 4, 50, ties=True)


def check_one_hot_ties():
    e = np.eye(4)
    rows = np.zeros((8, 4))
    rows[0] = e[0]; rows[4] = e[0]          # two identical destinations
    rows[1] = e[0]                           # cos 1 with both -> lowest dst (0)
    rows[2] = 0.0                            # zero row -> cos 0 everywhere -> dst 0
    rows[3] = e[1]                           # cos 0 with both -> dst 0
    rows[5] = e[0] + e[1]                    # cos 1/sqrt(2) with both -> dst 0
    rows[6] = -e[0]                          # cos -1 with both -> dst 0
    rows[7] = e[0]
    plan = _plan_single_block(rows, 4, 25)   # r_b = 2
    assert plan.best[0, [1, 2, 3, 5, 6, 7]].tolist() == [0, 0, 0, 0, 0, 0]
    assert plan.score[0, 1] == 1.0 and plan.score[0, 2] == 0.0 and plan.score[0, 6] == -1.0
    # two sources with score 1 (i = 1 and i = 7): both merge (score desc, index asc)
    assert plan.merged[0].tolist() == [False, True, False, False, False, False, False, True]


def test_one_hot_ties():
    check_one_hot_ties()


def test_topr_order_on_equal_scores():
    score = np.array([0.5, 0.9, 0.5, 0.9, 0.1])
    assert O.select_top_r(score, 3).tolist() == [True, True, False, True, False]
    with pytest.raises(ValueError):
        O.select_top_r(score, 6)


def test_identical_tokens_merge_with_zero_deviation():
    x = _rng(3).standard_normal(6)
    Q = np.tile(x, (1, 32, 1))                                  # [1, 32, 6]
    cfg = O.OracleConfig(h=1, T=2, P=16, d=6, n_s=16, n_t=2, q_stride=4, kv_stride=4,
                         q_pct=50, kv_pct=25, out_pct=10)
    res = O.forward_plan(cfg, Q, Q, Q)
    src = [i for i in range(32) if i % 4]
    r_b = 16
    assert res.q_plan.merged[0, src].tolist() == [True] * r_b + [False] * (24 - r_b)
    assert np.all(res.q_plan.best[0, src] == 0)
    assert np.allclose(res.q_means[0], x, rtol=0, atol=1e-15)
    assert np.all(res.dev < 1e-14)           # zero up to the rounding of the mean


# --------------------------------------------------------------------------
# Means, deviation, outlier filter, restore
# --------------------------------------------------------------------------

def test_two_member_group_closed_form():
    rng = _rng(7)
    rows = rng.standard_normal((8, 3)) * 0.01
    a, b = np.array([1.0, 0.2, 0.0]), np.array([0.9, 0.3, 0.05])
    rows[4] = a                      # a destination
    rows[5] = b                      # the only source merged (r_b = 1)
    rows[0] = np.array([0.0, 0.0, 1.0])
    rows[[1, 2, 3, 6, 7]] = np.array([0.0, -1.0, 0.3]) + rng.standard_normal((5, 3)) * 0.3
    Q = rows[None]
    cfg = O.OracleConfig(h=1, T=1, P=8, d=3, n_s=8, n_t=1, q_stride=4, kv_stride=4,
                         q_pct=13, kv_pct=13, out_pct=0)     # r_b = floor(13 * 8 / 100) = 1
    res = O.forward_plan(cfg, Q, Q, Q)
    merged_src = np.nonzero(res.q_plan.merged[0])[0].tolist()
    assert merged_src == [5] and res.q_plan.best[0, 5] == 4
    half = np.linalg.norm(a - b) / 2
    assert abs(res.dev[0, 4] - half) < 1e-15 and abs(res.dev[0, 5] - half) < 1e-15
    assert np.count_nonzero(res.dev) == 2
    assert np.allclose(res.q_means[0, res.q_plan.slot[0, 4]], (a + b) / 2, atol=1e-15)


def test_group_means_vs_bruteforce():
    rng = _rng(11)
    rows = rng.standard_normal((24, 4))
    best, score, merged = bf.match_block(rows.tolist(), 4, 60)
    plan = _plan_single_block(rows, 4, 60)
    means = O.group_means(rows[None], plan.slot, plan.n_slots)[0]
    for k, members in enumerate(bf.groups(24, 4, best, merged)):
        want = [sum(rows[m][c] for m in members) / len(members) for c in range(4)]
        assert np.allclose(means[k], want, rtol=0, atol=1e-14)


def test_restore_closed_form_and_drained():
    rows = np.array([[1.0, 0.0], [0.9, 0.1], [0.95, -0.1], [0.0, 1.0],
                     [1.0, 0.05], [0.1, 0.9], [0.2, 1.0], [0.0, 0.8]])
    Q = rows[None]
    blocks = [np.arange(8)]
    best = np.full((1, 8), -1)
    merged = np.zeros((1, 8), dtype=bool)
    # group of dst 0: {0, 1, 2}; group of dst 4: {4, 5}
    best[0, [1, 2, 3, 5, 6, 7]] = [0, 0, 0, 4, 4, 4]
    merged[0, [1, 2, 5]] = True
    plan = O.plan_from_choice(blocks, 4, best, merged)
    mask = np.zeros((1, 8), dtype=bool)
    mask[0, 2] = True                   # one outlier of the 3-member group
    mask[0, [4, 5]] = True              # the whole 2-member group: drained
    rest = O.restore_outliers(Q, plan.slot, plan.n_slots, mask)
    g0 = plan.slot[0, 0]
    s = rows[0] + rows[1] + rows[2]
    assert np.allclose(rest.means[0, g0], (s - rows[2]) / (3 - 1), atol=1e-15)
    assert not rest.live[0, plan.slot[0, 4]]
    # outlier slots after the regular ones, ascending n
    assert rest.slot_final[0, 2] == plan.n_slots and rest.slot_final[0, 4] == plan.n_slots + 1
    assert rest.slot_final[0, 5] == plan.n_slots + 2
    assert np.array_equal(rest.q_tilde[0][plan.n_slots:], rows[[2, 4, 5]])
    assert rest.n_out.tolist() == [3]


def test_outlier_select_vs_bruteforce():
    rng = _rng(5)
    h, N = 3, 40
    dev = np.round(rng.random((h, N)) * 4) / 4          # many exact ties
    eligible = rng.random((h, N)) < 0.7
    dev[~eligible] = 0.0
    for pct in (0, 5, 10, 37, 100):
        mask = O.select_outliers(dev, eligible, pct)
        k = min(pct * h * N // 100, int(eligible.sum()))
        want = bf.top_k_outliers(dev.reshape(-1).tolist(), eligible.reshape(-1).tolist(), k)
        assert set(np.nonzero(mask.reshape(-1))[0].tolist()) == want
        assert mask.sum() == k


def _tiny_cfg(**kw):
    base = dict(h=2, T=4, P=64, d=16, n_s=16, n_t=4, q_stride=4, kv_stride=4,
                q_pct=50, kv_pct=25, out_pct=10)
    base.update(kw)
    return O.OracleConfig(**base)


def _tiny_qkv(seed=0, h=2, N=256, d=16):
    rng = _rng(seed)
    return tuple(rng.standard_normal((h, N, d)) for _ in range(3))


def test_partition_and_counts():
    cfg = _tiny_cfg()
    Q, K, V = _tiny_qkv()
    res = O.forward_plan(cfg, Q, K, V)
    for plan, pct in ((res.q_plan, cfg.q_pct), (res.k_plan, cfg.kv_pct)):
        for hh in range(cfg.h):
            counts = np.bincount(plan.slot[hh], minlength=plan.n_slots)
            assert counts.sum() == cfg.N and counts.min() >= 1
        for toks in O.block_list(cfg):
            r_b = O.merge_count(toks.shape[0], pct)
            assert np.all(plan.merged[:, toks].sum(axis=1) == r_b)
        assert plan.n_slots == sum(t.shape[0] - O.merge_count(t.shape[0], pct) for t in O.block_list(cfg))
    k_o = O.outlier_count(cfg.h, cfg.N, cfg.out_pct, int(res.eligible.sum()))
    assert res.mask.sum() == k_o == 51


def test_zero_outlier_pct_keeps_the_merge():
    cfg = _tiny_cfg(out_pct=0)
    Q, K, V = _tiny_qkv(1)
    res = O.forward_plan(cfg, Q, K, V)
    assert not res.mask.any()
    for hh in range(cfg.h):
        assert np.allclose(res.restore.q_tilde[hh], res.q_means[hh], rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _sdpa(Q, K, V):
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x)) for x in (Q, K, V))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()


def check_no_merge_equals_dense_sdpa():
    cfg = _tiny_cfg(q_pct=0, kv_pct=0, out_pct=10)
    Q, K, V = _tiny_qkv(2)
    res = O.forward(cfg, Q, K, V)
    assert not res.mask.any()            # no merged query, nothing eligible
    assert np.allclose(res.out, _sdpa(Q, K, V), rtol=1e-10, atol=1e-12)


def test_no_merge_equals_dense_sdpa():
    check_no_merge_equals_dense_sdpa()


def test_dense_mode_equals_sdpa():
    cfg = _tiny_cfg(mode=O.DENSE)
    Q, K, V = _tiny_qkv(3)
    assert np.allclose(O.forward(cfg, Q, K, V).out, _sdpa(Q, K, V), rtol=1e-10, atol=1e-12)


def test_attention_special_cases():
    rng = _rng(9)
    q = rng.standard_normal((5, 8))
    k1, v1 = rng.standard_normal((1, 8)), rng.standard_normal((1, 3))
    assert np.allclose(O.attention(q, k1, v1, 0.3), np.repeat(v1, 5, 0), atol=1e-15)
    k = np.tile(rng.standard_normal((1, 8)), (6, 1))
    v = rng.standard_normal((6, 3))
    assert np.allclose(O.attention(q, k, v, 0.3), np.tile(v.mean(0), (5, 1)), atol=1e-14)


def test_attention_vs_bruteforce_rows():
    rng = _rng(10)
    q, k, v = rng.standard_normal((4, 6)), rng.standard_normal((9, 6)), rng.standard_normal((9, 5))
    got = O.attention(q, k, v, 1 / math.sqrt(6))
    for r in range(4):
        want = bf.softmax_attention_row(q[r].tolist(), k.tolist(), v.tolist(), 1 / math.sqrt(6))
        assert np.allclose(got[r], want, atol=1e-13)


def test_full_forward_vs_bruteforce_tiny():
    """The whole layer on the 4-frame, 8x8-grid case against loops only."""
    cfg = _tiny_cfg(h=1)
    Q, K, V = _tiny_qkv(4, h=1)
    res = O.forward(cfg, Q, K, V)
    enum = bf.blocks_by_enumeration(cfg.T, cfg.P, cfg.n_s, cfg.n_t)
    q_groups, k_groups = [], []
    dev, elig = [0.0] * cfg.N, [False] * cfg.N
    for b in sorted(enum):
        toks = enum[b]
        for X, stride, pct, acc in ((Q, cfg.q_stride, cfg.q_pct, q_groups),
                                    (K, cfg.kv_stride, cfg.kv_pct, k_groups)):
            rows = [X[0, n].tolist() for n in toks]
            best, _, merged = bf.match_block(rows, stride, pct)
            acc.append([[toks[i] for i in g] for g in bf.groups(len(toks), stride, best, merged)])
    q_slots = [g for blk in q_groups for g in blk]
    k_slots = [g for blk in k_groups for g in blk]

    def mean(X, g):
        return [sum(X[0, n, c] for n in g) / len(g) for c in range(cfg.d)]

    for g in q_slots:
        if len(g) >= 2:
            m = mean(Q, g)
            for n in g:
                dev[n] = math.sqrt(sum((Q[0, n, c] - m[c]) ** 2 for c in range(cfg.d)))
                elig[n] = True
    k_o = min(cfg.out_pct * cfg.N // 100, sum(elig))
    outl = bf.top_k_outliers(dev, elig, k_o)
    q_rows, slot_of = [], {}
    for k, g in enumerate(q_slots):
        keep = [n for n in g if n not in outl]
        for n in keep:
            slot_of[n] = k
        q_rows.append(mean(Q, keep) if keep else None)
    for n in sorted(outl):
        slot_of[n] = len(q_rows)
        q_rows.append(Q[0, n].tolist())
    Ks = [mean(K, g) for g in k_slots]
    Vs = [mean(V, g) for g in k_slots]
    scale = 1 / math.sqrt(cfg.d)
    assert res.mask[0].sum() == k_o
    assert set(np.nonzero(res.mask[0])[0].tolist()) == outl
    for n in range(cfg.N):
        want = bf.softmax_attention_row(q_rows[slot_of[n]], Ks, Vs, scale)
        assert np.allclose(res.out[0, n], want, atol=1e-12), n


def test_head_uniform_is_one_plan_for_all_heads():
    cfg = _tiny_cfg(mode=O.HEAD_UNIFORM)
    Q, K, V = _tiny_qkv(6)
    res = O.forward_plan(cfg, Q, K, V)
    assert np.array_equal(res.q_plan.slot[0], res.q_plan.slot[1])
    # the plan is the argmax of the head-mean cosine, by brute force on block 0
    toks = O.block_list(cfg)[0]
    src = [i for i in range(64) if i % 4]
    dst = [i for i in range(64) if i % 4 == 0]
    for s in src[:6]:
        cbar = [(bf.cos(Q[0, toks[s]], Q[0, toks[t]]) + bf.cos(Q[1, toks[s]], Q[1, toks[t]])) / 2 for t in dst]
        assert res.q_plan.best[0, toks[s]] == toks[dst[int(np.argmax(cbar))]]


# --------------------------------------------------------------------------
# The ratios and split the HTTM note prints
# --------------------------------------------------------------------------

def test_page_ratios():
    facts = json.load(open(os.path.join(GOLDEN, "page_facts.json")))
    n_b = facts["n_s"]["value"] * facts["n_t"]["value"]
    assert n_b == facts["n_b"]["value"]
    dst, src = O.split_dst_src(n_b, 4)
    assert dst.shape[0] / n_b == facts["dst_share"]["value"]
    assert src.shape[0] / n_b == facts["src_share"]["value"]
    assert abs(facts["dst_share"]["value"] * facts["src_share"]["value"] - facts["match_flops_coeff"]["value"]) < 0.01
    # one full 128 x 30 block per head; Q dst every 10th so 90% can merge
    h, d = 2, 8
    cfg = O.OracleConfig(h=h, T=30, P=128, d=d, n_s=128, n_t=30, q_stride=10, kv_stride=4,
                         q_pct=facts["q_merge_pct"]["value"], kv_pct=facts["kv_merge_pct"]["value"],
                         out_pct=facts["q_filter_pct"]["value"])
    rng = _rng(12)
    Q, K, V = (rng.standard_normal((h, cfg.N, d)) for _ in range(3))
    res = O.forward_plan(cfg, Q, K, V)
    lq = sum(q.shape[0] for q in res.restore.q_tilde)
    assert lq / (h * cfg.N) == pytest.approx(facts["q_final_ratio"]["value"], abs=1e-12)
    assert res.k_plan.n_slots / cfg.N == pytest.approx(facts["kv_final_ratio"]["value"], abs=1e-12)


# --------------------------------------------------------------------------
# Planted mistakes: each must make a pin fail
# --------------------------------------------------------------------------

def test_planted_argmax_tie_mistake_is_caught(monkeypatch):
    def last_max(sim):
        rev = sim[:, ::-1]
        best = sim.shape[1] - 1 - np.argmax(rev, axis=1)
        return best, sim[np.arange(sim.shape[0]), best]
    monkeypatch.setattr(O, "best_match", last_max)
    with pytest.raises(AssertionError):
        check_one_hot_ties()


def test_planted_topr_order_mistake_is_caught(monkeypatch):
    def ascending(score, r_b):
        order = np.lexsort((np.arange(score.shape[0]), score))
        m = np.zeros(score.shape[0], dtype=bool)
        m[order[:r_b]] = True
        return m
    monkeypatch.setattr(O, "select_top_r", ascending)
    with pytest.raises(AssertionError):
        check_match_vs_bruteforce(0, 16, 5, 4, 50)


def test_planted_transposed_block_mistake_is_caught(monkeypatch):
    real = O.temporal_blocks

    def region_major(T, P, n_s, n_t):
        out = []
        for b in real(T, P, n_s, n_t):
            t_g = len({int(n) // P for n in b})
            out.append(b.reshape(t_g, -1).T.reshape(-1))
        return out
    monkeypatch.setattr(O, "temporal_blocks", region_major)
    with pytest.raises(AssertionError):
        check_blocks_vs_enumeration(4, 64, 16, 4)


def test_planted_scale_mistake_is_caught(monkeypatch):
    real = O.attention
    monkeypatch.setattr(O, "attention", lambda q, k, v, s, chunk=1024: real(q, k, v, 1.0, chunk))
    with pytest.raises(AssertionError):
        check_no_merge_equals_dense_sdpa()


def test_planted_mean_mistake_is_caught(monkeypatch):
    def sum_not_mean(X, slot, n_slots):
        return O.group_sums(X, slot, n_slots)[0]
    monkeypatch.setattr(O, "group_means", sum_not_mean)
    with pytest.raises(AssertionError):
        test_group_means_vs_bruteforce()


# --------------------------------------------------------------------------
# The input generator (no method arithmetic; shape, determinism, scale)
# --------------------------------------------------------------------------

def test_generator_deterministic_and_unit_field():
    from token_merging_view_b200.inputs import make_qkv
    a = make_qkv(T=3, grid=37, h=2, d=8, seed=5)
    b = make_qkv(T=3, grid=37, h=2, d=8, seed=5)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert a[0].shape == (2, 3 * 1369, 8) and a[0].dtype == torch.bfloat16
    q = make_qkv(T=2, grid=37, h=4, d=64, seed=1, noise_sigma=0.0, max_shift=0, dtype=torch.float32)[0]
    assert 0.6 < float(q.std()) < 1.4          # unit-variance field
    # with no noise and no shift, frame 1 repeats frame 0 exactly
    assert torch.equal(q[:, :1369], q[:, 1369:])
