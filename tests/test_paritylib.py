"""The parity helpers themselves, on the CPU: the slot-sampled output check
finds no error in the oracle's own output, covers every token of each
sampled slot, and sees an error planted in one of them."""
from __future__ import annotations

import numpy as np

import oracle.httm_oracle as O
from tests import paritylib as PL
from token_merging_view_b200.workloads import Workload

W = Workload("t", T=3, grid=12, h=3, d=16, fp32=True, n_s=48, n_t=3, q_stride=4, kv_stride=4,
             q_pct=60, kv_pct=50, out_pct=10, seed=5, noise_sigma=0.3, max_shift=1)


def _oracle():
    Q, K, V = PL.inputs(W, device="cpu")
    cfg = PL.oracle_cfg(W)
    q, k, v = (PL.to64(t) for t in (Q, K, V))
    return cfg, O.forward_plan(cfg, q, k, v), O.forward(cfg, q, k, v).out


def test_slot_sampling_of_the_oracle_output_is_exact():
    cfg, res, out = _oracle()
    mx, rl2, n = PL.sample_slot_error(res, out, cfg, 10)
    assert mx < 1e-12 and rl2 < 1e-12 and n == 10 * W.h
    mx, rl2, n = PL.sample_slot_error(res, out, cfg, 1 << 30)
    assert mx < 1e-12 and n == sum(np.unique(res.restore.slot_final[hh]).size for hh in range(W.h))


def test_slot_sampling_sees_a_planted_error_in_a_fanned_out_token():
    cfg, res, out = _oracle()
    sf = res.restore.slot_final[1]
    slots, counts = np.unique(sf, return_counts=True)
    big = slots[np.argmax(counts)]                 # a merged slot with several tokens
    tok = np.nonzero(sf == big)[0][-1]             # its last member
    bad = out.copy()
    bad[1, tok, 0] += 0.5
    mx, _, _ = PL.sample_slot_error(res, bad, cfg, 1 << 30)
    assert abs(mx - 0.5) < 1e-9


def test_shared_slot_tokens_drops_exactly_the_moved_groups():
    """A plan that moves one token from one group to another and renumbers
    the slots: only the members of the two changed groups drop out, and a
    slot renumbering alone (same members) keeps every token."""
    cfg, res, out = _oracle()
    o = res.restore.slot_final
    perm = np.random.default_rng(0).permutation(int(o.max()) + 1)
    g = perm[o]                                     # renumbered, same members
    assert PL.shared_slot_tokens(o, g).all()
    sf = o[2]
    slots, counts = np.unique(sf, return_counts=True)
    a, b = slots[np.argsort(-counts)[:2]]           # two merged groups
    mover = np.nonzero(sf == a)[0][-1]
    g2 = g.copy()
    g2[2, mover] = perm[b]
    ok = PL.shared_slot_tokens(o, g2)
    assert ok[:2].all()
    changed = (sf == a) | (sf == b)
    assert np.array_equal(ok[2], ~changed)
    # the restricted output check still sees a planted error on a kept token
    bad = out.copy()
    keep = np.nonzero(~changed)[0][0]
    bad[2, keep, 1] -= 0.25
    mx, _, _ = PL.sample_slot_error(res, bad, cfg, 1 << 30, token_ok=ok)
    assert abs(mx - 0.25) < 1e-9
    bad2 = out.copy()
    bad2[2, mover, 1] -= 0.25                       # an excluded token is not compared
    mx, _, _ = PL.sample_slot_error(res, bad2, cfg, 1 << 30, token_ok=ok)
    assert mx < 1e-12
