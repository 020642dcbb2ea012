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
