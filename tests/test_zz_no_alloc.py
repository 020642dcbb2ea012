"""The allocation-free outlier selection, for callers that cannot allocate
device memory (they are handed only input/output buffers, or must not risk a
device-synchronising cudaMalloc), against the mask the forward exports.

Collected last on purpose: the entry point shares one scratch array inside
the library, and this file must pass both on its own in a fresh process and
after every other test has used the library."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.httm_oracle as O

from token_merging_view_b200 import binding as B
from token_merging_view_b200.inputs import make_qkv
from token_merging_view_b200.workloads import Workload

pytestmark = pytest.mark.gpu

# 8 frames of the 37 x 37 grid, 4 heads: several selection chunks per head.
W = Workload("noalloc_8f", T=8, grid=37, h=4, d=64, fp32=False, n_s=128, n_t=3, q_stride=4, kv_stride=4,
             q_pct=70, kv_pct=50, out_pct=10, seed=21, noise_sigma=0.3, max_shift=2)


def _eligible(q_best: torch.Tensor, q_merged: torch.Tensor) -> torch.Tensor:
    """Queries in a group of >= 2 tokens: every merged source, and every
    destination that received one."""
    elig = q_merged.clone()
    h = q_best.shape[0]
    for hh in range(h):
        m = q_merged[hh].bool()
        elig[hh, q_best[hh, m].long()] = 1
    return elig


def test_no_alloc_selection_matches_forward_twice():
    torch.cuda.set_device(0)
    Q, K, V = make_qkv(T=W.T, grid=W.grid, h=W.h, d=W.d, seed=W.seed, device="cuda")
    plan = B.httm_plan(B.LayerConfig.from_workload(W))
    ws = plan.new_workspace()
    dbg = B.debug_buffers(plan)
    B.httm_forward_debug(plan, Q, K, V, dbg, workspace=ws)
    assert B.httm_get_device_status(plan, ws) == 0
    dev = dbg["dev"].contiguous()
    elig = _eligible(dbg["q_best"], dbg["q_merged"])
    want_mask = dbg["outlier"]
    want_n = B.workspace_view(plan, ws, "n_out").clone()
    assert int(want_mask.sum()) == W.out_pct * W.h * W.N // 100
    for _ in range(2):   # the scratch keeps the last call's contents: a second call must not see them
        mask, n_out = B.httm_select_outliers_noalloc(dev, elig, W.out_pct)
        torch.cuda.synchronize()
        assert torch.equal(mask, want_mask)
        assert torch.equal(n_out, want_n)
    # a different budget in between, then the original again
    mask0, n0 = B.httm_select_outliers_noalloc(dev, elig, 0)
    torch.cuda.synchronize()
    assert int(mask0.sum()) == 0 and int(n0.sum()) == 0
    mask, n_out = B.httm_select_outliers_noalloc(dev, elig, W.out_pct)
    torch.cuda.synchronize()
    assert torch.equal(mask, want_mask) and torch.equal(n_out, want_n)


def test_no_alloc_rejects_sizes_beyond_its_scratch():
    dev = torch.zeros((65, 8), dtype=torch.float32, device="cuda")
    elig = torch.zeros((65, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(B.HttmError) as e:
        B.httm_select_outliers_noalloc(dev, elig, 10)          # 65 heads
    assert e.value.status == 2
    lib = B.load_library()
    big_n = (1 << 25) // 4 + 1                                  # 4 heads x this > 33,554,432 tokens
    st = lib.httm_select_outliers_noalloc(dev.data_ptr(), elig.data_ptr(), 4, big_n, 10, elig.data_ptr(),
                                          dev.data_ptr(), None)
    assert st == 2                                              # HTTM_ERR_UNSUPPORTED, nothing enqueued


def _tie_case(name: str):
    """Deviations with many exact ties (values on a coarse grid, exactly
    representable in fp32), eligibility masks and budgets that exercise the
    radix select's tie handling: equal keys spanning several 4096-query
    chunks and several heads, and a budget above the number of eligible
    queries."""
    rng = np.random.default_rng({"all_equal": 1, "few_eligible": 2, "grid": 3, "grid_big": 4}[name])
    if name == "all_equal":            # every eligible deviation equal: the first k flat indices win
        h, N, pct = 3, 9000, 10
        elig = rng.random((h, N)) < 0.6
        dev = np.where(elig, 1.5, 0.0)
    elif name == "few_eligible":       # pct = 100 with 50 eligible queries: all of them, no more
        h, N, pct = 4, 5000, 100
        elig = np.zeros((h, N), dtype=bool)
        elig.reshape(-1)[rng.choice(h * N, 50, replace=False)] = True
        dev = np.where(elig, np.round(rng.random((h, N)) * 2) / 2, 0.0)
    elif name == "grid":               # five values (0 included) shared by thousands of queries
        h, N, pct = 4, 10000, 10
        elig = rng.random((h, N)) < 0.7
        dev = np.where(elig, np.round(rng.random((h, N)) * 4) / 4, 0.0)
    else:                              # a larger budget with the threshold inside a big tie
        h, N, pct = 5, 13000, 37
        elig = rng.random((h, N)) < 0.8
        dev = np.where(elig, np.round(rng.random((h, N)) * 8) / 8, 0.0)
    return dev.astype(np.float32), elig, pct


@pytest.mark.parametrize("name", ["all_equal", "few_eligible", "grid", "grid_big"])
def test_no_alloc_selection_matches_oracle_on_ties(name):
    """The allocation-free selection against the oracle's global top-d%
    (deviation desc, flat index asc; k = min(floor(d% h N / 100), #eligible))
    on inputs where a radix select's tie handling decides the mask."""
    torch.cuda.set_device(0)
    dev32, elig, pct = _tie_case(name)
    want = O.select_outliers(dev32.astype(np.float64), elig, pct)
    dev_t = torch.from_numpy(dev32).cuda()
    elig_t = torch.from_numpy(elig.astype(np.uint8)).cuda()
    for _ in range(2):
        mask, n_out = B.httm_select_outliers_noalloc(dev_t, elig_t, pct)
        torch.cuda.synchronize()
        assert np.array_equal(mask.cpu().numpy().astype(bool), want)
        assert np.array_equal(n_out.cpu().numpy(), want.sum(axis=1).astype(np.int32))
