"""The head-sharded outlier selection, as a protocol, against the oracle's
global top-d% (key design 3 of the HTTM note: one budget over all heads'
queries, ties by flat index h * N + n).

Each shard holds a contiguous run of heads.  What the shards share is only
sums: the eligible count and the key histograms (so every shard finds the
same k-th largest key T and the same number `need` of keys equal to T that
the budget still takes), and one count per shard of its keys equal to T.
Shard s takes every key above T and the first
min(eq_s, max(0, need - sum of eq over the shards before s)) of its keys
equal to T in flat order.  This restates that rule in plain numpy, shard by
shard, and checks that the union of the shards' masks is the oracle's mask
for random deviations with many ties, random eligibility and uneven head
splits (the CUDA kernels take the same steps; they are compared with the
unsharded layer on the GPU)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle.httm_oracle as O


def keys_of(dev: np.ndarray, eligible: np.ndarray) -> np.ndarray:
    # 32-bit keys that order like the deviations (dev >= 0), 0 = ineligible
    bits = dev.astype(np.float32).view(np.uint32).astype(np.uint64)
    return np.where(eligible, bits + 1, 0)


def sharded_masks(dev, eligible, pct, bounds, prefix=True):
    h, N = dev.shape
    keys = keys_of(dev, eligible)
    # summed over shards: the eligible count and the key histogram (here the
    # sorted keys stand in for the three radix passes over summed histograms)
    n_elig = sum(int(eligible[a:b].sum()) for a, b in bounds)
    k = O.outlier_count(h, N, pct, n_elig)
    masks = []
    if k == 0:
        return [np.zeros((b - a, N), dtype=bool) for a, b in bounds]
    all_keys = np.concatenate([keys[a:b].ravel() for a, b in bounds])
    T = np.sort(all_keys)[::-1][k - 1]
    gt = sum(int((keys[a:b] > T).sum()) for a, b in bounds)
    need = k - gt
    eq = [int((keys[a:b] == T).sum()) for a, b in bounds]      # summed as a per-shard vector
    for s, (a, b) in enumerate(bounds):
        before = sum(eq[:s]) if prefix else 0     # prefix=False: the planted mistake below
        take = min(eq[s], max(0, need - before))
        local = keys[a:b].ravel()
        m = local > T
        ties = np.nonzero(local == T)[0][:take]                  # flat order inside the shard
        m[ties] = True
        masks.append(m.reshape(b - a, N))
    return masks


@pytest.mark.parametrize("seed", range(12))
def test_sharded_selection_equals_global_selection(seed):
    rng = np.random.default_rng(seed)
    h = int(rng.integers(2, 9))
    N = int(rng.integers(1, 300))
    levels = int(rng.integers(1, 6))          # few distinct deviations: many ties
    dev = rng.integers(0, levels, size=(h, N)).astype(np.float64) * 0.25
    eligible = rng.random((h, N)) < rng.uniform(0.2, 1.0)
    pct = int(rng.integers(0, 101))
    cuts = np.sort(rng.choice(np.arange(1, h), size=int(rng.integers(0, h)), replace=False))
    edges = [0, *cuts.tolist(), h]
    bounds = list(zip(edges[:-1], edges[1:]))
    want = O.select_outliers(dev, eligible, pct)
    got = np.concatenate(sharded_masks(dev, eligible, pct, bounds))
    assert np.array_equal(got, want)


def test_quota_crosses_shard_boundaries():
    # all eligible deviations equal: the budget is one tie, taken head by head
    h, N, pct = 4, 50, 60
    dev = np.zeros((h, N))
    eligible = np.ones((h, N), dtype=bool)
    masks = sharded_masks(dev, eligible, pct, [(0, 1), (1, 2), (2, 3), (3, 4)])
    assert [int(m.sum()) for m in masks] == [50, 50, 20, 0]
    assert np.array_equal(np.concatenate(masks), O.select_outliers(dev, eligible, pct))



def test_planted_quota_mistake_is_caught():
    """A shard that ignored the shards before it (taking min(eq_s, need)
    equal keys) would select too many: the comparison must see it."""
    h, N, pct = 4, 50, 60
    dev = np.zeros((h, N))
    eligible = np.ones((h, N), dtype=bool)
    bounds = [(0, 1), (1, 2), (2, 3), (3, 4)]
    got = np.concatenate(sharded_masks(dev, eligible, pct, bounds, prefix=False))
    assert not np.array_equal(got, O.select_outliers(dev, eligible, pct))
