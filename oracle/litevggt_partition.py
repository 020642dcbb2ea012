"""fp64 CPU oracle of LiteVGGT's token partition, used as the destination
rule inside HTTM's temporal blocks (the next alternative to the
i % stride rule; no CUDA path exists for it yet).

TEST INFRASTRUCTURE ONLY, like ``oracle.httm_oracle``: only the tests may
import it; the library never does, and it imports nothing from the library.

Source: the note "LiteVGGT: Boosting Vanilla VGGT via Geometry-aware Cached
Token Merging" (papernotes.org, CVPR 2026), sections

* key design 1 (geometry-aware feature map): every token gets a geometric
  importance score M_GA, a weighted sum of a normalised pixel-gradient map and
  a normalised local-variance map -- here the score is an INPUT, one float per
  token shared by all heads (the map needs images, which are not here; the
  tests pass a seeded smooth field in its place);
* key design 2 (three token classes): per frame, the top 10 % by score are
  geometry-aware (GA) tokens, excluded from merging; destinations are all
  tokens of the first frame plus, in every other frame, the lowest-scoring
  token of each 2x2 cell of the patch grid; the rest are sources, each
  assigned to the destination it is most similar to;
* key design 3 (merge and unmerge): cosine matching of source to
  destination, x_d <- (x_d + sum of its sources) / (1 + |S_d|), and unmerge
  copies the merged token back to every member -- the same mean and unmerge
  as HTTM's, so the rest of the layer is ``oracle.httm_oracle.forward_plan``
  with the plans built here passed in.

Readings taken where the note is silent or in conflict:

* "all first-frame tokens are destinations" and "GA tokens are excluded from
  merging" overlap on the first frame's GA tokens: exclusion wins, they stay
  singletons there too (a destination's value changes when sources join it);
* the GA count per frame is floor(ga_pct * P / 100); ties in the score go to
  the lower patch index, both for GA (higher score first) and for a cell's
  destination (lower score first);
* cells start at even grid rows and columns; on an odd-sized grid the last
  row and column of cells are 2x1, 1x2 or 1x1; a cell whose tokens are all GA
  has no destination;
* matching stays inside HTTM's temporal blocks and is per head (key design 1
  of the HTTM note); within a block every source merges into its most
  similar destination (no top-r: the partition fixes the ratio), ties to the
  lowest destination index; a block without destinations keeps its sources
  as singletons;
* the cells are those of each frame's full patch grid, whichever temporal
  block region their tokens fall in.
"""
from __future__ import annotations

import numpy as np

from oracle.httm_oracle import TensorPlan, best_match, block_slots, cosine_similarity

ROLE_SRC, ROLE_DST, ROLE_GA = 0, 1, 2


def ga_count(P: int, ga_pct: int) -> int:
    """GA tokens per frame: floor(ga_pct * P / 100)."""
    return (ga_pct * P) // 100


def cell_of_patch(grid: int) -> np.ndarray:
    """2x2 cell index of every raster patch p of a grid x grid patch grid."""
    p = np.arange(grid * grid)
    py, px = p // grid, p % grid
    return (py // 2) * ((grid + 1) // 2) + px // 2


def partition_roles(score: np.ndarray, grid: int, ga_pct: int = 10) -> np.ndarray:
    """Role of every token (ROLE_SRC / ROLE_DST / ROLE_GA), int8 [T, P], from
    the score [T, P] (p raster on the grid x grid patch grid)."""
    T, P = score.shape
    assert P == grid * grid
    roles = np.full((T, P), ROLE_SRC, dtype=np.int8)
    k = ga_count(P, ga_pct)
    p = np.arange(P)
    cell = cell_of_patch(grid)
    for t in range(T):
        ga = np.lexsort((p, -score[t]))[:k]             # highest scores, lower p first
        roles[t, ga] = ROLE_GA
        rest = np.nonzero(roles[t] != ROLE_GA)[0]
        if t == 0:
            roles[t, rest] = ROLE_DST                       # the first frame anchors the others
            continue
        order = rest[np.lexsort((rest, score[t, rest], cell[rest]))]   # by cell, then score asc, p asc
        first = np.ones(order.size, dtype=bool)
        first[1:] = cell[order[1:]] != cell[order[:-1]]
        roles[t, order[first]] = ROLE_DST
    return roles


def plan_tensor_partition(X: np.ndarray, blocks: list[np.ndarray], roles: np.ndarray) -> TensorPlan:
    """Per head and block: every source merges into its most similar
    destination of the block; GA tokens (and the sources of a block without
    destinations) stay singletons.  Slots as in HTTM's plan: the block's
    destinations' groups in ascending in-block order, then its singletons."""
    h, N, _ = X.shape
    roles = np.asarray(roles).reshape(-1)
    is_dst = roles == ROLE_DST
    best = np.full((h, N), -1, dtype=np.int64)
    score = np.full((h, N), np.nan)
    merged = np.zeros((h, N), dtype=bool)
    slot = np.empty((h, N), dtype=np.int64)
    base = 0
    bases = []
    for toks in blocks:
        n_b = toks.shape[0]
        r = roles[toks]
        dst_i = np.nonzero(r == ROLE_DST)[0]
        src_i = np.nonzero(r != ROLE_DST)[0]                # sources and GA tokens, ascending
        wants = r[src_i] == ROLE_SRC
        for hh in range(h):
            if dst_i.size:
                b, s = best_match(cosine_similarity(X[hh, toks[src_i]], X[hh, toks[dst_i]]))
                m = wants.copy()
                best[hh, toks[src_i]] = toks[dst_i[b]]
                score[hh, toks[src_i]] = s
            else:
                b = np.zeros(src_i.size, dtype=np.int64)
                m = np.zeros(src_i.size, dtype=bool)
            sl, n_slots_b = block_slots(n_b, dst_i, src_i, b, m)
            merged[hh, toks[src_i]] = m
            slot[hh, toks] = base + sl
        bases.append(base)
        base += n_slots_b
    return TensorPlan(is_dst, best, score, merged, slot, base, bases)
