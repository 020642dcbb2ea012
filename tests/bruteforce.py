"""Pure-Python brute force for tiny inputs, written independently of the oracle.

Block membership is derived token by token from (frame t, patch p) instead of
from the oracle's block table, cosines are double loops over plain floats, and
the orderings use Python's sorted() on explicit tuples.  Used only to pin the
oracle on inputs small enough for loops.
"""
from __future__ import annotations

import math


def block_of_token(n: int, P: int, n_s: int, n_t: int, T: int):
    """(block number, in-block index) of original token n under the temporal
    blocking: region j = p // n_s, group g = t // n_t, frame-major inside."""
    t, p = divmod(n, P)
    R = (P + n_s - 1) // n_s
    g, j = t // n_t, p // n_s
    s_j = min(n_s, P - j * n_s)
    tau, sigma = t - g * n_t, p - j * n_s
    return g * R + j, tau * s_j + sigma


def blocks_by_enumeration(T: int, P: int, n_s: int, n_t: int):
    """Dict block -> list of original tokens ordered by in-block index."""
    tmp = {}
    for n in range(T * P):
        b, i = block_of_token(n, P, n_s, n_t, T)
        tmp.setdefault(b, []).append((i, n))
    return {b: [n for _, n in sorted(v)] for b, v in tmp.items()}


def cos(a, b):
    na = math.sqrt(sum(x * x for x in a))
    nb = math.sqrt(sum(x * x for x in b))
    if na == 0.0 or nb == 0.0:
        return 0.0
    return sum(x * y for x, y in zip(a, b)) / (na * nb)


def match_block(rows, stride, pct):
    """rows: list of vectors in in-block order.  Returns (best, score, merged)
    dicts keyed by in-block source index; best is an in-block dst index."""
    n_b = len(rows)
    dst = [i for i in range(n_b) if i % stride == 0]
    src = [i for i in range(n_b) if i % stride != 0]
    best, score = {}, {}
    for s in src:
        bi, bv = None, None
        for t in dst:  # ascending: strict '>' keeps the lowest index on ties
            c = cos(rows[s], rows[t])
            if bv is None or c > bv:
                bi, bv = t, c
        best[s], score[s] = bi, bv
    r_b = pct * n_b // 100
    ranked = sorted(src, key=lambda s: (-score[s], s))
    merged = {s: False for s in src}
    for s in ranked[:r_b]:
        merged[s] = True
    return best, score, merged


def groups(n_b, stride, best, merged):
    """Member lists: one per dst (ascending), then one per kept src."""
    dst = [i for i in range(n_b) if i % stride == 0]
    src = [i for i in range(n_b) if i % stride != 0]
    out = [[t] + [s for s in src if merged[s] and best[s] == t] for t in dst]
    out += [[s] for s in src if not merged[s]]
    return out


def top_k_outliers(dev, eligible, k):
    """dev, eligible: lists over flat index h*N + n.  First k eligible by
    (dev desc, flat asc)."""
    cand = [f for f in range(len(dev)) if eligible[f]]
    ranked = sorted(cand, key=lambda f: (-dev[f], f))
    return set(ranked[:k])


def softmax_attention_row(q, Ks, Vs, scale):
    z = [scale * sum(a * b for a, b in zip(q, k)) for k in Ks]
    m = max(z)
    w = [math.exp(v - m) for v in z]
    s = sum(w)
    return [sum(w[j] * Vs[j][c] for j in range(len(Ks))) / s for c in range(len(Vs[0]))]


def partition_roles(score, grid, ga_pct):
    """LiteVGGT's token classes by loops: score is a list (frames) of lists
    (raster patches).  Returns a list of lists of 'ga' / 'dst' / 'src'."""
    P = grid * grid
    k = ga_pct * P // 100
    out = []
    for t, row in enumerate(score):
        by_importance = sorted(range(P), key=lambda p: (-row[p], p))
        ga = set(by_importance[:k])
        roles = ['ga' if p in ga else None for p in range(P)]
        if t == 0:
            roles = ['ga' if p in ga else 'dst' for p in range(P)]
            out.append(roles)
            continue
        for cy in range(0, grid, 2):
            for cx in range(0, grid, 2):
                members = [y * grid + x for y in range(cy, min(cy + 2, grid))
                           for x in range(cx, min(cx + 2, grid))]
                free = [p for p in members if p not in ga]
                if not free:
                    continue
                anchor = min(free, key=lambda p: (row[p], p))
                for p in free:
                    roles[p] = 'dst' if p == anchor else 'src'
        out.append(roles)
    return out


def match_block_roles(rows, roles):
    """rows, roles: in-block order.  Every 'src' joins its most similar 'dst'
    (ties: the lowest in-block index); 'ga' tokens and the sources of a block
    without destinations stay alone.  Returns the member lists: one per dst
    in ascending order, then one per singleton in ascending order."""
    dst = [i for i, r in enumerate(roles) if r == 'dst']
    join = {}
    for s, r in enumerate(roles):
        if r != 'src' or not dst:
            continue
        bi, bv = None, None
        for t in dst:
            c = cos(rows[s], rows[t])
            if bv is None or c > bv:
                bi, bv = t, c
        join[s] = bi
    groups_ = [[t] + [s for s in sorted(join) if join[s] == t] for t in dst]
    groups_ += [[i] for i, r in enumerate(roles) if r != 'dst' and i not in join]
    return groups_
