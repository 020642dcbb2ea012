"""fp64 CPU oracle for HTTM's merged global-attention layer.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain restatement of the
method that the CUDA library is checked against.  Only the tests, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import
it; the library never does, and it imports nothing from the library.

Source of the method: the note "HTTM: Head-wise Temporal Token Merging for
Faster VGGT" (papernotes.org, CVPR 2026), sections

* overall framework (flowchart): merge per head before the attention kernel,
  attend on the shortened Q~/K~/V~, unmerge and undo the reorder afterwards;
* key design 1 (head-wise merging): per head, split tokens into a source set S
  and a destination set D, Sim = RowNorm(S) . RowNorm(D)^T, every source keeps
  only its most similar destination, the top-r sources are merged, a merged
  token is the mean of its members, Q and K are merged independently and V
  follows K's plan, unmerge copies a merged token's output back to each member;
* key design 2 (temporal reordering + in-block merging): the n_s-token spatial
  region of n_t adjacent frames is stacked into one block of n_b = n_s * n_t
  tokens and merging happens only inside blocks;
* key design 3 (cross-head adaptive outlier filter): after a first merge, each
  original query's L2 deviation from its merged token (0 if it was not merged),
  a global top-d% over all heads gives a mask M_o in {0,1}^{h x N}, and each
  outlier's contribution is removed from its merged token and the outlier is
  kept as a token of its own (queries only);
* training strategy: n_s = 128, n_t = 30, bf16 + FlashAttention.

The mean update is the same as LiteVGGT's x_d <- (x_d + sum_{s in S_d} x_s) /
(1 + |S_d|) ("LiteVGGT: Boosting Vanilla VGGT via Geometry-aware Cached Token
Merging", key design 3).

Readings taken where the pages are silent:

* spatial regions are contiguous raster ranges of the patch index p, the last
  one partial; temporal groups are runs of n_t frames, the last one partial;
* tokens inside a block are frame-major (frame slice after frame slice);
  block b = g * R + j for temporal group g and region j;
* destinations are the in-block indices i with i % stride == 0, sources the
  rest (the pages give only the 25 % / 75 % split);
* r counts a fraction of the block: r_b = floor(r% * n_b / 100);
* argmax ties go to the lowest destination index; top-r orders sources by
  (score desc, in-block index asc); a zero-norm row has cosine 0;
* merged tokens are plain means (no size weighting in attention);
* a destination counts as merged for the deviation when its group has >= 2
  members; k_o = min(floor(d% * h * N / 100), #eligible), ordered by
  (deviation desc, flat index h*N + n asc), one shot;
* several outliers in one group are all subtracted; a group whose members are
  all outliers is left drained (its slot is read by no token);
* outlier slots are appended per head after the regular slots in ascending n;
* attention scale 1 / sqrt(d_head), plain max-subtracted softmax.

Every number here is fp64.  Nothing is blocked, fused or reordered beyond what
the definitions state; attention rows are evaluated in chunks only to bound
memory (each row's softmax is computed independently, exactly as defined).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

HEADWISE_TEMPORAL = 0
HEAD_UNIFORM = 1
CONTIGUOUS = 2
DENSE = 3


@dataclass(frozen=True)
class OracleConfig:
    h: int
    T: int
    P: int
    d: int
    n_s: int = 128
    n_t: int = 30
    q_stride: int = 4
    kv_stride: int = 4
    q_pct: int = 70
    kv_pct: int = 50
    out_pct: int = 10
    mode: int = HEADWISE_TEMPORAL
    contig_block: int = 3840
    scale: float | None = None

    @property
    def N(self) -> int:
        return self.T * self.P

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale else 1.0 / np.sqrt(self.d)


# --------------------------------------------------------------------------
# Blocks and temporal reordering (key design 2)
# --------------------------------------------------------------------------

def temporal_blocks(T: int, P: int, n_s: int, n_t: int) -> list[np.ndarray]:
    """Spatio-temporal merge blocks of key design 2.

    Block b = g * R + j stacks spatial region j (patches [j*n_s, j*n_s + s_j))
    of the n_t frames of temporal group g (frames [g*n_t, g*n_t + t_g)).  Entry
    i = tau * s_j + sigma of the returned array is the original token index
    (g*n_t + tau) * P + j*n_s + sigma.
    """
    G = -(-T // n_t)
    R = -(-P // n_s)
    blocks = []
    for g in range(G):
        t0 = g * n_t
        t_g = min(n_t, T - t0)
        for j in range(R):
            p0 = j * n_s
            s_j = min(n_s, P - p0)
            tau = np.arange(t_g).reshape(t_g, 1)
            sigma = np.arange(s_j).reshape(1, s_j)
            blocks.append(((t0 + tau) * P + p0 + sigma).reshape(-1))
    return blocks


def contiguous_blocks(N: int, n_b: int) -> list[np.ndarray]:
    """Blocks cut straight along the sequence (the un-reordered variant of key
    design 2, whose matches stay near the diagonal): runs of n_b tokens, the
    last one partial."""
    return [np.arange(s, min(N, s + n_b)) for s in range(0, N, n_b)]


def block_list(cfg: OracleConfig) -> list[np.ndarray]:
    if cfg.mode == CONTIGUOUS:
        return contiguous_blocks(cfg.N, cfg.contig_block)
    return temporal_blocks(cfg.T, cfg.P, cfg.n_s, cfg.n_t)


def reorder(X: np.ndarray, blocks: list[np.ndarray]) -> np.ndarray:
    """[h, N, d] in original order -> [h, N, d] in block order."""
    return X[:, np.concatenate(blocks)]


def inverse_reorder(Xb: np.ndarray, blocks: list[np.ndarray]) -> np.ndarray:
    """[h, N, d] in block order -> original order (the inverse permutation)."""
    out = np.empty_like(Xb)
    out[:, np.concatenate(blocks)] = Xb
    return out


# --------------------------------------------------------------------------
# Bipartite matching inside a block (key design 1)
# --------------------------------------------------------------------------

def split_dst_src(n_b: int, stride: int) -> tuple[np.ndarray, np.ndarray]:
    """Destination set = in-block indices divisible by ``stride``; the rest are
    sources, both ascending."""
    i = np.arange(n_b)
    return i[i % stride == 0], i[i % stride != 0]


def row_normalize(X: np.ndarray) -> np.ndarray:
    """RowNorm: each row divided by its L2 norm; an all-zero row stays zero
    (its cosine with anything is 0)."""
    n = np.sqrt((X * X).sum(axis=-1, keepdims=True))
    return np.divide(X, n, out=np.zeros_like(X), where=n > 0)


def cosine_similarity(S: np.ndarray, D: np.ndarray) -> np.ndarray:
    """Sim = RowNorm(S) . RowNorm(D)^T  (key design 1)."""
    return row_normalize(S) @ row_normalize(D).T


def best_match(sim: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Each source keeps only its most similar destination.  Ties go to the
    lowest destination index (numpy's argmax returns the first maximum)."""
    best = np.argmax(sim, axis=1)
    score = sim[np.arange(sim.shape[0]), best]
    return best, score


def merge_count(n_b: int, pct: int) -> int:
    """r_b = floor(pct * n_b / 100), in integers."""
    return (pct * n_b) // 100


def select_top_r(score: np.ndarray, r_b: int) -> np.ndarray:
    """Boolean mask of the r_b sources merged: order by (score desc, source
    position asc) and take the first r_b.  Sources are passed in ascending
    in-block order, so position order is in-block index order."""
    n_src = score.shape[0]
    if r_b > n_src:
        raise ValueError(f"r_b={r_b} exceeds the {n_src} sources of the block")
    order = np.lexsort((np.arange(n_src), -score))
    merged = np.zeros(n_src, dtype=bool)
    merged[order[:r_b]] = True
    return merged


def block_slots(n_b: int, dst_i: np.ndarray, src_i: np.ndarray,
                best: np.ndarray, merged: np.ndarray) -> tuple[np.ndarray, int]:
    """Slot of every in-block token.  Slot k < n_dst is destination k's group
    {t} + {merged s : best(s) = t}; the kept sources follow as singletons in
    ascending in-block order."""
    n_dst = dst_i.shape[0]
    slot = np.empty(n_b, dtype=np.int64)
    slot[dst_i] = np.arange(n_dst)
    kept = src_i[~merged]
    slot[kept] = n_dst + np.arange(kept.shape[0])
    slot[src_i[merged]] = best[merged]
    return slot, n_dst + kept.shape[0]


@dataclass
class TensorPlan:
    """Merge plan of one tensor (Q, or K which V follows), every array [h, N]
    in original token order."""
    is_dst: np.ndarray          # bool [N]
    best: np.ndarray            # int64 [h, N]: original index of the chosen dst, -1 on dst tokens
    score: np.ndarray           # fp64 [h, N]: cosine with that dst, nan on dst tokens
    merged: np.ndarray          # bool [h, N]: source merged into its best dst
    slot: np.ndarray            # int64 [h, N]: regular slot (group) of each token
    n_slots: int                # regular slots per head (the same for every head)
    block_slot_base: list = field(default_factory=list)


def plan_tensor(X: np.ndarray, blocks: list[np.ndarray], stride: int, pct: int,
                uniform: bool = False) -> TensorPlan:
    """Match + top-r for one tensor, per head and per block (key designs 1-2).

    ``uniform`` is the head-uniform baseline the note argues against: one plan
    per block from the mean over heads of the per-head cosine matrices, used
    by every head.
    """
    h, N, _ = X.shape
    is_dst = np.zeros(N, dtype=bool)
    best = np.full((h, N), -1, dtype=np.int64)
    score = np.full((h, N), np.nan)
    merged = np.zeros((h, N), dtype=bool)
    slot = np.empty((h, N), dtype=np.int64)
    base = 0
    bases = []
    for toks in blocks:
        n_b = toks.shape[0]
        dst_i, src_i = split_dst_src(n_b, stride)
        is_dst[toks[dst_i]] = True
        r_b = merge_count(n_b, pct)
        if uniform:
            sims = [cosine_similarity(X[hh, toks[src_i]], X[hh, toks[dst_i]]) for hh in range(h)]
            sim_bar = np.mean(sims, axis=0)
            b_all, s_all = best_match(sim_bar)
            m_all = select_top_r(s_all, r_b)
        for hh in range(h):
            if uniform:
                b, s, m = b_all, s_all, m_all
            else:
                sim = cosine_similarity(X[hh, toks[src_i]], X[hh, toks[dst_i]])
                b, s = best_match(sim)
                m = select_top_r(s, r_b)
            sl, n_slots_b = block_slots(n_b, dst_i, src_i, b, m)
            best[hh, toks[src_i]] = toks[dst_i[b]]
            score[hh, toks[src_i]] = s
            merged[hh, toks[src_i]] = m
            slot[hh, toks] = base + sl
        bases.append(base)
        base += n_slots_b
    return TensorPlan(is_dst, best, score, merged, slot, base, bases)


def plan_from_choice(blocks: list[np.ndarray], stride: int, best: np.ndarray,
                     merged: np.ndarray) -> TensorPlan:
    """Rebuild the slots of a plan given per-token (best dst, merged) arrays
    [h, N] in original order, e.g. a plan written by hand in a test."""
    h, N = best.shape
    is_dst = np.zeros(N, dtype=bool)
    slot = np.empty((h, N), dtype=np.int64)
    base = 0
    bases = []
    for toks in blocks:
        n_b = toks.shape[0]
        dst_i, src_i = split_dst_src(n_b, stride)
        is_dst[toks[dst_i]] = True
        pos_of = {int(t): k for k, t in enumerate(toks[dst_i])}
        for hh in range(h):
            b = np.array([pos_of[int(t)] for t in best[hh, toks[src_i]]], dtype=np.int64)
            sl, n_slots_b = block_slots(n_b, dst_i, src_i, b, merged[hh, toks[src_i]])
            slot[hh, toks] = base + sl
        bases.append(base)
        base += n_slots_b
    score = np.full((h, N), np.nan)
    return TensorPlan(is_dst, best.copy(), score, merged.copy(), slot, base, bases)


# --------------------------------------------------------------------------
# Merging (mean of members), deviation, outlier filter (key designs 1 and 3)
# --------------------------------------------------------------------------

def group_sums(X: np.ndarray, slot: np.ndarray, n_slots: int) -> tuple[np.ndarray, np.ndarray]:
    """Per head: sum of member rows and member count of every slot."""
    h, N, d = X.shape
    sums = np.zeros((h, n_slots, d))
    counts = np.zeros((h, n_slots), dtype=np.int64)
    for hh in range(h):
        np.add.at(sums[hh], slot[hh], X[hh])
        np.add.at(counts[hh], slot[hh], 1)
    return sums, counts


def group_means(X: np.ndarray, slot: np.ndarray, n_slots: int) -> np.ndarray:
    """A merged token is the mean of its members (key design 1)."""
    sums, counts = group_sums(X, slot, n_slots)
    return sums / counts[..., None]


def query_deviation(Q: np.ndarray, slot: np.ndarray, means: np.ndarray,
                    counts: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """dev(h, n) = || q_n - q~_{slot(n)} ||_2 for members of groups of >= 2
    tokens, 0 for singletons (key design 3).  Returns (dev, eligible)."""
    h, N, _ = Q.shape
    dev = np.zeros((h, N))
    eligible = np.zeros((h, N), dtype=bool)
    for hh in range(h):
        diff = Q[hh] - means[hh, slot[hh]]
        eligible[hh] = counts[hh, slot[hh]] >= 2
        dev[hh] = np.where(eligible[hh], np.sqrt((diff * diff).sum(axis=1)), 0.0)
    return dev, eligible


def outlier_count(h: int, N: int, pct: int, n_eligible: int) -> int:
    """k_o = min(floor(pct * h * N / 100), number of eligible queries)."""
    return min((pct * h * N) // 100, n_eligible)


def select_outliers(dev: np.ndarray, eligible: np.ndarray, pct: int) -> np.ndarray:
    """M_o: the global top-d% of deviations over all heads (key design 3),
    ordered by (dev desc, flat index h*N + n asc) among eligible queries."""
    h, N = dev.shape
    flat_dev = dev.reshape(-1)
    cand = np.nonzero(eligible.reshape(-1))[0]
    k = outlier_count(h, N, pct, cand.shape[0])
    order = np.lexsort((cand, -flat_dev[cand]))
    mask = np.zeros(h * N, dtype=bool)
    mask[cand[order[:k]]] = True
    return mask.reshape(h, N)


@dataclass
class QueryRestore:
    means: np.ndarray        # [h, n_slots, d] regular slots after removing outliers
    live: np.ndarray         # bool [h, n_slots]: False for drained slots
    slot_final: np.ndarray   # int64 [h, N]: regular slot, or n_slots + rank for an outlier
    n_out: np.ndarray        # int64 [h]: outliers per head
    q_tilde: list            # per head: [n_slots + n_out[h], d] (drained rows are nan)


def restore_outliers(Q: np.ndarray, slot: np.ndarray, n_slots: int,
                     mask: np.ndarray) -> QueryRestore:
    """Subtract every outlier from its merged token and keep it as a token of
    its own: q~ <- (sum_G q - sum_{O_g} q) / (|G| - |O_g|) (key design 3).
    Outlier slots follow the regular ones, per head, in ascending n."""
    h, N, d = Q.shape
    sums, counts = group_sums(Q, slot, n_slots)
    out_sums = np.zeros_like(sums)
    out_counts = np.zeros_like(counts)
    for hh in range(h):
        o = np.nonzero(mask[hh])[0]
        np.add.at(out_sums[hh], slot[hh, o], Q[hh, o])
        np.add.at(out_counts[hh], slot[hh, o], 1)
    remain = counts - out_counts
    live = remain > 0
    means = np.full_like(sums, np.nan)
    means[live] = (sums[live] - out_sums[live]) / remain[live][:, None]
    slot_final = slot.copy()
    n_out = mask.sum(axis=1)
    q_tilde = []
    for hh in range(h):
        o = np.nonzero(mask[hh])[0]          # ascending n
        slot_final[hh, o] = n_slots + np.arange(o.shape[0])
        q_tilde.append(np.concatenate([means[hh], Q[hh, o]], axis=0))
    return QueryRestore(means, live, slot_final, n_out, q_tilde)


# --------------------------------------------------------------------------
# Attention on the shortened sequences, and unmerge
# --------------------------------------------------------------------------

def attention(Qt: np.ndarray, Kt: np.ndarray, Vt: np.ndarray, scale: float,
              chunk: int = 1024) -> np.ndarray:
    """softmax(Qt Kt^T * scale) Vt for one head, fp64, max-subtracted."""
    out = np.empty((Qt.shape[0], Vt.shape[1]))
    for s in range(0, Qt.shape[0], chunk):
        z = (Qt[s:s + chunk] @ Kt.T) * scale
        z -= z.max(axis=1, keepdims=True)
        p = np.exp(z)
        out[s:s + chunk] = (p @ Vt) / p.sum(axis=1, keepdims=True)
    return out


def unmerge(O_slots: list, slot_final: np.ndarray) -> np.ndarray:
    """out[h, n] = Õ[h, slot(h, n)]: the merged token's output is copied back
    to each member, which also undoes the reorder (key designs 1-2)."""
    h, N = slot_final.shape
    d = O_slots[0].shape[1]
    out = np.empty((h, N, d))
    for hh in range(h):
        out[hh] = O_slots[hh][slot_final[hh]]
    return out


# --------------------------------------------------------------------------
# The whole layer
# --------------------------------------------------------------------------

@dataclass
class OracleResult:
    out: np.ndarray | None
    q_plan: TensorPlan | None = None
    k_plan: TensorPlan | None = None
    q_means: np.ndarray | None = None       # initial means (before the filter)
    q_counts: np.ndarray | None = None
    k_means: np.ndarray | None = None
    v_means: np.ndarray | None = None
    dev: np.ndarray | None = None
    eligible: np.ndarray | None = None
    mask: np.ndarray | None = None
    restore: QueryRestore | None = None
    o_slots: list | None = None


def forward_plan(cfg: OracleConfig, Q: np.ndarray, K: np.ndarray, V: np.ndarray,
                 q_plan: TensorPlan | None = None, k_plan: TensorPlan | None = None,
                 mask: np.ndarray | None = None) -> OracleResult:
    """Every step before attention.  A plan or outlier mask passed in replaces
    the one the oracle would compute (used to check later steps in isolation)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    blocks = block_list(cfg)
    uniform = cfg.mode == HEAD_UNIFORM
    if q_plan is None:
        q_plan = plan_tensor(Q, blocks, cfg.q_stride, cfg.q_pct, uniform)
    if k_plan is None:
        k_plan = plan_tensor(K, blocks, cfg.kv_stride, cfg.kv_pct, uniform)
    q_sums, q_counts = group_sums(Q, q_plan.slot, q_plan.n_slots)
    q_means = q_sums / q_counts[..., None]
    k_means = group_means(K, k_plan.slot, k_plan.n_slots)
    v_means = group_means(V, k_plan.slot, k_plan.n_slots)   # V follows K's plan
    dev, eligible = query_deviation(Q, q_plan.slot, q_means, q_counts)
    if mask is None:
        mask = select_outliers(dev, eligible, cfg.out_pct)
    rest = restore_outliers(Q, q_plan.slot, q_plan.n_slots, mask)
    return OracleResult(None, q_plan, k_plan, q_means, q_counts, k_means, v_means,
                        dev, eligible, mask, rest)


def forward(cfg: OracleConfig, Q: np.ndarray, K: np.ndarray, V: np.ndarray,
            **override) -> OracleResult:
    """The merged global-attention layer: merge -> filter -> attention ->
    unmerge (overall framework of the HTTM note).  DENSE runs plain attention."""
    scale = cfg.softmax_scale
    if cfg.mode == DENSE:
        Q = np.asarray(Q, dtype=np.float64)
        K = np.asarray(K, dtype=np.float64)
        V = np.asarray(V, dtype=np.float64)
        out = np.stack([attention(Q[hh], K[hh], V[hh], scale) for hh in range(Q.shape[0])])
        return OracleResult(out)
    res = forward_plan(cfg, Q, K, V, **override)
    o_slots = []
    for hh in range(Q.shape[0]):
        qt = res.restore.q_tilde[hh]
        o = np.full((qt.shape[0], qt.shape[1]), np.nan)
        live = np.concatenate([res.restore.live[hh], np.ones(res.restore.n_out[hh], dtype=bool)])
        o[live] = attention(qt[live], res.k_means[hh], res.v_means[hh], scale)
        o_slots.append(o)
    res.o_slots = o_slots
    res.out = unmerge(o_slots, res.restore.slot_final)
    return res
