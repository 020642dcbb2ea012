"""Named workloads: a VGGT-shaped global-attention layer at several lengths.

A VGGT global-attention layer sees T frames x P patch tokens (a 37 x 37 patch
grid, P = 1369) with 16 heads of 64 channels.  HTTM's published setting is
n_s = 128 spatial tokens x n_t = 30 frames per merge block, queries merged
hard and then partly restored by the outlier filter, keys/values merged less
("HTTM: Head-wise Temporal Token Merging for Faster VGGT", training-strategy
section and key designs 2-3).  Each workload here fixes every knob, plus the
seeded generator settings of :mod:`token_merging_view_b200.inputs`.

Modes: 0 = head-wise temporal (HTTM), 1 = head-uniform (one plan per block
from the head-mean cosine), 2 = contiguous blocks in the original order,
3 = dense (no merging), 4 = HTTM blocks with LiteVGGT's destination rule.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

HEADWISE_TEMPORAL = 0
HEAD_UNIFORM = 1
CONTIGUOUS = 2
DENSE = 3
PARTITION = 4


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    grid: int
    h: int
    d: int
    fp32: bool
    n_s: int
    n_t: int
    q_stride: int
    kv_stride: int
    q_pct: int
    kv_pct: int
    out_pct: int
    seed: int
    noise_sigma: float
    max_shift: int
    mode: int = HEADWISE_TEMPORAL
    contig_block: int = 3840

    @property
    def P(self) -> int:
        return self.grid * self.grid

    @property
    def N(self) -> int:
        return self.T * self.P

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # 4 frames of an 8x8 grid, 2 heads x 16, fp32: small enough for pure loops.
    "tiny_4f_8x8": Workload("tiny_4f_8x8", T=4, grid=8, h=2, d=16, fp32=True, n_s=16, n_t=4,
                            q_stride=4, kv_stride=4, q_pct=50, kv_pct=25, out_pct=10,
                            seed=0, noise_sigma=0.3, max_shift=0),
    # 30 frames x 1369 tokens = 41,070 tokens; 11 blocks per head (10 x 3840 + 1 x 2670).
    "vggt_30f": Workload("vggt_30f", T=30, grid=37, h=16, d=64, fp32=False, n_s=128, n_t=30,
                         q_stride=4, kv_stride=4, q_pct=70, kv_pct=50, out_pct=10,
                         seed=1, noise_sigma=0.3, max_shift=2),
    # 100 frames = 136,900 tokens: temporal groups of 30, 30, 30, 10.
    "vggt_100f": Workload("vggt_100f", T=100, grid=37, h=16, d=64, fp32=False, n_s=128, n_t=30,
                          q_stride=4, kv_stride=4, q_pct=70, kv_pct=50, out_pct=10,
                          seed=2, noise_sigma=0.3, max_shift=2),
    # 500 frames = 684,500 tokens; aggressive queries (dst every 8th, 85% merged).
    "vggt_500f": Workload("vggt_500f", T=500, grid=37, h=16, d=64, fp32=False, n_s=128, n_t=30,
                          q_stride=8, kv_stride=4, q_pct=85, kv_pct=60, out_pct=10,
                          seed=3, noise_sigma=0.5, max_shift=2),
    # 1000 frames = 1,369,000 tokens (sweep point Q r70 / d10).
    "vggt_1000f": Workload("vggt_1000f", T=1000, grid=37, h=16, d=64, fp32=False, n_s=128, n_t=30,
                           q_stride=4, kv_stride=4, q_pct=70, kv_pct=50, out_pct=10,
                           seed=4, noise_sigma=0.3, max_shift=2),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]
