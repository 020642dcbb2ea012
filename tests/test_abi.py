"""The C ABI library loads on the CPU, exports every symbol include/httm.h
declares, and its host-side planner validates configurations and sizes the
layout as the oracle's block table does (no device call is made here)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import oracle.httm_oracle as O
from token_merging_view_b200 import binding as B
from token_merging_view_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "httm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(httm_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = B.load_library()
    declared = _declared()
    assert set(declared) == set(B.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings():
    lib = B.load_library()
    for s in range(10):
        assert lib.httm_status_str(s).decode()
    assert lib.httm_status_str(99).decode() == "unknown status"


def _plan_status(**kw):
    lib = B.load_library()
    cfg = B.LayerConfig(**{**dict(h=2, T=4, P=64, d_head=16, n_s=16, n_t=4, q_dst_stride=4, kv_dst_stride=4,
                                   q_merge_pct=50, kv_merge_pct=25, outlier_pct=10), **kw}).to_c()
    h = ctypes.c_void_p()
    st = lib.httm_plan(ctypes.byref(cfg), ctypes.byref(h))
    if st == 0:
        lib.httm_plan_destroy(h)
    return st


def test_plan_validation():
    assert _plan_status() == 0
    assert _plan_status(h=0) == 1                     # HTTM_ERR_ARG
    assert _plan_status(h=65) == 1
    assert _plan_status(d_head=32) == 2               # HTTM_ERR_UNSUPPORTED
    assert _plan_status(mode=7) == 1
    assert _plan_status(q_dst_stride=1) == 1
    assert _plan_status(outlier_pct=101) == 1
    assert _plan_status(q_merge_pct=80) == 3          # r_b = 51 > 48 sources: infeasible
    assert _plan_status(T=400, n_t=400, n_s=64) == 2  # a block of 25,600 tokens
    assert _plan_status(softmax_scale=-1.0) == 1
    lib = B.load_library()
    assert lib.httm_plan(None, None) == 1
    assert lib.httm_forward(None, None, None, None, None, None, 0, None) == 1


def _oracle_cfg(w):
    return O.OracleConfig(h=w.h, T=w.T, P=w.P, d=w.d, n_s=w.n_s, n_t=w.n_t, q_stride=w.q_stride,
                          kv_stride=w.kv_stride, q_pct=w.q_pct, kv_pct=w.kv_pct, out_pct=w.out_pct, mode=w.mode,
                          contig_block=w.contig_block)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_plan_sizes_match_oracle_block_table(name):
    w = WORKLOADS[name]
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    ocfg = _oracle_cfg(w)
    blocks = O.block_list(ocfg)
    q_slots = sum(b.shape[0] - O.merge_count(b.shape[0], w.q_pct) for b in blocks)
    kv_slots = sum(b.shape[0] - O.merge_count(b.shape[0], w.kv_pct) for b in blocks)
    assert plan.info.N == w.N
    assert plan.info.n_blocks == len(blocks)
    assert plan.info.q_slots == q_slots
    assert plan.info.kv_slots == kv_slots
    assert plan.info.k_out_max == w.out_pct * w.h * w.N // 100
    assert plan.workspace_bytes > 0


def test_contiguous_and_uniform_plans():
    w = WORKLOADS["vggt_30f"]
    for mode in (B.HTTM_CONTIGUOUS, B.HTTM_HEAD_UNIFORM):
        plan = B.httm_plan(B.LayerConfig.from_workload(w, mode=mode))
        blocks = O.block_list(_oracle_cfg(w.with_(mode=mode)))
        assert plan.info.n_blocks == len(blocks)
        assert plan.info.q_slots == sum(b.shape[0] - O.merge_count(b.shape[0], w.q_pct) for b in blocks)


def test_head_shard_plan_sizes_and_errors():
    """A shard of a head-sharded layer keeps its own heads' plan but the
    whole layer's outlier budget (the filter is global across heads)."""
    w = WORKLOADS["vggt_30f"]
    full = B.httm_plan(B.LayerConfig.from_workload(w))
    half = B.httm_plan(B.LayerConfig.from_workload(w, h=w.h // 2))
    k_half = half.info.k_out_max
    half.shard(1, 2)
    assert half.info.k_out_max == w.out_pct * w.h * w.N // 100 == full.info.k_out_max
    assert half.info.k_out_max > k_half
    assert half.info.q_slots == full.info.q_slots and half.info.kv_slots == full.info.kv_slots
    assert half.info.q_rows_alloc >= half.info.k_out_max
    lib = B.load_library()
    for shard, shards in ((2, 2), (-1, 2), (0, 0), (0, 65)):
        assert lib.httm_plan_shard(half.handle, shard, shards) == 1      # HTTM_ERR_ARG
    uni = B.httm_plan(B.LayerConfig.from_workload(w, h=w.h // 2, mode=B.HTTM_HEAD_UNIFORM))
    assert lib.httm_plan_shard(uni.handle, 0, 2) == 2                     # HTTM_ERR_UNSUPPORTED
    assert lib.httm_plan_shard(uni.handle, 0, 1) == 0
    # a sharded plan runs only through httm_forward_sharded, with a collective;
    # both are host checks made before any device call
    fake = ctypes.c_void_p(1 << 20)
    assert lib.httm_forward(half.handle, fake, fake, fake, fake, fake, 1 << 40, None) == 1
    assert lib.httm_forward_reuse(half.handle, fake, fake, fake, fake, fake, 1 << 40, None) == 1
    assert lib.httm_forward_sharded(half.handle, fake, fake, fake, fake, fake, 1 << 40, None, None, None) == 1
    null_fn = B.httm_exchange()
    assert lib.httm_forward_sharded(half.handle, fake, fake, fake, fake, fake, 1 << 40,
                                    ctypes.byref(null_fn), None, None) == 1


def test_binding_rejects_bad_tensors_before_any_device_call():
    """The binding only marshals: host tensors, a wrong dtype or a strided
    view are refused in Python, so no pointer of the wrong kind reaches the
    library (which would treat it as device memory)."""
    import torch
    w = WORKLOADS["tiny_4f_8x8"]
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    shape = (w.h, w.N, w.d)
    Q = torch.zeros(shape, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.httm_forward(plan, Q, Q, Q, out=torch.empty_like(Q), workspace=torch.empty(plan.workspace_bytes,
                                                                                      dtype=torch.uint8))
    with pytest.raises(ValueError, match="contiguous"):
        B.httm_forward(plan, Q.to(torch.bfloat16), Q, Q)
    with pytest.raises(ValueError, match="contiguous"):
        B.httm_forward(plan, Q.transpose(1, 2).contiguous().transpose(1, 2), Q, Q)


def test_noalloc_binding_rejects_bad_buffers_before_the_call():
    """httm_select_outliers_noalloc writes h * N mask bytes and h int32
    counts and reads dev / eligible as dense [h, N] arrays: a buffer of the
    wrong dtype, shape, layout or device is refused in Python, before any
    pointer reaches the library."""
    import torch
    h, N = 3, 40
    dev = torch.zeros((h, N), dtype=torch.float32)
    elig = torch.zeros((h, N), dtype=torch.uint8)
    with pytest.raises(ValueError, match="mask"):
        B.httm_select_outliers_noalloc(dev, elig, 10, mask=torch.zeros((h, N - 1), dtype=torch.uint8))
    with pytest.raises(ValueError, match="mask"):
        B.httm_select_outliers_noalloc(dev, elig, 10, mask=torch.zeros((h, N), dtype=torch.int32))
    with pytest.raises(ValueError, match="n_out"):
        B.httm_select_outliers_noalloc(dev, elig, 10, n_out=torch.zeros((h,), dtype=torch.int64))
    with pytest.raises(ValueError, match="n_out"):
        B.httm_select_outliers_noalloc(dev, elig, 10, n_out=torch.zeros((h + 1,), dtype=torch.int32))
    with pytest.raises(ValueError, match="dev must be contiguous"):
        B.httm_select_outliers_noalloc(torch.zeros((N, h), dtype=torch.float32).t(), elig, 10)
    with pytest.raises(ValueError, match="eligible must be contiguous"):
        B.httm_select_outliers_noalloc(dev, torch.zeros((N, h), dtype=torch.uint8).t(), 10)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.httm_select_outliers_noalloc(dev, elig, 10)
    with pytest.raises(ValueError, match="float32"):
        B.httm_select_outliers_noalloc(dev.reshape(-1), elig, 10)


def test_partition_plan_host_checks():
    """HTTM_PARTITION: bf16 with d_head = 64 only; a plan that has not been
    partitioned refuses forward calls and sharding; the partition call
    refuses other modes (host checks, no device call)."""
    import ctypes
    w = WORKLOADS["tiny_4f_8x8"]
    with pytest.raises(B.HttmError) as e:
        B.httm_plan(B.LayerConfig.from_workload(w, mode=B.HTTM_PARTITION))      # fp32, d_head 16
    assert e.value.status == 2
    cfg = B.LayerConfig(h=2, T=3, P=64, d_head=64, mode=B.HTTM_PARTITION, n_s=16, n_t=2,
                        q_dst_stride=0, kv_dst_stride=0, q_merge_pct=-1, kv_merge_pct=-1)   # ignored in this mode
    plan = B.httm_plan(cfg)
    lib = B.load_library()
    fake = ctypes.c_void_p(1 << 20)
    assert lib.httm_forward(plan.handle, fake, fake, fake, fake, fake, 1 << 40, None) == 1
    assert lib.httm_plan_shard(plan.handle, 0, 2) == 2
    other = B.httm_plan(B.LayerConfig.from_workload(WORKLOADS["vggt_30f"]))
    assert lib.httm_plan_partition(other.handle, fake, 10, None, None) == 1
    assert lib.httm_plan_partition(plan.handle, None, 10, None, None) == 1
    assert lib.httm_plan_partition(plan.handle, fake, 101, None, None) == 1
    bad = B.httm_plan(B.LayerConfig(h=2, T=3, P=60, d_head=64, mode=B.HTTM_PARTITION, n_s=16, n_t=2))
    assert lib.httm_plan_partition(bad.handle, fake, 10, None, None) == 1       # 60 patches: not a square grid
