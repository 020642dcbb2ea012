"""Thin ctypes binding of the C ABI in ``include/httm.h``.

Only argument marshalling happens here: torch tensors become raw device
pointers and sizes, and a non-OK status becomes an exception.  Every step of
the layer runs in the CUDA library; if ``libhttm.so`` is missing or cannot be
loaded, every call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from .workloads import Workload

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhttm.so")

HTTM_BF16, HTTM_F32 = 0, 1
HTTM_HEADWISE_TEMPORAL, HTTM_HEAD_UNIFORM, HTTM_CONTIGUOUS, HTTM_DENSE, HTTM_PARTITION = 0, 1, 2, 3, 4
HTTM_DEV_BAD_PLAN, HTTM_DEV_BOUNDS, HTTM_DEV_TIMEOUT = 0x1, 0x2, 0x4

# every symbol include/httm.h declares
EXPORTS = (
    "httm_plan", "httm_plan_destroy", "httm_get_plan_info", "httm_workspace_bytes",
    "httm_forward", "httm_forward_debug", "httm_forward_with_plan", "httm_forward_reuse", "httm_reorder",
    "httm_get_device_status", "httm_forward_launches", "httm_profile_enable", "httm_profile_read",
    "httm_select_outliers_noalloc", "httm_set_wait_budget", "httm_status_str",
    "httm_plan_shard", "httm_forward_sharded", "httm_last_cuda_error", "httm_set_fused_unmerge",
    "httm_plan_partition",
)
STAGES = ("match", "merge", "outlier", "attention", "unmerge", "other")


class httm_cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "h", "T", "P", "d_head", "dtype", "mode", "n_s", "n_t", "contig_block",
        "q_dst_stride", "kv_dst_stride", "q_merge_pct", "kv_merge_pct", "outlier_pct")] + \
        [("softmax_scale", ctypes.c_float)]


class httm_plan_info(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("n_blocks", ctypes.c_int32), ("q_slots", ctypes.c_int32),
                ("kv_slots", ctypes.c_int32), ("k_out_max", ctypes.c_int64),
                ("q_rows_alloc", ctypes.c_int64), ("ws_q_tilde", ctypes.c_int64),
                ("ws_k_tilde", ctypes.c_int64), ("ws_v_tilde", ctypes.c_int64),
                ("ws_o_tilde", ctypes.c_int64), ("ws_n_out", ctypes.c_int64),
                ("ws_out_base", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64)]


_DEBUG_FIELDS = ("q_best", "q_score", "q_merged", "k_best", "k_score", "k_merged", "q_slot", "k_slot",
                 "dev", "outlier", "q_means", "q_restored", "k_means", "v_means")


class httm_debug(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _DEBUG_FIELDS]


class httm_merge_plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q_best", "q_merged", "k_best", "k_merged", "outlier")]


# int32_t (*allreduce_sum)(void* buf, int64_t count, int32_t elem_bytes, void* stream, void* user)
EXCHANGE_FN = ctypes.CFUNCTYPE(ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p,
                               ctypes.c_void_p)


class httm_exchange(ctypes.Structure):
    _fields_ = [("allreduce_sum", EXCHANGE_FN), ("user", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libhttm.so (once) and declare the signatures.  Raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run python -m token_merging_view_b200.build)")
    lib = ctypes.CDLL(path)
    P, V, S, I, U = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint32
    lib.httm_plan.argtypes = [ctypes.POINTER(httm_cfg), ctypes.POINTER(ctypes.c_void_p)]
    lib.httm_plan_destroy.argtypes = [P]
    lib.httm_plan_destroy.restype = None
    lib.httm_get_plan_info.argtypes = [P, ctypes.POINTER(httm_plan_info)]
    lib.httm_workspace_bytes.argtypes = [P]
    lib.httm_workspace_bytes.restype = S
    lib.httm_forward.argtypes = [P, V, V, V, V, V, S, V]
    lib.httm_forward_debug.argtypes = [P, V, V, V, V, V, S, ctypes.POINTER(httm_debug), V]
    lib.httm_forward_with_plan.argtypes = [P, V, V, V, V, V, S, ctypes.POINTER(httm_merge_plan),
                                           ctypes.POINTER(httm_debug), V]
    lib.httm_forward_reuse.argtypes = [P, V, V, V, V, V, S, V]
    lib.httm_reorder.argtypes = [P, V, V, I, V]
    lib.httm_get_device_status.argtypes = [P, V, V, ctypes.POINTER(U)]
    lib.httm_forward_launches.argtypes = [P]
    lib.httm_forward_launches.restype = ctypes.c_int32
    lib.httm_profile_enable.argtypes = [P, I]
    lib.httm_profile_read.argtypes = [P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32)]
    lib.httm_select_outliers_noalloc.argtypes = [V, V, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, V, V, V]
    lib.httm_select_outliers_noalloc.restype = ctypes.c_int
    lib.httm_set_wait_budget.argtypes = [P, ctypes.c_uint64]
    lib.httm_set_wait_budget.restype = ctypes.c_int
    lib.httm_set_fused_unmerge.argtypes = [P, I]
    lib.httm_set_fused_unmerge.restype = ctypes.c_int
    lib.httm_plan_partition.argtypes = [P, V, ctypes.c_int32, V, V]
    lib.httm_plan_partition.restype = ctypes.c_int
    lib.httm_plan_shard.argtypes = [P, ctypes.c_int32, ctypes.c_int32]
    lib.httm_forward_sharded.argtypes = [P, V, V, V, V, V, S, ctypes.POINTER(httm_exchange),
                                         ctypes.POINTER(httm_debug), V]
    lib.httm_status_str.argtypes = [I]
    lib.httm_status_str.restype = ctypes.c_char_p
    lib.httm_last_cuda_error.argtypes = []
    lib.httm_last_cuda_error.restype = ctypes.c_char_p
    for name in ("httm_plan", "httm_get_plan_info", "httm_forward", "httm_forward_debug",
                 "httm_forward_with_plan", "httm_forward_reuse", "httm_reorder", "httm_get_device_status",
                 "httm_profile_enable", "httm_profile_read", "httm_plan_shard", "httm_forward_sharded"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


class HttmError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load_library()
        msg = lib.httm_status_str(status).decode()
        if status == 6:                                   # HTTM_ERR_CUDA: which call, which error
            detail = lib.httm_last_cuda_error().decode()
            if detail:
                msg += f" [{detail}]"
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != 0:
        raise HttmError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class LayerConfig:
    h: int
    T: int
    P: int
    d_head: int
    fp32: bool = False
    mode: int = HTTM_HEADWISE_TEMPORAL
    n_s: int = 128
    n_t: int = 30
    contig_block: int = 3840
    q_dst_stride: int = 4
    kv_dst_stride: int = 4
    q_merge_pct: int = 70
    kv_merge_pct: int = 50
    outlier_pct: int = 10
    softmax_scale: float = 0.0

    @classmethod
    def from_workload(cls, w: Workload, **kw) -> "LayerConfig":
        base = dict(h=w.h, T=w.T, P=w.P, d_head=w.d, fp32=w.fp32, mode=w.mode, n_s=w.n_s, n_t=w.n_t,
                    contig_block=w.contig_block, q_dst_stride=w.q_stride, kv_dst_stride=w.kv_stride,
                    q_merge_pct=w.q_pct, kv_merge_pct=w.kv_pct, outlier_pct=w.out_pct)
        base.update(kw)
        return cls(**base)

    def to_c(self) -> httm_cfg:
        return httm_cfg(self.h, self.T, self.P, self.d_head, HTTM_F32 if self.fp32 else HTTM_BF16, self.mode,
                        self.n_s, self.n_t, self.contig_block, self.q_dst_stride, self.kv_dst_stride,
                        self.q_merge_pct, self.kv_merge_pct, self.outlier_pct, self.softmax_scale)


class Plan:
    """Owns an ``httm_plan_t``; created by :func:`httm_plan`."""

    def __init__(self, cfg: LayerConfig):
        lib = load_library()
        self.cfg = cfg
        h = ctypes.c_void_p()
        c = cfg.to_c()
        _check(lib.httm_plan(ctypes.byref(c), ctypes.byref(h)), "httm_plan")
        self.handle = h
        info = httm_plan_info()
        _check(lib.httm_get_plan_info(h, ctypes.byref(info)), "httm_get_plan_info")
        self.info = info
        self.dtype = torch.float32 if cfg.fp32 else torch.bfloat16

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.httm_plan_destroy(self.handle)
            self.handle = None

    def shard(self, shard: int, shards: int) -> "Plan":
        """Make this plan (cfg.h heads) shard `shard` of `shards` of a
        head-sharded layer (httm_plan_shard); before its first forward."""
        lib = load_library()
        _check(lib.httm_plan_shard(self.handle, shard, shards), "httm_plan_shard")
        info = httm_plan_info()
        _check(lib.httm_get_plan_info(self.handle, ctypes.byref(info)), "httm_get_plan_info")
        self.info = info
        self.shard_index, self.shards = shard, shards
        return self

    @property
    def workspace_bytes(self) -> int:
        return int(load_library().httm_workspace_bytes(self.handle))

    def new_workspace(self, device=None) -> torch.Tensor:
        return torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device or "cuda")

    def launches(self) -> int:
        return int(load_library().httm_forward_launches(self.handle))

    def profile(self, enable: bool) -> None:
        _check(load_library().httm_profile_enable(self.handle, int(enable)), "httm_profile_enable")

    def profile_read(self) -> dict:
        """{stage: (milliseconds, launches)} accumulated since the last read."""
        ms = (ctypes.c_float * len(STAGES))()
        n = (ctypes.c_int32 * len(STAGES))()
        _check(load_library().httm_profile_read(self.handle, ms, n), "httm_profile_read")
        return {s: (float(ms[i]), int(n[i])) for i, s in enumerate(STAGES)}


def httm_plan(cfg: LayerConfig) -> Plan:
    return Plan(cfg)


def _prep(plan: Plan, Q, K, V, out, workspace):
    for t in (Q, K, V):
        if t.dtype != plan.dtype or not t.is_contiguous():
            raise ValueError(f"inputs must be contiguous {plan.dtype}")
    if out is None:
        out = torch.empty_like(Q)
    if workspace is None:
        workspace = plan.new_workspace(Q.device)
    return out, workspace


def httm_forward(plan: Plan, Q, K, V, out=None, workspace=None, stream=None):
    out, workspace = _prep(plan, Q, K, V, out, workspace)
    _check(load_library().httm_forward(plan.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(out), _ptr(workspace),
                                       workspace.numel(), _stream(stream)), "httm_forward")
    return out


def _debug_struct(dbg: dict | None) -> httm_debug:
    d = httm_debug()
    for k, v in (dbg or {}).items():
        setattr(d, k, v.data_ptr() if v is not None else None)
    return d


def debug_buffers(plan: Plan, device="cuda") -> dict:
    """Allocate every debug export of :class:`httm_debug` for one forward."""
    h, N, d = plan.cfg.h, plan.info.N, plan.cfg.d_head
    qs, ks = plan.info.q_slots, plan.info.kv_slots
    i32, f32, u8 = torch.int32, torch.float32, torch.uint8
    e = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)
    return dict(q_best=e((h, N), i32), q_score=e((h, N), f32), q_merged=e((h, N), u8),
                k_best=e((h, N), i32), k_score=e((h, N), f32), k_merged=e((h, N), u8),
                q_slot=e((h, N), i32), k_slot=e((h, N), i32), dev=e((h, N), f32), outlier=e((h, N), u8),
                q_means=e((h, qs, d), f32), q_restored=e((h, qs, d), f32),
                k_means=e((h, ks, d), f32), v_means=e((h, ks, d), f32))


def httm_forward_debug(plan: Plan, Q, K, V, dbg: dict, out=None, workspace=None, stream=None):
    out, workspace = _prep(plan, Q, K, V, out, workspace)
    d = _debug_struct(dbg)
    _check(load_library().httm_forward_debug(plan.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(out),
                                             _ptr(workspace), workspace.numel(), ctypes.byref(d),
                                             _stream(stream)), "httm_forward_debug")
    return out


def httm_forward_with_plan(plan: Plan, Q, K, V, injected: dict, dbg: dict | None = None, out=None,
                           workspace=None, stream=None):
    """``injected``: dict with q_best/q_merged/k_best/k_merged ([h, N] int32 /
    uint8 CUDA tensors) and/or outlier ([h, N] uint8)."""
    out, workspace = _prep(plan, Q, K, V, out, workspace)
    mp = httm_merge_plan()
    for k, v in injected.items():
        setattr(mp, k, v.data_ptr() if v is not None else None)
    d = _debug_struct(dbg)
    _check(load_library().httm_forward_with_plan(plan.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(out),
                                                 _ptr(workspace), workspace.numel(), ctypes.byref(mp),
                                                 ctypes.byref(d) if dbg else None, _stream(stream)),
           "httm_forward_with_plan")
    return out


def httm_forward_reuse(plan: Plan, Q, K, V, out=None, workspace=None, stream=None):
    """The layer on new Q/K/V with the merge indices (both plans' member lists)
    that the last full forward on ``plan`` left in ``workspace``; matching and
    top-r selection are skipped (cached merge indices, LiteVGGT note, key
    design 3).  ``workspace`` must be the one that forward used."""
    if workspace is None:
        raise ValueError("httm_forward_reuse needs the workspace of an earlier forward")
    out, workspace = _prep(plan, Q, K, V, out, workspace)
    _check(load_library().httm_forward_reuse(plan.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(out),
                                             _ptr(workspace), workspace.numel(), _stream(stream)),
           "httm_forward_reuse")
    return out


def httm_reorder(plan: Plan, X, inverse: bool = False, out=None, stream=None):
    out = torch.empty_like(X) if out is None else out
    _check(load_library().httm_reorder(plan.handle, _ptr(X), _ptr(out), int(inverse), _stream(stream)),
           "httm_reorder")
    return out


def httm_set_wait_budget(plan: Plan, nanoseconds: int) -> None:
    """Bound of every device-side wait of later forward calls on ``plan``
    (default 2e9 ns); 0 makes every wait that is not already complete run
    out (HTTM_DEV_TIMEOUT), for checking the failure path."""
    _check(load_library().httm_set_wait_budget(plan.handle, int(nanoseconds)), "httm_set_wait_budget")


def httm_plan_partition(plan: Plan, score, ga_pct: int = 10, roles_out=None, stream=None):
    """LiteVGGT's token partition as the destination rule of an
    HTTM_PARTITION plan: ``score`` is a [T, P] float32 CUDA tensor (one
    geometric-importance score per token).  Synchronises the stream and
    resizes the plan (its workspace size changes).  Returns the token
    classes [T, P] uint8 (0 source, 1 destination, 2 GA)."""
    T, P = plan.cfg.T, plan.cfg.P
    if score.dtype != torch.float32 or tuple(score.shape) != (T, P) or not score.is_contiguous():
        raise ValueError(f"score must be a contiguous float32 [{T}, {P}] tensor")
    if roles_out is None:
        roles_out = torch.empty((T, P), dtype=torch.uint8, device=score.device)
    if roles_out.dtype != torch.uint8 or tuple(roles_out.shape) != (T, P) or not roles_out.is_contiguous():
        raise ValueError(f"roles_out must be a contiguous uint8 [{T}, {P}] tensor")
    lib = load_library()
    _check(lib.httm_plan_partition(plan.handle, _ptr(score), int(ga_pct), _ptr(roles_out), _stream(stream)),
           "httm_plan_partition")
    info = httm_plan_info()
    _check(lib.httm_get_plan_info(plan.handle, ctypes.byref(info)), "httm_get_plan_info")
    plan.info = info
    return roles_out


def httm_set_fused_unmerge(plan: Plan, enable: bool) -> None:
    """Write attention output rows straight to their tokens from the
    attention epilogue (no separate unmerge launch) on later calls."""
    _check(load_library().httm_set_fused_unmerge(plan.handle, int(bool(enable))), "httm_set_fused_unmerge")


def httm_get_device_status(plan: Plan, workspace, stream=None) -> int:
    """Synchronises the stream; returns the device status bits (0 = clean)."""
    v = ctypes.c_uint32(0)
    st = load_library().httm_get_device_status(plan.handle, _ptr(workspace), _stream(stream), ctypes.byref(v))
    if st not in (0, 7, 8):
        _check(st, "httm_get_device_status")
    return int(v.value)


def workspace_view(plan: Plan, workspace, which: str):
    """A typed view of one shortened tensor inside the workspace ("q", "k",
    "v", "o" -> the Q~ / K~ / V~ / O~ rows) or of the per-head outlier counts
    ("n_out") and outlier row bases ("out_base")."""
    info, d = plan.info, plan.cfg.d_head
    es = 4 if plan.cfg.fp32 else 2
    if which in ("n_out", "out_base"):
        off = info.ws_n_out if which == "n_out" else info.ws_out_base
        return workspace[off:off + 4 * plan.cfg.h].view(torch.int32)
    if which in ("q", "o"):
        off = info.ws_q_tilde if which == "q" else info.ws_o_tilde
        rows = info.q_rows_alloc
    else:
        off = info.ws_k_tilde if which == "k" else info.ws_v_tilde
        rows = plan.cfg.h * info.kv_slots
    return workspace[off:off + rows * d * es].view(plan.dtype).view(rows, d)


def httm_select_outliers_noalloc(dev, eligible, outlier_pct: int, mask=None, n_out=None, stream=None):
    """Outlier selection that allocates no device memory inside the library
    (its scratch is a fixed array in the library).  dev: [h, N] fp32 CUDA
    tensor, eligible: [h, N] uint8.  Returns (mask [h, N] uint8, n_out [h]
    int32).  Calls that overlap on the GPU race (they share the scratch)."""
    if dev.dim() != 2:
        raise ValueError("dev must be float32 [h, N]")
    h, N = dev.shape
    if dev.dtype != torch.float32 or eligible.dtype != torch.uint8 or eligible.shape != dev.shape:
        raise ValueError("dev must be float32 [h, N] and eligible uint8 [h, N]")
    mask = torch.empty((h, N), dtype=torch.uint8, device=dev.device) if mask is None else mask
    n_out = torch.empty((h,), dtype=torch.int32, device=dev.device) if n_out is None else n_out
    # the kernels read and write these as dense arrays of exactly these sizes
    # on dev's device: anything else would be read in the wrong order or
    # written out of bounds
    if mask.dtype != torch.uint8 or tuple(mask.shape) != (h, N):
        raise ValueError("mask must be uint8 [h, N]")
    if n_out.dtype != torch.int32 or tuple(n_out.shape) != (h,):
        raise ValueError("n_out must be int32 [h]")
    bufs = (("dev", dev), ("eligible", eligible), ("mask", mask), ("n_out", n_out))
    for name, t in bufs:
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    for name, t in bufs:
        if not t.is_cuda or t.device != dev.device:
            raise ValueError(f"{name} must be a CUDA tensor on {dev.device}")
    _check(load_library().httm_select_outliers_noalloc(_ptr(dev), _ptr(eligible), h, N, outlier_pct, _ptr(mask),
                                                       _ptr(n_out), _stream(stream)),
           "httm_select_outliers_noalloc")
    return mask, n_out


def exchange_view(ws: torch.Tensor, buf, count: int, elem_bytes: int) -> torch.Tensor:
    """The int32 / int64 view of `ws` (a uint8 workspace tensor) at the
    address `buf` that an httm_exchange call names; raises if it is not
    inside the workspace or not aligned."""
    if ws is None or not buf:
        raise ValueError("no workspace for this exchange")
    off, n = int(buf) - ws.data_ptr(), int(count) * int(elem_bytes)
    if off < 0 or off + n > ws.numel() or elem_bytes not in (4, 8) or off % elem_bytes:
        raise ValueError("exchange buffer outside the workspace")
    return ws[off: off + n].view(torch.int32 if elem_bytes == 4 else torch.int64)


class TorchExchange:
    """``httm_exchange`` over torch.distributed: every sum the library asks
    for is ``dist.all_reduce`` of a view of the call's workspace (the library
    only sums buffers inside it), issued on the library's stream -- NCCL for
    CUDA workspaces, gloo for CPU tensors.  One object per thread of calls."""

    def __init__(self, group=None):
        self.group = group
        self.workspace = None
        self.calls = 0
        self._fn = EXCHANGE_FN(self._allreduce_sum)
        self.c = httm_exchange(self._fn, None)

    def _allreduce_sum(self, buf, count, elem_bytes, stream, user) -> int:
        import torch.distributed as dist
        try:
            t = exchange_view(self.workspace, buf, count, elem_bytes)
            if t.is_cuda:
                s = torch.cuda.ExternalStream(stream, device=t.device) if stream else \
                    torch.cuda.default_stream(t.device)
                with torch.cuda.stream(s):
                    dist.all_reduce(t, group=self.group)
            else:
                dist.all_reduce(t, group=self.group)
            self.calls += 1
            return 0
        except Exception:   # reported to the library, which returns HTTM_ERR_EXCHANGE
            return 1


def httm_forward_sharded(plan: Plan, Q, K, V, exchange, out=None, workspace=None, dbg: dict | None = None,
                         stream=None):
    """One shard of a head-sharded layer (Q, K, V: this shard's heads).
    ``exchange`` has a ``c`` (httm_exchange) and a ``workspace`` attribute,
    set here to the call's workspace (:class:`TorchExchange`), or is None
    for a single-shard plan."""
    out, workspace = _prep(plan, Q, K, V, out, workspace)
    ex = None
    if exchange is not None:
        exchange.workspace = workspace
        ex = ctypes.byref(exchange.c)
    d = ctypes.byref(_debug_struct(dbg)) if dbg is not None else None
    _check(load_library().httm_forward_sharded(plan.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(out),
                                               _ptr(workspace), workspace.numel(), ex, d, _stream(stream)),
           "httm_forward_sharded")
    return out
