"""Throughput of the merged global-attention layer (HTTM) on B200.

One step = one httm_forward over one VGGT-shaped layer: match, merge, the
outlier filter, attention and unmerge, with Q/K/V already resident in HBM.
On one GPU, value = the layer's tokens / step time.  Under torchrun with N > 1
ranks the layer is split by heads (16 / N heads per GPU, the outlier
filter's counts summed over NCCL between its steps): value = the layer's
tokens / step time, max over ranks (strong scaling).  --replicas instead
runs an independent layer per GPU (value = tokens of all ranks / step time,
weak scaling, no data-path collective).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload vggt_100f] [--replicas]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample
    python bench.py --sweep                # 1000-frame sweep of merge / outlier ratios and plan variants
    python bench.py --block-sweep          # block shapes n_s x n_t on the 100-frame layer

Prints one JSON line (rank 0); --sweep prints one line per sweep point.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "merged global-attn layer tokens/s at 100/500 frames; % of HBM & tensor roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="vggt_100f")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the 500-frame layer")
    ap.add_argument("--sweep", action="store_true",
                    help="1000-frame sweep: Q r x outlier d x (head-wise temporal, head-uniform, contiguous)")
    ap.add_argument("--sweep-rows", type=int, default=128, help="sampled query rows per head for the output error")
    ap.add_argument("--block-sweep", action="store_true",
                    help="100-frame layer: spatial (n_t = 1) against spatio-temporal block shapes at three block sizes")
    ap.add_argument("--skewed", action="store_true",
                    help="100-frame layer with identical query and key tokens: every source of a block picks the "
                         "same destination (one group of ~2,700 members per block and head)")
    ap.add_argument("--shard-heads", action="store_true",
                    help="run the head-sharded layer even on one rank (through httm_forward_sharded)")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1 ranks: an independent layer per GPU (weak scaling) instead of one layer "
                         "split by heads over the ranks")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ----------------------------------------------------------------------------

def oracle_sample(w, Q, K, V, attn_rows: int, seed: int = 0) -> dict:
    """The fp64 oracle, as it stands, on one head of the layer: the full plan
    (matching, merging, outlier filter on that head's share of the budget)
    plus attention for `attn_rows` seeded query slots, scaled linearly to all
    slots and all heads.  Returns the extrapolated layer throughput."""
    import numpy as np

    import oracle.httm_oracle as O

    q, k, v = (t[:1].float().cpu().numpy().astype(np.float64) for t in (Q, K, V))
    cfg = O.OracleConfig(h=1, T=w.T, P=w.P, d=w.d, n_s=w.n_s, n_t=w.n_t, q_stride=w.q_stride,
                         kv_stride=w.kv_stride, q_pct=w.q_pct, kv_pct=w.kv_pct, out_pct=w.out_pct,
                         mode=w.mode, contig_block=w.contig_block)
    t0 = time.perf_counter()
    res = O.forward_plan(cfg, q, k, v)
    t_plan = time.perf_counter() - t0
    qt = res.restore.q_tilde[0]
    live = np.concatenate([res.restore.live[0], np.ones(res.restore.n_out[0], dtype=bool)])
    rows = np.nonzero(live)[0]
    rng = np.random.default_rng(seed)
    pick = np.sort(rng.choice(rows, min(attn_rows, rows.shape[0]), replace=False))
    O.attention(qt[pick[:8]], res.k_means[0], res.v_means[0], cfg.softmax_scale)  # wake the BLAS threads
    t1 = time.perf_counter()
    O.attention(qt[pick], res.k_means[0], res.v_means[0], cfg.softmax_scale)
    t_attn = time.perf_counter() - t1
    head_s = t_plan + t_attn * rows.shape[0] / pick.shape[0]
    layer_s = head_s * w.h
    return {"value": w.N / layer_s, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"head 0 of {w.h}: full plan of all {len(O.block_list(cfg))} blocks "
                       f"({t_plan:.2f} s) + attention of {pick.shape[0]} of {rows.shape[0]} query slots "
                       f"({t_attn:.2f} s), scaled linearly to all slots and heads"),
            "measured_s": t_plan + t_attn}


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        if self.proc is not None:
            time.sleep(0.3)   # let the sampler start before the timed region does

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.f.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(n)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def traffic_record(kernel_file: str, workload: str):
    """DRAM bytes per launch of a kernel on a workload, from a committed ncu
    summary (profiles/traffic.json), if the kernel source is unchanged since
    the counters were taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(os.path.basename(kernel_file), {}).get(workload)
    if not rec:
        return None
    sha = hashlib.sha256(open(kernel_file, "rb").read()).hexdigest()[:16]
    return rec if rec.get("source_sha") == sha else None


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of every rank's value (each rank times its own layer; the
    job's step time is the slowest rank's)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measure_layer(w, steps: int, warmup: int, rank: int, world: int, dev, with_e2e: bool = True):
    """Time `steps` forward calls of one layer (inputs resident in HBM) with
    stage events on, then the same call end to end from pinned host memory."""
    import torch
    import torch.distributed as dist

    from token_merging_view_b200 import binding as B
    from token_merging_view_b200.inputs import make_qkv

    Q, K, V = make_qkv(T=w.T, grid=w.grid, h=w.h, d=w.d, seed=w.seed + 1000 * rank, noise_sigma=w.noise_sigma,
                       max_shift=w.max_shift, dtype=torch.float32 if w.fp32 else torch.bfloat16, device=dev)
    plan = B.httm_plan(B.LayerConfig.from_workload(w))
    ws = plan.new_workspace(dev)
    out = torch.empty_like(Q)
    stream = torch.cuda.current_stream()

    def step():
        B.httm_forward(plan, Q, K, V, out=out, workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert B.httm_get_device_status(plan, ws) == 0
    n_out = B.workspace_view(plan, ws, "n_out").cpu()
    sum_lq = w.h * plan.info.q_slots + int(n_out.sum())

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, n):
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        barrier()
        return max_over_ranks(a.elapsed_time(b), world, dev)

    # the timed steps run as a caller runs them: without stage timing, the
    # key branch beside the query branch on the library's side stream; the
    # stage breakdown comes from a second pass with stage timing on (the
    # stages then run in order, each between two events)
    clocks = Clocks(dev.index if dev.index is not None else 0)
    total_ms = timed(step, steps)
    clk = clocks.stop()
    launches = plan.launches() * steps
    plan.profile(True)
    plan.profile_read()
    timed(step, steps)
    stages = plan.profile_read()
    plan.profile(False)
    res = {"plan": plan, "Q": Q, "K": K, "V": V, "ms_step": total_ms / steps, "stages": stages, "sum_lq": sum_lq,
           "launches": launches, "clocks": clk}
    if with_e2e:
        # the unmerge folded into the attention epilogue (httm_set_fused_unmerge),
        # timed the same two ways, then switched back off
        B.httm_set_fused_unmerge(plan, True)
        step()
        torch.cuda.synchronize()
        assert B.httm_get_device_status(plan, ws) == 0
        fused_ms = timed(step, steps) / steps
        plan.profile(True)
        plan.profile_read()
        timed(step, steps)
        fstages = plan.profile_read()
        plan.profile(False)
        B.httm_set_fused_unmerge(plan, False)
        res["fused_unmerge"] = {"ms_per_step": round(fused_ms, 4), "launches": plan.launches(),
                                "attention_ms_with_unmerge": round(fstages["attention"][0] / steps, 4),
                                "default_attention_plus_unmerge_ms": round(
                                    (stages["attention"][0] + stages["unmerge"][0]) / steps, 4)}
    if with_e2e:
        # Cached merge indices (LiteVGGT note, key design 3): the following
        # layers reuse the member lists the last full call left in `ws`.
        # Same inputs here; the reused call skips matching and top-r planning.
        def reuse():
            B.httm_forward_reuse(plan, Q, K, V, out=out, workspace=ws, stream=stream)

        reuse()
        torch.cuda.synchronize()
        assert B.httm_get_device_status(plan, ws) == 0
        reuse_ms = timed(reuse, steps) / steps
        reuse_launches = plan.launches()
        plan.profile(True)
        plan.profile_read()
        timed(reuse, steps)
        rstages = plan.profile_read()
        plan.profile(False)
        res["reuse"] = {"ms": reuse_ms, "launches": reuse_launches,
                        "stages": {k: round(v[0] / steps, 4) for k, v in rstages.items()}}
    if with_e2e:
        # End to end through the same C ABI call, from pinned host memory:
        # every step copies its Q/K/V in and its output back.  Two device
        # buffer sets and one copy stream per direction pipeline the steps,
        # as a caller of the asynchronous API would: step i+1's inputs travel
        # in while step i computes and step i-1's output travels back (the
        # link carries both directions at once).
        hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
        hO = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        dIn = [(Q, K, V), tuple(torch.empty_like(t) for t in (Q, K, V))]
        dOut = [out, torch.empty_like(out)]
        ws2 = [ws, plan.new_workspace(dev)]
        c_in = torch.cuda.Stream(device=dev)
        c_out = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_out:
            e.record(c_out)
        for e in ev_done:
            e.record(stream)

        def e2e_run(n):
            c_in.wait_stream(stream)
            c_out.wait_stream(stream)
            with torch.cuda.stream(c_in):
                for t, h in zip(dIn[0], (hQ, hK, hV)):
                    t.copy_(h, non_blocking=True)
                ev_in[0].record(c_in)
            for i in range(n):
                b = i & 1
                if i + 1 < n:                   # prefetch the next step's inputs
                    nb = (i + 1) & 1
                    with torch.cuda.stream(c_in):
                        c_in.wait_event(ev_done[nb])
                        for t, h in zip(dIn[nb], (hQ, hK, hV)):
                            t.copy_(h, non_blocking=True)
                        ev_in[nb].record(c_in)
                stream.wait_event(ev_in[b])
                stream.wait_event(ev_out[b])    # the output buffer has been drained
                B.httm_forward(plan, *dIn[b], out=dOut[b], workspace=ws2[b], stream=stream)
                ev_done[b].record(stream)
                with torch.cuda.stream(c_out):
                    c_out.wait_event(ev_done[b])
                    hO[b].copy_(dOut[b], non_blocking=True)
                    ev_out[b].record(c_out)
            stream.wait_stream(c_in)
            stream.wait_stream(c_out)

        e2e_run(2)
        n = max(3, steps)
        res["e2e_ms"] = timed(lambda: e2e_run(n), 1) / n
        res["h2d"] = 3 * Q.numel() * Q.element_size()
        res["d2h"] = out.numel() * out.element_size()
        del ws2, dIn, dOut
    return res


def roofline_of(w, r, steps: int):
    """Attention (the dominant kernel) against the bf16 tensor peak, and the
    memory-bound stages against the HBM copy bandwidth.

    The attention peak is the measured burst figure: the timed region is
    short and the SM clock stays near its maximum (the run's clock record
    shows it), while the sustained figure was measured at the ~1.3 GHz a
    seconds-long GEMM loop settles to under the power cap.  For context the
    line also gives the fraction of the sustained peak scaled to this run's
    median SM clock."""
    import token_merging_view_b200 as pkg
    pk, pk_kind = peaks()
    plan = r["plan"]
    att_ms, att_n = r["stages"]["attention"]
    att_avg_ms = att_ms / max(1, att_n)
    flops = 4.0 * w.d * plan.info.kv_slots * r["sum_lq"]
    achieved = flops / (att_avg_ms / 1e3) / 1e12
    peak = pk["bf16_tflops"]
    sus = pk.get("bf16_tflops_sustained")
    sus_mhz = (pk.get("clocks_under_load") or {}).get("sm_mhz_median")
    run_mhz = (r.get("clocks") or {}).get("sm_mhz")
    att_src = os.path.join(os.path.dirname(pkg.__file__), "csrc", "attn_tc.cu")
    tr = traffic_record(att_src, w.name)
    roof = {"bound": "tensor", "kernel": "attention (attn_tc_kernel)", "achieved": round(achieved, 2),
            "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "peak_kind": f"{pk_kind} bf16 burst (short timed region at full SM clock)",
            "traffic": tr["bytes_per_launch"] if tr else None,
            "algorithmic_flops_per_launch": flops, "avg_launch_ms": round(att_avg_ms, 4)}
    if sus:
        roof["frac_of_sustained"] = round(achieved / sus, 4)
        if sus_mhz and run_mhz:
            scaled = min(peak, sus * run_mhz / sus_mhz)
            roof["frac_of_sustained_at_run_clock"] = round(achieved / scaled, 4)
            roof["sustained_at_run_clock_note"] = (f"sustained {sus} TFLOP/s measured at {sus_mhz:.0f} MHz, "
                                                   f"scaled to this run's {run_mhz:.0f} MHz median "
                                                   f"(capped at the burst peak): {scaled:.1f}")
    es = 4 if w.fp32 else 2
    row = w.d * es
    hn = w.h * w.N
    sum_lq = r["sum_lq"]
    n_out = sum_lq - w.h * plan.info.q_slots
    kv_rows = w.h * plan.info.kv_slots
    hbm = pk["hbm_gbs"]

    def per_ms(b, ms):
        return {"algorithmic_bytes": int(b), "ms": round(ms, 4), "GBps": round(b / ms / 1e6, 1),
                "frac_of_measured_hbm": round(b / ms / 1e6 / hbm, 4), "frac_of_8TBps": round(b / ms / 8e9, 4)}

    st = {k: v[0] / steps for k, v in r["stages"].items()}
    # the memory stages as one row: top-r merge, outlier filter and restore,
    # unmerge.  Bytes the method must move: read Q, K, V; re-read the
    # outliers' rows; write Q~ (regular and outlier rows), K~, V~; slot maps
    # and deviations (~20 B per token and head); read O~ and write out.
    total = (3 * hn * row + n_out * row + (sum_lq + 2 * kv_rows) * row + 20 * hn + sum_lq * row + hn * row)
    mem = {"merge+outlier+unmerge": per_ms(total, st["merge"] + st["outlier"] + st["unmerge"])}
    # per stage: merge reads Q, K, V and writes Q~ regular rows, K~, V~, the
    # slot map and the deviation keys; unmerge reads O~ and the slot map and
    # writes out
    parts = {"merge": 3 * hn * row + (w.h * plan.info.q_slots + 2 * kv_rows) * row + 8 * hn,
             "unmerge": hn * row + sum_lq * row + 4 * hn}
    for k, b in parts.items():
        if st[k] > 0:
            mem[k] = per_ms(b, st[k])
    # matching: 2 * n_dst * d flops per source on the tensor cores, and one
    # argmax element per (source, destination) pair on the CUDA cores
    pairs = 0
    for stride in (w.q_stride, w.kv_stride):
        for nb in block_sizes(w):
            nd = -(-nb // stride)
            pairs += (nb - nd) * nd
    pairs *= w.h
    mflops = 2.0 * pairs * w.d
    match = None
    if st["match"] > 0:
        tf = mflops / (st["match"] / 1e3) / 1e12
        match = {"ms": round(st["match"], 4), "algorithmic_flops": mflops, "TFLOPs": round(tf, 2),
                 "frac_of_tensor_burst": round(tf / peak, 4), "argmax_elements": pairs,
                 "argmax_G_per_s": round(pairs / (st["match"] / 1e3) / 1e9, 1)}
    return roof, mem, match


def workload_config(w, world: int) -> dict:
    """The bench line's `config`: the workload's definition only (both arms
    print the same dict for the same workload)."""
    es = 4 if w.fp32 else 2
    return {"workload": w.name, "frames": w.T, "patches_per_frame": w.P, "tokens": w.N, "heads": w.h,
            "d_head": w.d, "n_s": w.n_s, "n_t": w.n_t, "q_dst_stride": w.q_stride,
            "kv_dst_stride": w.kv_stride, "q_merge_pct": w.q_pct, "kv_merge_pct": w.kv_pct,
            "outlier_pct": w.out_pct,
            "parallelism": f"independent layer per GPU x{world}" if world > 1 else "single GPU",
            "l2": f"inputs larger than L2 ({3 * w.h * w.N * w.d * es / 2**20:.0f} MiB of Q/K/V vs 126 MB)"}


def block_sizes(w):
    """Token counts of the merge blocks of one head (HTTM note, key design 2:
    n_s patches of n_t frames; contiguous runs in the contiguous variant)."""
    from token_merging_view_b200.workloads import CONTIGUOUS
    if w.mode == CONTIGUOUS:
        return [min(w.contig_block, w.N - s) for s in range(0, w.N, w.contig_block)]
    out = []
    for t0 in range(0, w.T, w.n_t):
        tg = min(w.n_t, w.T - t0)
        for p0 in range(0, w.P, w.n_s):
            out.append(tg * min(w.n_s, w.P - p0))
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    from token_merging_view_b200 import binding as B
    from token_merging_view_b200.inputs import make_qkv
    from token_merging_view_b200.workloads import WORKLOADS

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev)
    w = WORKLOADS[args.workload]
    r = measure_layer(w, args.steps, args.warmup, rank, world, dev)
    ms_step = r["ms_step"]
    value = world * w.N / (ms_step / 1e3)
    roof, mem, match = roofline_of(w, r, args.steps)
    Q = r["Q"]
    es = 4 if w.fp32 else 2

    dense = None
    if not args.no_dense and rank == 0 and world == 1:
        dplan = B.httm_plan(B.LayerConfig.from_workload(w, mode=B.HTTM_DENSE))
        dws = dplan.new_workspace(dev)
        out = torch.empty_like(Q)
        Kd, Vd = r["K"], r["V"]
        B.httm_forward(dplan, Q, Kd, Vd, out=out, workspace=dws)
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        B.httm_forward(dplan, Q, Kd, Vd, out=out, workspace=dws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        dms = a.elapsed_time(b)
        dflops = 4.0 * w.d * w.h * float(w.N) * w.N
        dense = {"tokens_per_s": round(w.N / (dms / 1e3), 1), "ms": round(dms, 3),
                 "TFLOPs": round(dflops / (dms / 1e3) / 1e12, 2)}
        del dws, dplan, out, Kd, Vd
    plan_info = (r["plan"].info.q_slots, r["plan"].info.kv_slots)
    sum_lq = r["sum_lq"]
    e2e = {"value": round(world * w.N / (r["e2e_ms"] / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]}
    launches, clk, stages = r["launches"], r["clocks"], r["stages"]
    fused_unmerge = r.get("fused_unmerge")
    ru = r["reuse"]
    group = ms_step + 5 * ru["ms"]          # indices computed on one layer of six, reused on five
    cached = {"ms_per_reused_layer": round(ru["ms"], 4), "launches_per_reused_layer": ru["launches"],
              "stage_ms_per_reused_layer": ru["stages"],
              "six_layer_group_ms": round(group, 4), "six_layer_group_saving_pct": round(100 * (1 - group / (6 * ms_step)), 2),
              "layer_tokens_per_s_six_layer_group": round(world * 6 * w.N / (group / 1e3), 1)}
    del r, Q
    torch.cuda.empty_cache()

    secondary = None
    if not args.no_secondary and world == 1 and args.workload != "vggt_500f":
        w2 = WORKLOADS["vggt_500f"]
        r2 = measure_layer(w2, 3, 2, rank, world, dev, with_e2e=False)
        roof2, mem2, match2 = roofline_of(w2, r2, 3)
        secondary = {"workload": w2.name, "tokens": w2.N, "value": round(w2.N / (r2["ms_step"] / 1e3), 1),
                     "unit": "tokens/s", "ms_per_step": round(r2["ms_step"], 3), "steps": 3,
                     "roofline": roof2, "memory_stages": mem2, "match": match2,
                     "stage_ms_per_step": {k: round(v[0] / 3, 4) for k, v in r2["stages"].items()}}
        del r2
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Qc, Kc, Vc = make_qkv(T=w.T, grid=w.grid, h=1, d=w.d, seed=w.seed, noise_sigma=w.noise_sigma,
                              max_shift=w.max_shift, dtype=torch.float32 if w.fp32 else torch.bfloat16)
        cpu = oracle_sample(w, Qc, Kc, Vc, 512 if w.N <= 200_000 else 128)
        cpu.pop("measured_s", None)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            # one GPU: the first point of the head-sharded series (one layer split
            # over the ranks, total work fixed); replicas on several GPUs: weak
            "higher_is_better": True, "scaling": "strong" if world == 1 else "weak", "vs_baseline": None,
            "dtype": "f32" if w.fp32 else "bf16",
            "data": "synthetic (seeded blurred-field Q/K/V, VGGT global-attention shapes)",
            "config": workload_config(w, world),
            "layer_rows": {"q_rows": sum_lq, "kv_rows_per_head": plan_info[1]},
            "e2e": e2e,
            "gpu_launches": launches,
            "roofline": roof,
            "memory_stages": mem,
            "match": match,
            "stage_ms_per_step": {k: round(v[0] / args.steps, 4) for k, v in stages.items()},
            "stage_ms_note": "stages timed in a second pass with stage timing on (stages in order); "
                             "value and ms_per_step from the pass without (key branch beside query branch)",
            "dense_attention_same_length": dense,
            "cached_merge_indices": cached,
            "fused_unmerge": fused_unmerge,
            "secondary_workload": secondary,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# 1000-frame sweep of the merge settings and the plan variants
# ----------------------------------------------------------------------------

def sweep_points(w):
    """Q merge ratio r x outlier ratio d (K/V r = 50 %), each with the three
    plans: head-wise temporal blocks (HTTM), one head-uniform plan per block
    (the mean over heads of the cosines, as ToMe/FastVGGT merge), and
    contiguous un-reordered blocks of 3840 tokens (HTTM note, background
    section and key design 2).  r = 85 % needs destinations every 8th token:
    every 4th leaves only 75 % of a block as sources."""
    from token_merging_view_b200.workloads import CONTIGUOUS, HEAD_UNIFORM, HEADWISE_TEMPORAL
    pts = []
    for r in (50, 70, 85):
        for d in (0, 5, 10):
            for mode, name in ((HEADWISE_TEMPORAL, "headwise_temporal"), (HEAD_UNIFORM, "head_uniform"),
                               (CONTIGUOUS, "contiguous_3840")):
                pts.append((name, w.with_(q_pct=r, q_stride=8 if r == 85 else 4, kv_pct=50, kv_stride=4,
                                          out_pct=d, mode=mode, contig_block=3840)))
    return pts


def dense_rows(Q, K, V, idx, scale):
    """softmax(q K^T * scale) V for the sampled query rows of every head, in
    float64 on the device (torch), as the unmerged layer's reference."""
    import torch
    outs = []
    for hh in range(Q.shape[0]):
        q = Q[hh, idx[hh]].double()
        s = (q @ K[hh].double().T) * scale
        p = torch.softmax(s, dim=-1)
        outs.append(p @ V[hh].double())
        del s, p
    return torch.stack(outs)


def deviation_stats(Q, dbg, n_q_slots):
    """Pre-filter query deviation ||q_n - q~_G(n)|| (mean, p99 over all h x N
    tokens, 0 for singletons) and the deviation of each non-outlier from its
    restored slot (mean over all non-outliers, and over those whose restored
    slot still holds >= 2 tokens)."""
    import torch
    dev = dbg["dev"]
    flat = dev.flatten()
    k = max(1, int(0.99 * flat.numel()))
    p99 = float(flat.kthvalue(k).values)
    post_sum, post_n, post_m_sum, post_m_n = 0.0, 0, 0.0, 0
    for hh in range(Q.shape[0]):
        slot = dbg["q_slot"][hh].long()
        # outliers own slots past the regular ones: never index with those
        keep = (dbg["outlier"][hh] == 0) & (slot >= 0) & (slot < n_q_slots)
        s_reg = torch.where(keep, slot, torch.zeros_like(slot))
        cnt = torch.bincount(s_reg[keep], minlength=n_q_slots)
        merged = cnt[s_reg] >= 2
        diff = Q[hh].float() - dbg["q_restored"][hh][s_reg]
        dn = diff.norm(dim=-1)
        post_sum += float(dn[keep].sum())
        post_n += int(keep.sum())
        sel = keep & merged
        post_m_sum += float(dn[sel].sum())
        post_m_n += int(sel.sum())
    return {"pre_filter_dev_mean": round(float(flat.mean()), 5), "pre_filter_dev_p99": round(p99, 5),
            "restored_dev_mean_non_outliers": round(post_sum / max(1, post_n), 5),
            "restored_dev_mean_merged_non_outliers": round(post_m_sum / max(1, post_m_n), 5)}


def run_sweep(args):
    import torch

    from token_merging_view_b200 import binding as B
    from token_merging_view_b200.inputs import make_qkv
    from token_merging_view_b200.workloads import WORKLOADS

    rank, world, local = dist_env()
    if rank != 0:
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = WORKLOADS["vggt_1000f"]
    Q, K, V = make_qkv(T=w.T, grid=w.grid, h=w.h, d=w.d, seed=w.seed, noise_sigma=w.noise_sigma,
                       max_shift=w.max_shift, dtype=torch.bfloat16, device=dev)
    g = torch.Generator(device="cpu").manual_seed(1234)
    idx = torch.stack([torch.randperm(w.N, generator=g)[: args.sweep_rows].sort().values for _ in range(w.h)]).to(dev)
    scale = w.d ** -0.5
    ref = dense_rows(Q, K, V, idx, scale)
    out = torch.empty_like(Q)
    stream = torch.cuda.current_stream()
    base_rows = {}
    clocks = Clocks(dev.index if dev.index is not None else 0)
    for name, pw in sweep_points(w):
        plan = B.httm_plan(B.LayerConfig.from_workload(pw))
        ws = plan.new_workspace(dev)
        dbg = B.debug_buffers(plan, dev)
        B.httm_forward_debug(plan, Q, K, V, dbg, out=out, workspace=ws)     # also the warm-up
        status = B.httm_get_device_status(plan, ws)
        n_out = int(B.workspace_view(plan, ws, "n_out").sum())
        stats = deviation_stats(Q, dbg, plan.info.q_slots)
        rows = torch.stack([out[hh, idx[hh]] for hh in range(w.h)]).double()
        err = (rows - ref).norm() / ref.norm()
        key = (pw.q_pct, pw.out_pct)
        if name == "headwise_temporal":
            base_rows[key] = rows
        vs_ht = (rows - base_rows[key]).norm() / base_rows[key].norm() if key in base_rows else None
        del dbg
        steps = 2
        plan.profile(True)
        plan.profile_read()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            B.httm_forward(plan, Q, K, V, out=out, workspace=ws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
        stages = {k: round(v[0] / steps, 3) for k, v in plan.profile_read().items()}
        line = {"sweep": w.name, "plan": name, "q_merge_pct": pw.q_pct, "q_dst_stride": pw.q_stride,
                "kv_merge_pct": pw.kv_pct, "outlier_pct": pw.out_pct, "status": status,
                "tokens_per_s": round(w.N / (ms / 1e3), 1), "ms_per_step": round(ms, 2), "steps": steps,
                "q_rows": w.h * plan.info.q_slots + n_out, "kv_rows_per_head": plan.info.kv_slots,
                "stage_ms": stages, **stats,
                "out_rel_l2_vs_dense_sampled": round(float(err), 5),
                "out_rel_l2_vs_headwise_temporal_sampled": None if vs_ht is None else round(float(vs_ht), 5),
                "sampled_rows_per_head": args.sweep_rows}
        print(json.dumps(line), flush=True)
        del ws, plan
        torch.cuda.empty_cache()
    print(json.dumps({"sweep": w.name, "clocks": clocks.stop()}), flush=True)


def block_shapes():
    """(n_s, n_t) pairs at three block sizes: a purely spatial block (n_t = 1,
    n_s <= 1369 patches of one frame) against the same number of tokens
    spread over more frames (HTTM note, key design 2 and the spatial /
    temporal trade-off of its analysis section)."""
    return {
        "~800": [(800, 1), (400, 2), (200, 4), (100, 8), (50, 16), (27, 30)],
        "~1369": [(1369, 1), (685, 2), (343, 4), (172, 8), (92, 15), (46, 30)],
        "~3840": [(1280, 3), (640, 6), (384, 10), (256, 15), (128, 30), (64, 60)],
    }


def run_block_sweep(args):
    import torch

    from token_merging_view_b200 import binding as B
    from token_merging_view_b200.inputs import make_qkv
    from token_merging_view_b200.workloads import WORKLOADS

    rank, world, local = dist_env()
    if rank != 0:
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = WORKLOADS["vggt_100f"]
    Q, K, V = make_qkv(T=w.T, grid=w.grid, h=w.h, d=w.d, seed=w.seed, noise_sigma=w.noise_sigma,
                       max_shift=w.max_shift, dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(Q)
    stream = torch.cuda.current_stream()
    clocks = Clocks(dev.index if dev.index is not None else 0)
    for size, shapes in block_shapes().items():
        for n_s, n_t in shapes:
            pw = w.with_(n_s=n_s, n_t=n_t)
            plan = B.httm_plan(B.LayerConfig.from_workload(pw))
            ws = plan.new_workspace(dev)
            dbg = B.debug_buffers(plan, dev)
            B.httm_forward_debug(plan, Q, K, V, dbg, out=out, workspace=ws)     # also the warm-up
            status = B.httm_get_device_status(plan, ws)
            stats = deviation_stats(Q, dbg, plan.info.q_slots)
            kdev = None
            if dbg.get("k_means") is not None:
                # key deviation from the key means, per token (0 for singletons)
                ks, tot, n = dbg["k_slot"], 0.0, 0
                for hh in range(w.h):
                    sl = ks[hh].long()
                    d = (K[hh].float() - dbg["k_means"][hh][sl]).norm(dim=-1)
                    tot += float(d.sum())
                    n += d.numel()
                kdev = round(tot / max(1, n), 5)
            del dbg
            steps = 5
            plan.profile(True)
            plan.profile_read()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                B.httm_forward(plan, Q, K, V, out=out, workspace=ws, stream=stream)
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
            stages = {k: round(v[0] / steps, 4) for k, v in plan.profile_read().items()}
            line = {"block_sweep": w.name, "block_size": size, "n_s": n_s, "n_t": n_t,
                    "n_b_full": n_s * n_t, "blocks_per_head": plan.info.n_blocks, "status": status,
                    "tokens_per_s": round(w.N / (ms / 1e3), 1), "ms_per_step": round(ms, 3), "stage_ms": stages,
                    "q_pre_filter_dev_mean": stats["pre_filter_dev_mean"],
                    "q_pre_filter_dev_p99": stats["pre_filter_dev_p99"],
                    "q_restored_dev_mean_non_outliers": stats["restored_dev_mean_non_outliers"],
                    "k_dev_mean": kdev}
            print(json.dumps(line), flush=True)
            del ws, plan
            torch.cuda.empty_cache()
    print(json.dumps({"block_sweep": w.name, "clocks": clocks.stop()}), flush=True)


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return
    import torch

    from token_merging_view_b200.inputs import make_qkv
    from token_merging_view_b200.workloads import WORKLOADS

    w = WORKLOADS[args.workload]
    Q, K, V = make_qkv(T=w.T, grid=w.grid, h=1, d=w.d, seed=w.seed, noise_sigma=w.noise_sigma,
                       max_shift=w.max_shift, dtype=torch.float32 if w.fp32 else torch.bfloat16)
    rows = 128
    for _ in range(args.warmup):
        oracle_sample(w, Q, K, V, rows)
    vals, secs, last = [], 0.0, None
    for i in range(args.steps):
        last = oracle_sample(w, Q, K, V, rows, seed=i)
        vals.append(last["value"])
        secs += last.pop("measured_s")
    value = statistics.median(vals)
    value = round(value, 2)
    cpu = {"value": value, "unit": "tokens/s", "cores": last["cores"], "kind": "oracle", "sample": last["sample"]}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded blurred-field Q/K/V, VGGT global-attention shapes)",
            "config": workload_config(w, world),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "cpu_baseline": cpu}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# one layer split by heads over the ranks (HTTM note, key design 3: every step
# is per head except the outlier filter's global top-d%, whose counts the
# ranks sum over NCCL between the filter's steps)
# ----------------------------------------------------------------------------

def shard_heads(H: int, world: int) -> int:
    """Heads per rank of an H-head layer split over `world` ranks."""
    if world < 1 or H % world != 0:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    return H // world


def sharded_line(w, world: int, steps: int, warmup: int, ms_step: float, e2e_ms: float, h2d: int, d2h: int,
                 launches: int, exchanges: int, roof: dict, stages: dict, clocks) -> dict:
    """The bench line of a head-sharded layer: `value` counts the layer's
    tokens once (the ranks split one layer: strong scaling)."""
    h = shard_heads(w.h, world)
    cfg = workload_config(w, world)
    cfg["parallelism"] = (f"head-sharded x{world} ({h} of {w.h} heads per GPU; the outlier filter's counts "
                          f"summed over the ranks by NCCL all-reduce)")
    return {
        "metric": METRIC, "value": round(w.N / (ms_step / 1e3), 1), "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f32" if w.fp32 else "bf16",
        "data": "synthetic (seeded blurred-field Q/K/V, VGGT global-attention shapes)",
        "config": cfg,
        "e2e": {"value": round(w.N / (e2e_ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches, "collectives_per_step": exchanges,
        "roofline": roof, "stage_ms_per_step_rank0": stages, "clocks": clocks,
    }


def run_sharded(args):
    import torch
    import torch.distributed as dist

    from token_merging_view_b200 import binding as B
    from token_merging_view_b200.inputs import make_qkv
    from token_merging_view_b200.workloads import WORKLOADS

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    w = WORKLOADS[args.workload]
    h = shard_heads(w.h, world)
    # every rank draws the whole layer from the same seed and keeps its heads
    Qa, Ka, Va = make_qkv(T=w.T, grid=w.grid, h=w.h, d=w.d, seed=w.seed, noise_sigma=w.noise_sigma,
                          max_shift=w.max_shift, dtype=torch.float32 if w.fp32 else torch.bfloat16, device=dev)
    Q, K, V = (t[rank * h:(rank + 1) * h].contiguous() for t in (Qa, Ka, Va))
    del Qa, Ka, Va
    torch.cuda.empty_cache()
    plan = B.httm_plan(B.LayerConfig.from_workload(w, h=h)).shard(rank, world)
    ws = plan.new_workspace(dev)
    out = torch.empty_like(Q)
    stream = torch.cuda.current_stream()
    ex = B.TorchExchange() if world > 1 else None

    def step(q=Q, k=K, v=V, o=out, wsp=ws):
        B.httm_forward_sharded(plan, q, k, v, ex, out=o, workspace=wsp, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert B.httm_get_device_status(plan, ws) == 0
    n_out = B.workspace_view(plan, ws, "n_out").cpu()
    sum_lq = h * plan.info.q_slots + int(n_out.sum())

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, n):
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        barrier()
        return max_over_ranks(a.elapsed_time(b), world, dev)

    calls0 = ex.calls if ex else 0
    clocks = Clocks(dev.index if dev.index is not None else 0)
    total_ms = timed(step, args.steps)
    clk = clocks.stop()
    exchanges = ((ex.calls - calls0) // args.steps) if ex else 0
    launches = plan.launches() * args.steps * world
    plan.profile(True)
    plan.profile_read()
    timed(step, args.steps)
    stages = plan.profile_read()
    plan.profile(False)
    # end to end: this rank's heads of Q, K, V from pinned host memory, its
    # output back, every step
    hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
    hO = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

    def e2e_step():
        for t, hsrc in zip((Q, K, V), (hQ, hK, hV)):
            t.copy_(hsrc, non_blocking=True)
        step()
        hO.copy_(out, non_blocking=True)

    e2e_step()
    e2e_ms = timed(e2e_step, args.steps) / args.steps
    h2d = 3 * Q.numel() * Q.element_size() * world
    d2h = out.numel() * out.element_size() * world
    ms_step = total_ms / args.steps
    att_ms, att_n = stages["attention"]
    flops = 4.0 * w.d * plan.info.kv_slots * sum_lq
    pk, pk_kind = peaks()
    achieved = flops / (att_ms / max(1, att_n) / 1e3) / 1e12
    roof = {"bound": "tensor", "kernel": "attention (attn_tc_kernel), rank 0's heads", "achieved": round(achieved, 2),
            "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
            "peak_kind": f"{pk_kind} bf16 burst", "traffic": None}
    if rank == 0:
        line = sharded_line(w, world, args.steps, args.warmup, ms_step, e2e_ms, h2d, d2h, launches, exchanges, roof,
                            {k: round(v[0] / args.steps, 4) for k, v in stages.items()}, clk)
        print(json.dumps(line), flush=True)
    del plan, ws
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_skewed(args):
    """The degenerate case of the merge plan: Q and K identical across every
    token of a head (V as usual), so every cosine ties, every source takes
    its block's first destination (lowest index) and the top-r merge puts
    ~70 % of each block into one group.  Times the layer with stage timing
    next to the regular layer."""
    import torch

    from token_merging_view_b200 import binding as B
    from token_merging_view_b200.inputs import make_qkv
    from token_merging_view_b200.workloads import WORKLOADS

    rank, world, local = dist_env()
    if rank != 0:
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    Q, K, V = make_qkv(T=w.T, grid=w.grid, h=w.h, d=w.d, seed=w.seed, noise_sigma=w.noise_sigma,
                       max_shift=w.max_shift, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    clocks = Clocks(dev.index if dev.index is not None else 0)
    lines = {}
    for name, (q, k) in (("regular", (Q, K)),
                         ("identical_qk", (Q[:, :1].expand_as(Q).contiguous(), K[:, :1].expand_as(K).contiguous()))):
        plan = B.httm_plan(B.LayerConfig.from_workload(w))
        ws = plan.new_workspace(dev)
        out = torch.empty_like(Q)
        for _ in range(args.warmup):
            B.httm_forward(plan, q, k, V, out=out, workspace=ws, stream=stream)
        torch.cuda.synchronize()
        status = B.httm_get_device_status(plan, ws)
        steps = max(3, args.steps)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            B.httm_forward(plan, q, k, V, out=out, workspace=ws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        plan.profile(True)
        plan.profile_read()
        for _ in range(steps):
            B.httm_forward(plan, q, k, V, out=out, workspace=ws, stream=stream)
        stages = {kk: round(v[0] / steps, 4) for kk, v in plan.profile_read().items()}
        lines[name] = {"status": status, "ms_per_step": round(a.elapsed_time(b) / steps, 3), "stage_ms": stages}
        del ws, plan
        torch.cuda.empty_cache()
    print(json.dumps({"skewed_groups": w.name, **lines, "clocks": clocks.stop()}), flush=True)


def main():
    args = parse()
    _, world, _ = dist_env()
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.block_sweep:
        run_block_sweep(args)
    elif args.skewed:
        run_skewed(args)
    elif (world > 1 and not args.replicas) or args.shard_heads:
        run_sharded(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
