"""bench.py's command-line contract on the CPU: the reference arm (the
oracle on a bounded sample of the 100-frame layer) prints one JSON line
with the fields the driver reads, ranks other than 0 print nothing, and the
CUDA arm fails loudly on a machine without a GPU instead of falling back."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None, timeout=300):
    e = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        e.pop(k, None)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=e,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_json_line():
    import bench
    r = _bench("--impl", "reference", "--steps", "2", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "vggt_100f" and d["config"]["tokens"] == 136_900
    from token_merging_view_b200.workloads import WORKLOADS
    assert d["config"] == bench.workload_config(WORKLOADS["vggt_100f"], 1)   # the dict our arm prints
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]


def test_reference_arm_other_ranks_print_nothing():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "1",
               env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_cuda_arm_fails_without_a_gpu():
    r = _bench("--steps", "1", "--warmup", "1", "--no-cpu-baseline")
    assert r.returncode != 0
    assert not any(ln.startswith("{") for ln in r.stdout.splitlines())


def test_head_sharded_line_names_the_split():
    """With N > 1 ranks bench.py splits one layer by heads: its line counts
    the layer's tokens once (strong scaling) and names the split."""
    import bench
    from token_merging_view_b200.workloads import WORKLOADS
    w = WORKLOADS["vggt_100f"]
    assert [bench.shard_heads(16, n) for n in (1, 2, 4, 8, 16)] == [16, 8, 4, 2, 1]
    for bad in (3, 5, 32):
        with pytest.raises(ValueError):
            bench.shard_heads(16, bad)
    d = bench.sharded_line(w, 4, 10, 3, 5.0, 6.0, 111, 222, 100, 5, {"bound": "tensor"}, {}, None)
    assert d["scaling"] == "strong" and d["n_gpus"] == 4 and d["higher_is_better"] is True
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["value"] == round(w.N / 0.005, 1) and d["ms_per_step"] == 5.0
    assert d["e2e"] == {"value": round(w.N / 0.006, 1), "unit": "tokens/s", "h2d_bytes_per_step": 111,
                        "d2h_bytes_per_step": 222}
    assert d["config"]["workload"] == "vggt_100f"
    assert d["config"]["parallelism"].startswith("head-sharded x4 (4 of 16 heads per GPU")
    assert d["collectives_per_step"] == 5
