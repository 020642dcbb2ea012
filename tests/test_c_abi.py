"""The boundary from plain C: include/httm.h compiles as C99 and C++11 with
-pedantic, and a C program linked against libhttm.so plans a layer, reads
its sizes, shards it and reports errors through the host-only calls (no
device call, so it runs without a GPU)."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

from token_merging_view_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INC = os.path.join(ROOT, "include")

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "httm.h"

int main(void) {
  httm_cfg c;
  memset(&c, 0, sizeof c);
  c.h = 8; c.T = 30; c.P = 1369; c.d_head = 64; c.dtype = HTTM_BF16; c.mode = HTTM_HEADWISE_TEMPORAL;
  c.n_s = 128; c.n_t = 30; c.q_dst_stride = 4; c.kv_dst_stride = 4;
  c.q_merge_pct = 70; c.kv_merge_pct = 50; c.outlier_pct = 10;
  httm_plan_t p = NULL;
  if (httm_plan(&c, &p) != HTTM_OK) return 1;
  httm_plan_info a, b;
  if (httm_get_plan_info(p, &a) != HTTM_OK) return 2;
  if (httm_plan_shard(p, 1, 2) != HTTM_OK) return 3;
  if (httm_get_plan_info(p, &b) != HTTM_OK) return 4;
  if (httm_plan_shard(p, 2, 2) != HTTM_ERR_ARG) return 5;
  c.q_merge_pct = 80;
  httm_plan_t bad = NULL;
  httm_status s = httm_plan(&c, &bad);
  printf("%lld %d %d %lld %lld %zu %d %s\n", (long long)a.N, a.q_slots, a.kv_slots, (long long)a.k_out_max,
         (long long)b.k_out_max, httm_workspace_bytes(p), (int)s, httm_status_str(s));
  httm_plan_destroy(p);
  return bad == NULL ? 0 : 6;
}
"""


@pytest.mark.parametrize("std", ["-std=c99", "-std=c11"])
def test_header_is_plain_c(tmp_path, std):
    src = tmp_path / "t.c"
    src.write_text('#include "httm.h"\nint main(void) { httm_cfg c = {0}; (void)c; return 0; }\n')
    subprocess.run(["gcc", std, "-Wall", "-Wextra", "-pedantic", "-Werror", f"-I{INC}", "-fsyntax-only", str(src)],
                   check=True)


def test_header_is_plain_cxx(tmp_path):
    src = tmp_path / "t.cpp"
    src.write_text('#include "httm.h"\nint main() { return 0; }\n')
    subprocess.run(["g++", "-std=c++11", "-Wall", "-Wextra", "-pedantic", "-Werror", f"-I{INC}", "-fsyntax-only",
                    str(src)], check=True)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_plans_and_shards_a_layer(tmp_path):
    B.load_library()
    lib_dir = os.path.dirname(B.LIB_PATH)
    src = tmp_path / "plan.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "plan"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", f"-I{INC}", str(src), f"-L{lib_dir}", "-lhttm",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    N, q_slots, kv_slots, k1, k2, ws, status, msg = r.stdout.split(maxsplit=7)
    assert int(N) == 30 * 1369
    assert int(k1) == 10 * 8 * 30 * 1369 // 100 and int(k2) == 2 * int(k1)   # the layer's 16 heads after sharding
    assert int(q_slots) > 0 and int(kv_slots) > 0 and int(ws) > 0
    assert int(status) == 3 and "merge ratio" in msg                          # HTTM_ERR_INFEASIBLE_RATIO
