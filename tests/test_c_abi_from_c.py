"""The boundary is a C ABI: a C11 program (gcc -std=c11 -pedantic, warnings as
errors) includes include/moe.h, links libmoe.so and calls the host-side entry
points, which return what the Python binding and the oracle return.  No GPU
is touched (size queries, status strings and argument validation only)."""
import os
import shutil
import subprocess

import pytest

import oracle
import mixture_experts_layer_36_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "mixture_experts_layer_36_b200")

PROGRAM = r"""
#include "moe.h"
#include <stdio.h>
int main(void) {
  int bad = moe_route((const void*)0, (const float*)0, (const float*)0, 4, 128, 0, 1,
                      (float*)0, (int32_t*)0, (float*)0, (void*)0, 0, (int32_t*)0, (void*)0);
  printf("%lld %lld %zu %s %d\n", (long long)moe_capacity(4096, 8, 2, 1.25),
         (long long)moe_max_rows(64, 8, 2, 1.25), moe_workspace_size(64, 128, 8, 2, 256, 1.25),
         moe_status_string(MOE_ERR_WORKSPACE), bad);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c11_and_links(tmp_path):
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    cc = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-L", LIBDIR, "-lmoe",
                         f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)],
                        capture_output=True, text=True, timeout=120)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    cap, rows, ws, name, bad = run.stdout.split()
    assert int(cap) == oracle.capacity(4096, 8, 2, 1.25) == moe.moe_capacity(4096, 8, 2, 1.25)
    assert int(rows) == moe.moe_max_rows(64, 8, 2, 1.25)
    assert int(ws) == moe.moe_workspace_size(64, 128, 8, 2, 256, 1.25)
    assert name == "MOE_ERR_WORKSPACE" and int(bad) == 1        # MOE_ERR_INVALID_ARG
