"""The boundary from C: include/moe.h compiles as strict C99 (no C++ or CUDA
types leak into it), a C program links against libmoe.so, and the host-side
entry points answer from C as they do through the Python binding (no GPU:
nothing here launches a kernel).

The capacity case is the worked example of "负载均衡策略：MoE训练稳定性保障",
section "专家容量裁剪": 1024 tokens, 8 experts, capacity factor 1.25, one
expert per token -> 160."""
import os
import shutil
import subprocess

import pytest

moe = pytest.importorskip("expert_router_gemm_b200.moe",
                          reason="libmoe.so not built (python -m expert_router_gemm_b200.build)")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moe.h"

int main(void) {
  moe_config_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.T = 1024; cfg.d = 128; cfg.N = 8; cfg.k = 1; cfg.f = 128;
  cfg.capacity_factor = 1.25; cfg.capacity = -1; cfg.act_dtype = MOE_BF16;
  int32_t cap = -1;
  moe_status_t s = moe_capacity(&cfg, &cap);
  size_t layer = 0, op = 0;
  int64_t rows = 0;
  moe_status_t w = moe_workspace_size(&cfg, &layer, &op, &rows);
  int32_t cap0 = -1;
  cfg.N = 0;                                     /* no experts */
  moe_status_t bad = moe_capacity(&cfg, &cap0);
  size_t split = 0;
  moe_status_t sp = moe_router_split_bytes(4096, 128, &split);
  printf("%d %d %d %zu %zu %lld %d %d %zu %s\n", (int)s, (int)cap, (int)w, layer, op, (long long)rows,
         (int)bad, (int)sp, split, moe_status_string(MOE_ERR_MISALIGNED));
  return 0;
}
"""


def test_header_compiles_as_c99_and_links():
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(moe.LIB_PATH)
    build = os.path.join(ROOT, "_build")
    os.makedirs(build, exist_ok=True)
    src = os.path.join(build, "moe_c_abi_check.c")
    exe = os.path.join(build, "moe_c_abi_check")
    with open(src, "w") as fh:
        fh.write(_PROGRAM)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), src, "-o", exe,
                        "-L", lib_dir, "-lmoe", f"-Wl,-rpath,{lib_dir}"],
                       capture_output=True, text=True)
    if r.returncode != 0 and "cannot find -lmoe" in r.stderr:
        # the library is named libmoe.so: link it by path
        r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                            "-I", os.path.join(ROOT, "include"), src, "-o", exe, moe.LIB_PATH,
                            f"-Wl,-rpath,{lib_dir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    f = out.stdout.split()
    cfg = moe.make_config(T=1024, d=128, N=8, k=1, f=128, capacity_factor=1.25, dtype="bf16")
    layer, op, rows = moe.moe_workspace_size(cfg)
    assert int(f[0]) == moe.MOE_OK and int(f[1]) == 160
    assert int(f[2]) == moe.MOE_OK and (int(f[3]), int(f[4]), int(f[5])) == (layer, op, rows)
    assert int(f[6]) == moe.MOE_ERR_INVALID_ARG
    assert int(f[7]) == moe.MOE_OK and int(f[8]) == moe.moe_router_split_bytes(4096, 128)
    assert " ".join(f[9:]) == moe.moe_status_string(moe.MOE_ERR_MISALIGNED)
