"""The boundary is a C ABI: a C99 program (gcc -std=c99 -pedantic, warnings as errors)
includes include/fused_moe.h, links libfused_moe.so and calls the host-only entry points
without a GPU."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "mixture_experts_layer_26_b200")

PROGRAM = r"""
#include "fused_moe.h"
#include <stdio.h>
int main(void) {
  fmoe_routing r = {FMOE_ROUTE_SIGMOID_GROUPED, 8, 4, 2.5f, NULL, 1};
  fmoe_dims d = {16, 7168, 2048, 256, 8, FMOE_FP8_E4M3, FMOE_VARIANT_AUTO, &r};
  fmoe_dims bad = d;
  fmoe_rope_dims rd = {8, 4, 128, 96, 0, 64};   /* rot_dim 96: not a power of two */
  bad.top_k = 0;
  printf("%d %d %d %d %d\n", fused_moe_abi_version(), fused_moe_workspace_size(&d) > 0,
         fused_moe_launches_per_call(&d), (int)fused_moe_workspace_size(&bad),
         (int)fused_inv_rope_fp8_quant_per_head(&rd, NULL, NULL, NULL, NULL, NULL, NULL, NULL));
  printf("%s\n", fused_moe_status_string(FMOE_ERR_TIMEOUT));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_is_c99_and_host_calls_work(tmp_path):
    if not os.path.exists(os.path.join(LIBDIR, "libfused_moe.so")):
        pytest.skip("libfused_moe.so not built")
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-L", LIBDIR, "-lfused_moe",
                    f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    abi, ws_ok, launches, bad_ws, rope = (int(v) for v in out[0].split())
    assert abi == 4 and ws_ok == 1 and bad_ws == 0
    # router (+ permutation and plan: 144 rows), gather (144 x 7168 x 2 B > 128 KB), gemm1,
    # finalize1, quant_h, gemm2, combine of the split-K partials
    assert launches == 7
    assert rope == 1              # FMOE_ERR_INVALID_ARG, before any CUDA call
    assert out[1].strip() != ""
