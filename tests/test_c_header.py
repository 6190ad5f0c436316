"""The boundary from C: include/moe.h compiles as C99 (no C++ or CUDA headers
needed) with warnings as errors, and a C program links against the library
and gets the same host-only answers as the Python binding (sizes, launch
counts, status names, argument errors), without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "moe.h"

int main(void)
{
    size_t l1 = 0, l2 = 0, ws = 0, ep = 0, sh = 0;
    int launches = 0;
    if (moe_transformed_weight_bytes(384, 7168, 3072, &l1, &l2) != MOE_OK) return 1;
    if (moe_workspace_bytes(8192, 384, 6, 7168, 3072, &ws) != MOE_OK) return 2;
    if (moe_ep_workspace_bytes(8192, 384, 6, 7168, &ep) != MOE_OK) return 3;
    if (moe_shared_workspace_bytes(8, 7168, 2048, &sh) != MOE_OK) return 4;
    if (moe_forward_kernel_launches(8, 384, 6, 7168, 3072, &launches) != MOE_OK) return 5;
    if (moe_workspace_bytes(8, 384, 6, 7000, 3072, &ws) != MOE_ERR_UNSUPPORTED_SHAPE) return 6;
    printf("%zu %zu %zu %zu %zu %d %s %d\n", l1, l2, ws, ep, sh, launches,
           moe_status_string(MOE_ERR_WORKSPACE_TOO_SMALL), moe_abi_version());
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_links(moelib, tmp_path):
    import moe_expert_layer_08_b200 as m
    src = tmp_path / "use_moe.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_moe"
    libdir = os.path.dirname(m.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lmoe_b200", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True, text=True, cwd=libdir)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    l1, l2, ws, ep, sh, launches, name, abi = r.stdout.split()
    assert (int(l1), int(l2)) == m.transformed_weight_bytes(384, 7168, 3072)
    # the rejected call (H = 7000) left the earlier size in place: a rejected call writes nothing
    assert int(ws) == m.workspace_bytes(8192, 384, 6, 7168, 3072)
    assert int(ep) == m.ep_workspace_bytes(8192, 384, 6, 7168)
    assert int(sh) == m.shared_workspace_bytes(8, 7168, 2048)
    assert int(launches) == m.forward_kernel_launches(8, 384, 6, 7168, 3072)
    assert name == "MOE_ERR_WORKSPACE_TOO_SMALL" and int(abi) == m.abi_version()
