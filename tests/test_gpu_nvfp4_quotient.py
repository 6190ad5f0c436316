"""The NVFP4 requantisation's quotient h / s without a division per value
(moe_common.cuh, nvfp4_quotient: reciprocal, product and one correction from
the exact remainder) against CUDA's correctly rounded division, on the GPU:
bit-identical quotients wherever the helper claims the exact one (2^-60 <=
|h|, |h / s| < 8) and identical E2M1 codes for every finite fp32 h, for all
126 nonzero UE4M3 scale magnitudes.  The probe is built here with nvcc from
tests/cuda/nvfp4_quotient_check.cu."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def probe(tmp_path_factory, moelib):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    out = str(tmp_path_factory.mktemp("quotient") / "libquotient.so")
    src = os.path.join(ROOT, "tests", "cuda", "nvfp4_quotient_check.cu")
    csrc = os.path.join(ROOT, "moe_expert_layer_08_b200", "csrc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                    "-shared", "-I", os.path.join(ROOT, "include"), "-I", csrc, "-o", out, src], check=True)
    return ctypes.CDLL(out)


def test_quotient_exhaustive(probe):
    counts = np.zeros(2, np.uint64)
    assert probe.run_quotient_check(1, ctypes.c_void_p(counts.ctypes.data)) == 0
    assert counts[0] == 0, f"{int(counts[0])} quotients differ from the IEEE division"
    assert counts[1] == 0, f"{int(counts[1])} E2M1 codes differ from those of the IEEE division"
