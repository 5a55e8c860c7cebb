"""The library used from plain C: tests/c/abi_step.c includes only
include/lmhead.h, links liblmhead.so and the CUDA runtime, runs the five
calls on a small integer-valued problem and checks them against definitions
it writes out itself (exact integer sums for the GEMMs, row maximum, target
logit and zero-sum gradient rows for the cross-entropy).  Compiled with gcc
as C99; no Python or torch in the process."""
import os
import subprocess

import pytest

from lm_head_fp32_b200 import lmhead

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_LIB = "/usr/local/cuda/lib64"


def test_five_calls_from_c(tmp_path):
    lmhead.lib()                                   # the library is built
    exe = tmp_path / "abi_step"
    src = os.path.join(ROOT, "tests", "c", "abi_step.c")
    pkg = os.path.dirname(lmhead.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-O2", "-I", os.path.join(ROOT, "include"), src,
                    "-o", str(exe), "-L", pkg, "-llmhead", "-L", CUDA_LIB, "-lcudart", "-lm",
                    f"-Wl,-rpath,{pkg}", f"-Wl,-rpath,{CUDA_LIB}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert "abi step ok" in out.stdout
