"""The C-ABI check as a collected GPU test: a C++ program that links
libmoenf4.so and calls the entry points directly (no Python binding, no
torch) on inputs the oracle prepared -- the MXFP4 quantize and decode GEMV,
the transposed grouped NF4 GEMM, SwiGLU, combine and routing backward --
then its outputs are compared with the oracle on the host (the MXFP4
quantizer bit for bit, the rest at the parity tolerance)."""

import os
import shutil
import subprocess
import sys

import pytest

from bit_mixture_experts_route_b200 import _lib

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CDIR = os.path.join(ROOT, "tests", "c_abi")


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not installed")
def test_c_program_through_the_abi_matches_the_oracle(tmp_path):
    _lib.load()
    libdir = os.path.dirname(_lib.LIB_PATH)
    d_in, d_out = str(tmp_path / "in") + "/", str(tmp_path / "out") + "/"
    os.makedirs(d_out)
    subprocess.run([sys.executable, os.path.join(CDIR, "make_inputs.py"), d_in], check=True,
                   capture_output=True)
    exe = str(tmp_path / "c_abi_check")
    subprocess.run(["nvcc", "-O2", "-std=c++17", "-I", os.path.join(ROOT, "include"),
                    os.path.join(CDIR, "c_abi_check.cu"), "-o", exe, "-L", libdir, "-lmoenf4",
                    "-Xlinker", "-rpath", "-Xlinker", libdir], check=True, capture_output=True)
    run = subprocess.run([exe, d_in, d_out], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout + run.stderr
    cmp = subprocess.run([sys.executable, os.path.join(CDIR, "compare.py"), d_in, d_out],
                         capture_output=True, text=True, timeout=600)
    assert cmp.returncode == 0 and "ALL OK" in cmp.stdout, cmp.stdout + cmp.stderr
