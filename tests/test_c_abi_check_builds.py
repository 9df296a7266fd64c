"""The C-ABI GPU check under tests/c_abi stays runnable: its input generator
writes every file at the size the C program reads, and the program compiles
and links against the library (CPU only; running it needs a B200)."""

import os
import shutil
import subprocess
import sys

import pytest

from bit_mixture_experts_route_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CDIR = os.path.join(ROOT, "tests", "c_abi")

# file -> bytes, as c_abi_check.cu reads them
SIZES = {
    "mx_W.bin": 3 * 256 * 768 * 4, "mx_P.bin": 6 * 384 * 256, "mx_S.bin": 6 * 384 * 16,
    "mx_X.bin": 83 * 512 * 2, "mx_off.bin": 7 * 4,
    "gt_P.bin": 4 * 2048 * 512, "gt_A.bin": 4 * 2048 * 16 * 4, "gt_G.bin": 58 * 2048 * 4,
    "gt_off.bin": 5 * 4,
    "gt2_P.bin": 4 * 70 * 160, "gt2_A.bin": 4 * 70 * 5 * 4, "gt2_G.bin": 13 * 70 * 4,
    "gt2_off.bin": 5 * 4,
    "sb_gu.bin": 37 * 192 * 4, "sb_dh.bin": 37 * 96 * 4,
    "cb_lg.bin": 33 * 16 * 4, "cb_Yp.bin": 132 * 256 * 4, "cb_dY.bin": 33 * 256 * 4,
    **{f"cb_{n}{r}.bin": 132 * 4 for n in ("idx", "w", "inv") for r in (0, 1)},
}


def test_inputs_have_the_sizes_the_program_reads(tmp_path):
    d = str(tmp_path) + "/"
    subprocess.run([sys.executable, os.path.join(CDIR, "make_inputs.py"), d], check=True,
                   capture_output=True)
    assert sorted(os.listdir(d)) == sorted(SIZES)
    for name, n in SIZES.items():
        assert os.path.getsize(d + name) == n, name


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not installed")
def test_program_compiles_and_links(tmp_path):
    if not os.path.exists(_lib.LIB_PATH):
        from bit_mixture_experts_route_b200 import build
        build.build()
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    subprocess.run(["nvcc", "-O2", "-std=c++17", "-I", os.path.join(ROOT, "include"),
                    os.path.join(CDIR, "c_abi_check.cu"), "-o", exe, "-L", libdir, "-lmoenf4",
                    "-Xlinker", "-rpath", "-Xlinker", libdir], check=True, capture_output=True)
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 2 and "usage" in out.stdout     # argument check, no GPU touched
