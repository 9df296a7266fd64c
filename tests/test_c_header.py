"""include/moe_nf4.h is a C header: a C99 program that includes it compiles
with gcc (-Wall -Werror), links against libmoenf4.so and makes host-only
calls and calls that validation must reject before touching a GPU."""

import os
import shutil
import subprocess

import pytest

from bit_mixture_experts_route_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "moe_nf4.h"

int main(void) {
  float levels[16];
  size_t ws = 0;
  if (moe_abi_version() != MOE_NF4_ABI_VERSION) return 1;
  if (strcmp(moe_status_string(MOE_ERR_WORKSPACE), "MOE_ERR_WORKSPACE") != 0) return 2;
  if (moe_nf4_levels(levels) != MOE_OK || levels[7] != 0.0f || levels[15] != 1.0f) return 3;
  if (moe_route_permute_workspace_size(4096, 128, 8, &ws) != MOE_OK || ws == 0) return 4;
  /* rejected on the host: K not a multiple of 64, a null weight pointer */
  if (moe_nf4_quantize((const float*)0x70000000, 1, 64, 100, 64, (uint8_t*)0x70000000,
                       (float*)0x70000000, NULL, NULL) != MOE_ERR_INVALID_ARG) return 5;
  if (moe_lora_delta((const void*)0x70000000, 8, (const int32_t*)0x70000000, 2, 64, 256, 16,
                     NULL, (const void*)0x70000000, 1.0f, 8, (float*)0x70000000, NULL,
                     NULL) != MOE_ERR_INVALID_ARG) return 6;
  printf("ok %zu\n", ws);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_compiles_as_c99_and_links(tmp_path):
    if not os.path.exists(_lib.LIB_PATH):
        from bit_mixture_experts_route_b200 import build
        build.build()
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lmoenf4", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.startswith("ok ")
