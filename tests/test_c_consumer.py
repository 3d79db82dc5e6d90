"""The boundary is a C ABI: a plain C99 program, compiled with gcc -pedantic
against include/nvq.h and linked with libnvq.so, calls the host-side entry
points and gets the documented answers -- no Python, no torch, no GPU."""
import os
import shutil
import subprocess

import pytest

from phase_disaggregated_quantized_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdint.h>
#include <stdio.h>
#include "nvq.h"

int main(void) {
  void* fake = (void*)(uintptr_t)0x7F0000000000ull;    /* never dereferenced: validation fails first */
  void* odd = (void*)(uintptr_t)0x7F0000000008ull;
  printf("abi %d\n", nvq_abi_version());
  printf("status %s\n", nvq_status_string(NVQ_ERR_WORKSPACE));
  printf("scales_bytes %zu\n", nvfp4_scales_bytes(130, 512));
  printf("scale_offset %lld %lld\n", (long long)nvfp4_scale_offset(129, 5, 130, 512),
         (long long)nvfp4_scale_offset(130, 0, 130, 512));
  printf("ws %zu %zu\n", nvq_workspace_bytes(NVQ_OP_NVFP4_GEMM, 8192, 4096, 4096),
         nvq_workspace_bytes(NVQ_OP_W4A16_GEMM, 16, 4096, 4096));
  printf("quantize_k %d\n", (int)nvfp4_quantize(fake, 4, 100, NULL, fake, fake, fake, NULL, 0, NULL));
  printf("gemm_align %d\n", (int)nvfp4_gemm_w4a4(fake, fake, fake, fake, fake, fake, odd, 128, 512, 512, NULL));
  printf("w4a16_n %d\n", (int)w4a16_gemm(fake, fake, fake, fake, 4, 48, 128, NULL, 0, NULL));
  printf("detail %s\n", nvq_last_error_detail());
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_uses_the_library(tmp_path):
    lib = build_lib.build()
    src = tmp_path / "consumer.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-o", str(exe), str(src), "-L", libdir, "-lnvq", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    got = dict(line.split(" ", 1) for line in out)
    assert got["abi"] == "1"
    assert got["status"] == "NVQ_ERR_WORKSPACE"
    assert got["scales_bytes"] == str(256 * 32)
    assert got["scale_offset"] == "4625 -1"         # (129 // 128) * 8 + 5 // 4 = atom 9; 9*512 + 16*1 + 0 + 1
    assert got["ws"] == "0 0"
    assert got["quantize_k"] == "2"                  # NVQ_ERR_UNSUPPORTED_SHAPE: K % 64
    assert got["gemm_align"] == "3"                  # NVQ_ERR_MISALIGNED
    assert got["w4a16_n"] == "2"                     # N % 32
    assert "w4a16" in got["detail"]
