"""The boundary from plain C: include/lbq.h compiles as C99, and a C program linked
against liblbq.so computes layouts and gets argument errors back (host-only calls:
no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_weight_only_ternary_b200")

C_CLIENT = r"""
#include <stdio.h>
#include "lbq.h"

int main(void) {
  int64_t cs = 0, ss = 0;
  size_t cb = 0, sb = 0;
  lbq_status st = lbq_packed_layout(LBQ_TERN5, 5120, 7168, &cs, &ss, &cb, &sb);
  printf("%d %lld %lld %zu %zu\n", (int)st, (long long)cs, (long long)ss, cb, sb);
  st = lbq_packed_layout(LBQ_SIGN1, 17408, 5, &cs, &ss, &cb, &sb);
  printf("%d %lld %lld %zu %zu\n", (int)st, (long long)cs, (long long)ss, cb, sb);
  printf("%d\n", (int)lbq_packed_layout(LBQ_TERN5, 100, 4, &cs, &ss, &cb, &sb));
  printf("%d\n", (int)lbq_gemv(NULL, NULL, NULL, NULL, NULL, 0, NULL));
  printf("%s\n", lbq_status_string(LBQ_ERR_SHAPE));
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib_dir():
    from bit_weight_only_ternary_b200 import build
    build.build()
    return PKG


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_plain_c(tmp_path):
    src = tmp_path / "h.c"
    src.write_text('#include "lbq.h"\nint main(void) { return 0; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only",
                    "-I", os.path.join(ROOT, "include"), str(src)], check=True)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_calls_the_boundary(tmp_path, lib_dir):
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", lib_dir, "-llbq", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    # ternary K = 5120: 40 blocks x 28 bytes = 1120 bytes a row; 7168 rows
    assert out[0].split() == ["0", "1120", "0", str(7168 * 1120), "0"]
    # 1-bit K = 17408: 2176 bytes a row; 136 scales padded to 136; rows padded to 8
    assert out[1].split() == ["0", "2176", "136", str(8 * 2176), str(8 * 136 * 2)]
    assert out[2] == "2"                                       # K not a multiple of 128
    assert out[3] == "1"                                       # null arguments
    assert out[4] == "invalid shape or stride"
