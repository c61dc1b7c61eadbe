"""CPU check that the boundary is a plain C ABI: a C99 program that includes
include/moe.h, links against libmoe.so and calls its host-only entry points
(sizes and error strings; no device work) builds with gcc and runs."""
import os
import shutil
import subprocess

import pytest

from grouped_gemm_route_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include "moe.h"

int main(void) {
    moe_shape_t s = {0};
    size_t f = 0, b = 0, sizes[MOE_SAVED_FIELDS];
    int64_t p_cap = 0;
    s.T = 16384; s.d = 2048; s.E = 128; s.k = 8; s.I = 768; s.dtype = MOE_BF16;
    if (moe_workspace_size(&s, &f, &b) != MOE_OK) return 1;
    if (moe_saved_sizes(&s, sizes, &p_cap) != MOE_OK) return 2;
    s.d = 200;  /* not a multiple of 128 */
    if (moe_workspace_size(&s, &f, &b) != MOE_ERR_SHAPE) return 3;
    printf("%zu %zu %lld %zu %s\n", f, b, (long long)p_cap, sizes[0], moe_error_string(MOE_ERR_SHAPE));
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_program_builds_links_and_runs(tmp_path):
    lib = B.build()
    libdir = os.path.dirname(lib)
    src = tmp_path / "consumer.c"
    src.write_text(C_SRC)
    exe = tmp_path / "consumer"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", str(src),
                        "-I", os.path.join(ROOT, "include"), "-L", libdir, "-l:" + os.path.basename(lib),
                        "-Wl,-rpath," + libdir, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    f, b, p_cap, idx_bytes, msg = r.stdout.split(" ", 4)
    assert int(f) > 0 and int(b) > 0 and int(p_cap) % 128 == 0
    assert int(idx_bytes) == 16384 * 8 * 4
    assert "unsupported shape" in msg
