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


LAYOUT_SRC = r"""
#include <stddef.h>
#include <stdio.h>
#include "moe.h"
#define F(S, m) printf(#m " %zu %zu\n", offsetof(S, m), sizeof(((S *)0)->m))
int main(void) {
    printf("moe_shape_t %zu\n", sizeof(moe_shape_t));
    F(moe_shape_t, T); F(moe_shape_t, d); F(moe_shape_t, E); F(moe_shape_t, k); F(moe_shape_t, I);
    F(moe_shape_t, dtype); F(moe_shape_t, max_sms); F(moe_shape_t, swiglu_limit);
    printf("moe_saved_t %zu\n", sizeof(moe_saved_t));
    F(moe_saved_t, topk_idx); F(moe_saved_t, topk_w); F(moe_saved_t, counts); F(moe_saved_t, offsets);
    F(moe_saved_t, group_start); F(moe_saved_t, tile_expert); F(moe_saved_t, perm); F(moe_saved_t, inv);
    F(moe_saved_t, h); F(moe_saved_t, aw); F(moe_saved_t, xs);
    printf("MOE_SAVED_FIELDS %d\n", MOE_SAVED_FIELDS);
    printf("codes %d %d %d %d %d %d %d %d %d %d\n", MOE_OK, MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_WS, MOE_ERR_ARCH,
           MOE_ERR_LAUNCH, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE, MOE_ERR_UNSUPPORTED, MOE_ERR_SCRATCH_LIMIT);
    printf("dtypes %d %d %d\n", MOE_BF16, MOE_MXFP8, MOE_MXFP8_FWD);
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_python_binding_structs_and_constants_match_the_header(tmp_path):
    from grouped_gemm_route_b200 import moe as M
    src = tmp_path / "layout.c"
    src.write_text(LAYOUT_SRC)
    exe = tmp_path / "layout"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", str(src), "-I", os.path.join(ROOT, "include"),
                        "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines()
    c = {}
    for line in out:
        name, *vals = line.split()
        c[name] = [int(v) for v in vals]
    assert c["moe_shape_t"] == [M.ctypes.sizeof(M.MoeShape)]
    assert c["moe_saved_t"] == [M.ctypes.sizeof(M.MoeSaved)]
    for struct in (M.MoeShape, M.MoeSaved):
        for name, ctype in struct._fields_:
            field = getattr(struct, name)
            assert c[name] == [field.offset, M.ctypes.sizeof(ctype)], name
    assert c["MOE_SAVED_FIELDS"] == [len(M.SAVED_FIELDS)]
    assert [n for n, _ in M.MoeSaved._fields_] == list(M.SAVED_FIELDS)
    assert c["codes"] == [M.MOE_OK, M.MOE_ERR_ARG, M.MOE_ERR_SHAPE, M.MOE_ERR_WS, M.MOE_ERR_ARCH, M.MOE_ERR_LAUNCH,
                          M.MOE_ERR_TIMEOUT, M.MOE_ERR_DEVICE, M.MOE_ERR_UNSUPPORTED, M.MOE_ERR_SCRATCH_LIMIT]
    assert c["dtypes"] == [M.MOE_BF16, M.MOE_MXFP8, M.MOE_MXFP8_FWD]
