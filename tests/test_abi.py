"""CPU checks of the C ABI: the library loads, exports every declared entry
point, sizes its buffers, and rejects bad arguments on the host before any GPU
work (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from grouped_gemm_route_b200 import build as B
from grouped_gemm_route_b200 import moe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(M.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_sizes_for_the_30b_shape(lib):
    sh = M.make_shape(16384, 2048, 128, 8, 768)
    sizes, p_cap = M.saved_sizes(sh)
    P = 16384 * 8
    assert p_cap % 128 == 0 and P <= p_cap <= P + 128 * 128
    assert sizes[0] == P * 4 and sizes[8] == p_cap * 2 * 768 * 2 and sizes[9] == p_cap * 768 * 2
    assert sizes[10] == p_cap * 2048 * 2  # the optional sorted copy of x
    f, b = M.workspace_size(sh)
    assert f >= P * 2048 * 2 and b >= p_cap * 2 * 768 * 2


@pytest.mark.parametrize("T,d,E,k,I,dtype,code", [
    (0, 256, 8, 2, 128, 0, M.MOE_ERR_ARG),
    (16, 256, 8, 0, 128, 0, M.MOE_ERR_ARG),
    (16, 256, 8, 9, 128, 0, M.MOE_ERR_ARG),
    (16, 200, 8, 2, 128, 0, M.MOE_ERR_SHAPE),
    (16, 256, 8, 2, 96, 0, M.MOE_ERR_SHAPE),
    (16, 256, 1024, 2, 128, 0, M.MOE_ERR_SHAPE),
    (16, 256, 128, 65, 128, 0, M.MOE_ERR_SHAPE),
    (16, 256, 8, 2, 128, 3, M.MOE_ERR_ARG),
    (16, 256, 8, 2, 128, 7, M.MOE_ERR_ARG),
])
def test_invalid_shapes_are_rejected(lib, T, d, E, k, I, dtype, code):
    sh = M.make_shape(T, d, E, k, I, dtype)
    f = ctypes.c_size_t()
    assert lib.moe_workspace_size(ctypes.byref(sh), ctypes.byref(f), None) == code
    assert lib.moe_fwd(ctypes.byref(sh), None, None, None, None, None, None, None, 0, None) == code


@pytest.mark.parametrize("T,d,E,k,I", [
    (1 << 31, 128, 8, 1, 128),          # T past 2^31
    (1 << 62, 128, 8, 8, 128),          # T * k would overflow 64 bits
    (1 << 30, 1 << 30, 64, 64, 128),    # P_cap * d would overflow 64 bits
    (1 << 20, 2048, 8, 8, 128),         # P_cap * d = 2^34
    (1, (1 << 23) - 128, 512, 1, 128),  # P_cap * d just below 2^31, E * d past it (W_down rows)
])
def test_index_range_limits_are_rejected(lib, T, d, E, k, I):
    sh = M.make_shape(T, d, E, k, I)
    f = ctypes.c_size_t()
    assert lib.moe_workspace_size(ctypes.byref(sh), ctypes.byref(f), None) == M.MOE_ERR_SHAPE
    assert lib.moe_saved_sizes(ctypes.byref(sh), None, None) == M.MOE_ERR_SHAPE


def test_index_range_limit_boundary(lib):
    # P_cap * max(d, 2I) < 2^31 exactly at the edge: d = 2048, so P_cap < 2^20
    d, E, k, I = 2048, 8, 1, 128
    ok_T = (1 << 20) - 128 - 127 * E  # P_cap = T*k + 127*E rounded up to 128 = 2^20 - 128
    sizes, p_cap = M.saved_sizes(M.make_shape(ok_T, d, E, k, I))
    assert p_cap * d < (1 << 31) and p_cap == (1 << 20) - 128
    bad = M.make_shape(ok_T + 1, d, E, k, I)  # P_cap = 2^20
    assert lib.moe_saved_sizes(ctypes.byref(bad), None, None) == M.MOE_ERR_SHAPE


@pytest.mark.parametrize("limit", [-1.0, float("inf"), float("nan")])
def test_invalid_swiglu_limits_are_rejected(lib, limit):
    sh = M.make_shape(256, 256, 8, 2, 128, swiglu_limit=limit)
    f = ctypes.c_size_t()
    assert lib.moe_workspace_size(ctypes.byref(sh), ctypes.byref(f), None) == M.MOE_ERR_ARG
    assert lib.moe_fwd(ctypes.byref(sh), None, None, None, None, None, None, None, 0, None) == M.MOE_ERR_ARG


def test_swiglu_limit_changes_no_size(lib):
    plain = M.make_shape(16384, 2048, 128, 8, 768)
    clamped = M.make_shape(16384, 2048, 128, 8, 768, swiglu_limit=7.0)
    assert M.saved_sizes(plain) == M.saved_sizes(clamped)
    assert M.workspace_size(plain) == M.workspace_size(clamped)
    assert ctypes.sizeof(M.MoeShape) == 40  # int64 T, six int32, float swiglu_limit: 36 bytes, padded to 8


def test_mxfp8_sizes(lib):
    sh = M.make_shape(16384, 2048, 128, 8, 768, M.MOE_MXFP8)
    f_mx, b_mx = M.workspace_size(sh)
    f_bf, b_bf = M.workspace_size(M.make_shape(16384, 2048, 128, 8, 768))
    assert f_mx > f_bf and b_mx > b_bf  # room for E4M3 codes and scales
    assert M.saved_sizes(sh) == M.saved_sizes(M.make_shape(16384, 2048, 128, 8, 768))


def test_mxfp8_forward_bf16_backward_sizes(lib):
    # MXFP8 operands in the forward workspace only; the backward's is the bf16 one
    shape = (16384, 2048, 128, 8, 768)
    f_bf, b_bf = M.workspace_size(M.make_shape(*shape))
    f_mx, b_mx = M.workspace_size(M.make_shape(*shape, M.MOE_MXFP8))
    f_mf, b_mf = M.workspace_size(M.make_shape(*shape, M.MOE_MXFP8_FWD))
    assert f_mf == f_mx and b_mf == b_bf and b_mf < b_mx
    assert M.saved_sizes(M.make_shape(*shape, M.MOE_MXFP8_FWD)) == M.saved_sizes(M.make_shape(*shape))


def test_null_and_misaligned_pointers_are_rejected_before_launch(lib):
    sh = M.make_shape(256, 256, 8, 2, 128)
    saved = M.MoeSaved(*([16] * len(M.SAVED_FIELDS)))
    # null x
    assert lib.moe_fwd(ctypes.byref(sh), None, 16, 16, 16, 16, ctypes.byref(saved), 16, 1 << 40, None) == M.MOE_ERR_ARG
    # misaligned out
    assert lib.moe_fwd(ctypes.byref(sh), 16, 16, 16, 16, 17, ctypes.byref(saved), 16, 1 << 40, None) == M.MOE_ERR_ARG
    # misaligned saved field
    bad = M.MoeSaved(*([16] * (len(M.SAVED_FIELDS) - 1) + [24]))
    assert lib.moe_fwd(ctypes.byref(sh), 16, 16, 16, 16, 16, ctypes.byref(bad), 16, 1 << 40, None) == M.MOE_ERR_ARG
    # the optional sorted x: NULL is accepted (the misaligned field above was it)
    no_xs = M.MoeSaved(*([16] * (len(M.SAVED_FIELDS) - 1) + [None]))
    assert lib.moe_fwd(ctypes.byref(sh), 16, 16, 16, 16, 16, ctypes.byref(no_xs), 16, 64, None) == M.MOE_ERR_WS
    # workspace too small
    assert lib.moe_fwd(ctypes.byref(sh), 16, 16, 16, 16, 16, ctypes.byref(saved), 16, 64, None) == M.MOE_ERR_WS
    assert lib.moe_bwd(ctypes.byref(sh), 16, 16, 16, 16, ctypes.byref(saved), 16, 16, 16, 16, None, 16, 64,
                       None) == M.MOE_ERR_WS


def test_error_strings_and_kernel_names(lib):
    for code in range(-8, 1):
        assert M.error_string(code)
    assert M.error_string(-99) == "unknown error code"
    names = M.kernel_names()
    assert names[0] == "route_topk" and "gemm_gateup_fwd" in names
    assert {"route_bwd", "sort_rows", "mx_quant"} <= set(names)


def test_other_entry_points_reject_bad_arguments_on_the_host(lib):
    sh = M.make_shape(256, 256, 8, 2, 128)
    bad_shape = M.make_shape(256, 200, 8, 2, 128)
    saved = M.MoeSaved(*([16] * len(M.SAVED_FIELDS)))
    misaligned = M.MoeSaved(*([16] * 2 + [20] + [16] * (len(M.SAVED_FIELDS) - 3)))
    # moe_route: shape, pointers, workspace size
    assert lib.moe_route(ctypes.byref(bad_shape), 16, ctypes.byref(saved), 16, 1 << 40, None) == M.MOE_ERR_SHAPE
    assert lib.moe_route(ctypes.byref(sh), None, ctypes.byref(saved), 16, 1 << 40, None) == M.MOE_ERR_ARG
    assert lib.moe_route(ctypes.byref(sh), 16, ctypes.byref(misaligned), 16, 1 << 40, None) == M.MOE_ERR_ARG
    assert lib.moe_route(ctypes.byref(sh), 16, None, 16, 1 << 40, None) == M.MOE_ERR_ARG
    assert lib.moe_route(ctypes.byref(sh), 16, ctypes.byref(saved), 16, 64, None) == M.MOE_ERR_WS
    # moe_recompute
    assert lib.moe_recompute(ctypes.byref(bad_shape), 16, 16, ctypes.byref(saved), 16, 1 << 40,
                             None) == M.MOE_ERR_SHAPE
    assert lib.moe_recompute(ctypes.byref(sh), 16, 24, ctypes.byref(saved), 16, 1 << 40, None) == M.MOE_ERR_ARG
    assert lib.moe_recompute(ctypes.byref(sh), 16, 16, ctypes.byref(saved), 16, 64, None) == M.MOE_ERR_WS
    # moe_route_noalloc: shape, pointers, and the fixed scratch's capacity (ceil(T/64) * E <= 131072)
    assert lib.moe_route_noalloc(ctypes.byref(bad_shape), 16, ctypes.byref(saved), None) == M.MOE_ERR_SHAPE
    assert lib.moe_route_noalloc(ctypes.byref(sh), 16, None, None) == M.MOE_ERR_ARG
    assert lib.moe_route_noalloc(ctypes.byref(sh), 16, ctypes.byref(misaligned), None) == M.MOE_ERR_ARG
    big = M.make_shape(64 * 1025, 128, 128, 1, 128)  # 1025 blocks x 128 experts > 131072
    assert lib.moe_route_noalloc(ctypes.byref(big), 16, ctypes.byref(saved), None) == M.MOE_ERR_SCRATCH_LIMIT
    # status word, self-test
    st = ctypes.c_int()
    assert lib.moe_get_status(None, None, ctypes.byref(st)) == M.MOE_ERR_ARG
    assert lib.moe_get_status(16, None, None) == M.MOE_ERR_ARG
    assert lib.moe_selftest_wait_timeout(None, None) == M.MOE_ERR_ARG
    assert lib.moe_selftest_wait_timeout(20, None) == M.MOE_ERR_ARG


def test_profile_read_without_records_returns_zeros(lib):
    n = len(M.kernel_names())
    assert lib.moe_profile_enable(0) == M.MOE_OK
    ms = (ctypes.c_double * n)(*([7.0] * n))
    cnt = (ctypes.c_int64 * n)(*([7] * n))
    assert lib.moe_profile_read(ms, cnt, n) == M.MOE_OK
    assert list(ms) == [0.0] * n and list(cnt) == [0] * n
    assert lib.moe_kernel_name(-1) is None and lib.moe_kernel_name(n) is None
