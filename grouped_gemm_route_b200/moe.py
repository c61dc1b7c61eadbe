"""Python binding of libmoe.so (the fused MoE layer's C ABI, include/moe.h).

Argument marshalling only: every step of routing, dispatch, the expert GEMMs,
SwiGLU, the combine and the backward runs inside the CUDA library.  PyTorch is
used here only to allocate device memory and to name the current stream.  If
the library is missing or no sm_100 GPU is present the calls raise; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_BF16, MOE_MXFP8 = 0, 1
MOE_MXFP8_FWD = 2  # MXFP8 forward GEMMs, bf16 backward GEMMs
MOE_OK = 0
MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_WS, MOE_ERR_ARCH = -1, -2, -3, -4
MOE_ERR_LAUNCH, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE, MOE_ERR_UNSUPPORTED = -5, -6, -7, -8
MOE_ERR_SCRATCH_LIMIT = -9

SAVED_FIELDS = ("topk_idx", "topk_w", "counts", "offsets", "group_start", "tile_expert", "perm", "inv", "h", "aw",
                "xs")
EXPORTS = ("moe_saved_sizes", "moe_workspace_size", "moe_route", "moe_fwd", "moe_bwd", "moe_get_status",
           "moe_error_string", "moe_profile_enable", "moe_profile_read", "moe_kernel_name",
           "moe_selftest_wait_timeout", "moe_route_noalloc", "moe_recompute", "moe_ep_expert_layout",
           "moe_ep_dispatch", "moe_expert_fwd", "moe_expert_bwd", "moe_ep_combine", "moe_ep_backward_finish")


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("dtype", ctypes.c_int32), ("max_sms", ctypes.c_int32),
                ("swiglu_limit", ctypes.c_float)]


class MoeSaved(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in SAVED_FIELDS]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {code} ({error_string(code)})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so once (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with grouped_gemm_route_b200.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.POINTER(MoeShape)
    L.moe_saved_sizes.argtypes = [S, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_int64)]
    L.moe_workspace_size.argtypes = [S, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
    L.moe_route.argtypes = [S, P, ctypes.POINTER(MoeSaved), P, ctypes.c_size_t, P]
    L.moe_fwd.argtypes = [S, P, P, P, P, P, ctypes.POINTER(MoeSaved), P, ctypes.c_size_t, P]
    L.moe_bwd.argtypes = [S, P, P, P, P, ctypes.POINTER(MoeSaved), P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_get_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int)]
    L.moe_error_string.argtypes = [ctypes.c_int]
    L.moe_error_string.restype = ctypes.c_char_p
    L.moe_profile_enable.argtypes = [ctypes.c_int]
    L.moe_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), ctypes.c_int]
    L.moe_route_noalloc.argtypes = [S, P, ctypes.POINTER(MoeSaved), P]
    L.moe_recompute.argtypes = [S, P, P, ctypes.POINTER(MoeSaved), P, ctypes.c_size_t, P]
    L.moe_recompute.restype = ctypes.c_int
    L.moe_route_noalloc.restype = ctypes.c_int
    L.moe_selftest_wait_timeout.argtypes = [P, P]
    L.moe_selftest_wait_timeout.restype = ctypes.c_int
    L.moe_kernel_name.argtypes = [ctypes.c_int]
    L.moe_kernel_name.restype = ctypes.c_char_p
    i64p = ctypes.POINTER(ctypes.c_int64)
    L.moe_ep_expert_layout.argtypes = [ctypes.c_int, ctypes.c_int, P, i64p, i64p, i64p, i64p]
    L.moe_ep_dispatch.argtypes = [S, P, ctypes.POINTER(MoeSaved), P, P, P]
    L.moe_expert_fwd.argtypes = [S, ctypes.c_int, P, P, P, P, P, ctypes.POINTER(MoeSaved), P, ctypes.c_size_t, P]
    L.moe_expert_bwd.argtypes = [S, P, P, P, P, ctypes.POINTER(MoeSaved), P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_ep_combine.argtypes = [S, ctypes.POINTER(MoeSaved), P, P, P]
    L.moe_ep_backward_finish.argtypes = [S, ctypes.POINTER(MoeSaved), P, P, P, P, P, P]
    for name in ("moe_ep_expert_layout", "moe_ep_dispatch", "moe_expert_fwd", "moe_expert_bwd", "moe_ep_combine",
                 "moe_ep_backward_finish"):
        getattr(L, name).restype = ctypes.c_int
    for name in ("moe_saved_sizes", "moe_workspace_size", "moe_route", "moe_fwd", "moe_bwd", "moe_get_status",
                 "moe_profile_enable", "moe_profile_read"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def error_string(code: int) -> str:
    try:
        return lib().moe_error_string(int(code)).decode()
    except Exception:  # library not loadable: still give a readable message
        return "unknown"


def _check(rc: int, where: str):
    if rc != MOE_OK:
        raise MoeError(rc, where)


def make_shape(T, d, E, k, I, dtype=MOE_BF16, max_sms=0, swiglu_limit=0.0) -> MoeShape:
    """swiglu_limit: 0 for SwiGLU, L > 0 for the clamped SwiGLU (see include/moe.h)."""
    return MoeShape(int(T), int(d), int(E), int(k), int(I), int(dtype), int(max_sms), float(swiglu_limit))


def saved_sizes(shape: MoeShape):
    sizes = (ctypes.c_size_t * len(SAVED_FIELDS))()
    p_cap = ctypes.c_int64()
    _check(lib().moe_saved_sizes(ctypes.byref(shape), sizes, ctypes.byref(p_cap)), "moe_saved_sizes")
    return [int(s) for s in sizes], int(p_cap.value)


def workspace_size(shape: MoeShape):
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().moe_workspace_size(ctypes.byref(shape), ctypes.byref(f), ctypes.byref(b)), "moe_workspace_size")
    return int(f.value), int(b.value)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, t):
    """The stream to launch on: the given one, else the current stream of t's device."""
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(stream.cuda_stream)


def _on(t):
    """The library launches on the current CUDA device: make it t's device for the call."""
    return torch.cuda.device(t.device)


def saved_struct(saved: dict) -> MoeSaved:
    return MoeSaved(*[saved[n].data_ptr() if saved.get(n) is not None else None for n in SAVED_FIELDS])


def route(shape, logits, saved: dict, ws, stream=None):
    st = saved_struct(saved)
    with _on(logits):
        _check(lib().moe_route(ctypes.byref(shape), _ptr(logits), ctypes.byref(st), _ptr(ws), ws.numel(),
                               _stream(stream, logits)), "moe_route")


def route_noalloc(shape, logits, saved: dict, stream=None):
    """Routing for callers that cannot allocate device memory: same results as
    route(), with the kernels' scratch in a fixed array inside the library
    instead of a caller workspace (see moe_route_noalloc in include/moe.h)."""
    st = saved_struct(saved)
    with _on(logits):
        _check(lib().moe_route_noalloc(ctypes.byref(shape), _ptr(logits), ctypes.byref(st),
                                       _stream(stream, logits)), "moe_route_noalloc")


def fwd(shape, x, logits, wgu, wd, out, saved: dict, ws, stream=None):
    st = saved_struct(saved)
    with _on(x):
        _check(lib().moe_fwd(ctypes.byref(shape), _ptr(x), _ptr(logits), _ptr(wgu), _ptr(wd), _ptr(out),
                             ctypes.byref(st), _ptr(ws), ws.numel(), _stream(stream, x)), "moe_fwd")


def bwd(shape, gout, x, wgu, wd, saved: dict, dx, dwgu, dwd, dscore, dlogits, ws, stream=None):
    st = saved_struct(saved)
    with _on(gout):
        _check(lib().moe_bwd(ctypes.byref(shape), _ptr(gout), _ptr(x), _ptr(wgu), _ptr(wd), ctypes.byref(st),
                             _ptr(dx), _ptr(dwgu), _ptr(dwd), _ptr(dscore), _ptr(dlogits), _ptr(ws), ws.numel(),
                             _stream(stream, gout)), "moe_bwd")


def recompute(shape, x, wgu, saved: dict, ws, stream=None):
    """Rewrite saved h and aw from x and W_gate_up for the routing in `saved`
    (the gate/up GEMM again, for a backward whose forward dropped them)."""
    st = saved_struct(saved)
    with _on(x):
        _check(lib().moe_recompute(ctypes.byref(shape), _ptr(x), _ptr(wgu), ctypes.byref(st), _ptr(ws),
                                   ws.numel(), _stream(stream, x)), "moe_recompute")


# ----------------------------------------------------------------------------
# expert parallelism (see include/moe.h): the device steps; grouped_gemm_route_b200.ep
# runs the exchanges between them
# ----------------------------------------------------------------------------
def ep_expert_layout(G: int, E_loc: int, recv_counts):
    """Host only.  recv_counts: int array-like [G, E_loc] (rows of local expert e
    from source s).  Returns (row_off [G, E_loc], cmp_off [G, E_loc], rows,
    padded_rows) as Python ints: where each (source, expert) segment lands in
    the padded local layout and in compact order."""
    flat = [int(c) for c in torch.as_tensor(recv_counts).reshape(-1).tolist()]
    if len(flat) != G * E_loc:
        raise ValueError("recv_counts must hold G * E_loc counts")
    rc = (ctypes.c_int32 * len(flat))(*flat)
    row_off = (ctypes.c_int64 * len(flat))()
    cmp_off = (ctypes.c_int64 * len(flat))()
    rows, padded = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().moe_ep_expert_layout(G, E_loc, rc, row_off, cmp_off, ctypes.byref(rows), ctypes.byref(padded)),
           "moe_ep_expert_layout")
    ro = [[row_off[s * E_loc + e] for e in range(E_loc)] for s in range(G)]
    co = [[cmp_off[s * E_loc + e] for e in range(E_loc)] for s in range(G)]
    return ro, co, int(rows.value), int(padded.value)


def ep_dispatch(shape, src, saved: dict, dst, w_rows=None, stream=None):
    st = saved_struct(saved)
    with _on(src):
        _check(lib().moe_ep_dispatch(ctypes.byref(shape), _ptr(src), ctypes.byref(st), _ptr(dst), _ptr(w_rows),
                                     _stream(stream, src)), "moe_ep_dispatch")


def expert_fwd(shape, G, recv_counts, xr, wgu, wd, y_rows, saved: dict, ws, stream=None):
    st = saved_struct(saved)
    with _on(xr):
        _check(lib().moe_expert_fwd(ctypes.byref(shape), int(G), _ptr(recv_counts), _ptr(xr), _ptr(wgu), _ptr(wd),
                                    _ptr(y_rows), ctypes.byref(st), _ptr(ws), ws.numel(), _stream(stream, xr)),
               "moe_expert_fwd")


def expert_bwd(shape, gr, xr, wgu, wd, saved: dict, dx_rows, dwgu, dwd, ds_rows, ws, stream=None):
    st = saved_struct(saved)
    with _on(gr):
        _check(lib().moe_expert_bwd(ctypes.byref(shape), _ptr(gr), _ptr(xr), _ptr(wgu), _ptr(wd), ctypes.byref(st),
                                    _ptr(dx_rows), _ptr(dwgu), _ptr(dwd), _ptr(ds_rows), _ptr(ws), ws.numel(),
                                    _stream(stream, gr)), "moe_expert_bwd")


def ep_combine(shape, saved: dict, rows, out, stream=None):
    st = saved_struct(saved)
    with _on(rows):
        _check(lib().moe_ep_combine(ctypes.byref(shape), ctypes.byref(st), _ptr(rows), _ptr(out),
                                    _stream(stream, rows)), "moe_ep_combine")


def ep_backward_finish(shape, saved: dict, dx_rows, ds_rows, dx, dscore, dlogits, stream=None):
    st = saved_struct(saved)
    with _on(dx_rows):
        _check(lib().moe_ep_backward_finish(ctypes.byref(shape), ctypes.byref(st), _ptr(dx_rows), _ptr(ds_rows),
                                            _ptr(dx), _ptr(dscore), _ptr(dlogits), _stream(stream, dx_rows)),
               "moe_ep_backward_finish")


def get_status(ws, stream=None) -> int:
    s = ctypes.c_int()
    with _on(ws):
        _check(lib().moe_get_status(_ptr(ws), _stream(stream, ws), ctypes.byref(s)), "moe_get_status")
    return int(s.value)


def selftest_wait_timeout(ws, stream=None):
    """Launch the kernel whose bounded wait must expire (see include/moe.h)."""
    with _on(ws):
        _check(lib().moe_selftest_wait_timeout(_ptr(ws), _stream(stream, ws)), "moe_selftest_wait_timeout")


def kernel_names():
    names, i = [], 0
    while True:
        n = lib().moe_kernel_name(i)
        if n is None:
            return names
        names.append(n.decode())
        i += 1


def profile_enable(on: bool):
    _check(lib().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def profile_read():
    """{kernel name: (summed ms, launches)} since the last read."""
    names = kernel_names()
    ms = (ctypes.c_double * len(names))()
    n = (ctypes.c_int64 * len(names))()
    _check(lib().moe_profile_read(ms, n, len(names)), "moe_profile_read")
    return {name: (ms[i], int(n[i])) for i, name in enumerate(names)}


# ----------------------------------------------------------------------------
# buffer allocation for one layer (torch allocates, the library computes)
# ----------------------------------------------------------------------------
_SAVED_DTYPES = dict(topk_idx=torch.int32, topk_w=torch.float32, counts=torch.int32, offsets=torch.int32,
                     group_start=torch.int32, tile_expert=torch.int32, perm=torch.int32, inv=torch.int32,
                     h=torch.bfloat16, aw=torch.bfloat16, xs=torch.bfloat16)


def alloc_saved(shape: MoeShape, device, keep_sorted_x: bool = True) -> dict:
    """Every saved buffer; keep_sorted_x=False leaves the optional xs out (None):
    the backward then sorts x itself, 2 * P_cap * d bytes less between the passes."""
    sizes, p_cap = saved_sizes(shape)
    T, E, k, I = shape.T, shape.E, shape.k, shape.I
    shapes = dict(topk_idx=(T, k), topk_w=(T, k), counts=(E,), offsets=(E + 1,), group_start=(E + 1,),
                  tile_expert=(p_cap // 128,), perm=(p_cap,), inv=(T, k), h=(p_cap, 2 * I), aw=(p_cap, I),
                  xs=(p_cap, shape.d))
    out = {}
    for name, nbytes in zip(SAVED_FIELDS, sizes):
        if name == "xs" and not keep_sorted_x:
            out[name] = None
            continue
        t = torch.empty(shapes[name], dtype=_SAVED_DTYPES[name], device=device)
        assert t.numel() * t.element_size() == nbytes, name
        out[name] = t
    return out


def alloc_saved_routing(shape: MoeShape, device) -> dict:
    """Saved buffers for moe_route alone: the routing fields at full size,
    16-byte placeholders for h and aw, which routing does not touch, and no xs."""
    sizes, p_cap = saved_sizes(shape)
    T, E, k = shape.T, shape.E, shape.k
    shapes = dict(topk_idx=(T, k), topk_w=(T, k), counts=(E,), offsets=(E + 1,), group_start=(E + 1,),
                  tile_expert=(p_cap // 128,), perm=(p_cap,), inv=(T, k), h=(8,), aw=(8,))
    out = {name: torch.empty(shapes[name], dtype=_SAVED_DTYPES[name], device=device) for name in SAVED_FIELDS[:-1]}
    out["xs"] = None
    return out


def alloc_workspace(shape: MoeShape, device) -> torch.Tensor:
    f, b = workspace_size(shape)
    return torch.empty(max(f, b), dtype=torch.uint8, device=device)


@dataclass
class MoELayer:
    """One fused MoE layer's buffers on a device; forward/backward call the C ABI."""
    T: int
    d: int
    E: int
    k: int
    I: int
    device: str = "cuda"
    max_sms: int = 0
    dtype: int = MOE_BF16  # MOE_BF16, MOE_MXFP8 or MOE_MXFP8_FWD (GEMM operand precision)
    swiglu_limit: float = 0.0  # 0: SwiGLU; L > 0: clamped SwiGLU
    keep_sorted_x: bool = True  # keep x's sorted copy from forward to backward (saves re-sorting it)

    def __post_init__(self):
        if not torch.cuda.is_available():
            raise RuntimeError("the fused MoE layer needs a CUDA device (sm_100)")
        self.shape = make_shape(self.T, self.d, self.E, self.k, self.I, self.dtype, self.max_sms, self.swiglu_limit)
        self.saved = alloc_saved(self.shape, self.device, self.keep_sorted_x)
        self.ws = alloc_workspace(self.shape, self.device)
        dev = self.device
        self.out = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=dev)
        self.dx = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=dev)
        self.dwgu = torch.empty(self.E, 2 * self.I, self.d, dtype=torch.bfloat16, device=dev)
        self.dwd = torch.empty(self.E, self.d, self.I, dtype=torch.bfloat16, device=dev)
        self.dscore = torch.empty(self.T, self.k, dtype=torch.float32, device=dev)
        self.dlogits = torch.empty(self.T, self.E, dtype=torch.float32, device=dev)

    def forward(self, x, logits, wgu, wd, stream=None):
        fwd(self.shape, x, logits, wgu, wd, self.out, self.saved, self.ws, stream)
        return self.out

    def backward(self, gout, x, wgu, wd, with_dlogits=True, stream=None):
        bwd(self.shape, gout, x, wgu, wd, self.saved, self.dx, self.dwgu, self.dwd, self.dscore,
            self.dlogits if with_dlogits else None, self.ws, stream)
        return dict(dx=self.dx, dwgu=self.dwgu, dwd=self.dwd, dscore=self.dscore,
                    dlogits=self.dlogits if with_dlogits else None)

    def status(self, stream=None) -> int:
        return get_status(self.ws, stream)
