"""ctypes binding of the C++ fp64 oracle (moe_oracle.cpp).

TEST INFRASTRUCTURE ONLY: used by tests/, __graft_entry__.smoke() and
bench.py's CPU baseline / reference arm, never by the product path.  The
library is compiled here with g++ (no fast-math, no FMA contraction); it shares
no code with the CUDA library.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "libmoe_oracle.so")
STAMP = LIB + ".src"

_lib = None


def _src_hash() -> str:
    with open(SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def build(force: bool = False) -> str:
    """Compile the oracle library if it is missing or older than its source."""
    h = _src_hash()
    if not force and os.path.exists(LIB) and os.path.exists(STAMP) and open(STAMP).read().strip() == h:
        return LIB
    tmp = LIB + ".tmp"
    subprocess.run(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                    "-pthread", SRC, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(h + "\n")
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        L.moe_oracle_route.argtypes = [i64, i32, i32, p, p, p]
        L.moe_oracle_dispatch.argtypes = [i64, i32, i32, p, p, p, p, p]
        f64 = ctypes.c_double
        L.moe_oracle_forward.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, p, p, p, p, i32, f64]
        L.moe_oracle_backward.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, p, p, p, p, p, i32, f64]
        L.moe_oracle_hardware_threads.restype = ctypes.c_uint
        for f in (L.moe_oracle_route, L.moe_oracle_dispatch, L.moe_oracle_forward, L.moe_oracle_backward):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def hardware_threads() -> int:
    return int(lib().moe_oracle_hardware_threads())


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ok(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected its arguments ({rc})")


def route(logits, k):
    lg = _f32(logits)
    T, E = lg.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _ok(lib().moe_oracle_route(T, E, k, _p(lg), _p(idx), _p(w)), "route")
    return idx, w


def dispatch(idx, E):
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    _ok(lib().moe_oracle_dispatch(T, E, k, _p(idx), _p(counts), _p(offsets), _p(perm), _p(inv)), "dispatch")
    return counts, offsets, perm, inv.reshape(T, k)


def forward(x, logits, wgu, wd, k, nthreads: int = 1, keep_intermediates: bool = True, limit: float = 0.0):
    x, lg, wgu, wd = _f64(x), _f32(logits), _f64(wgu), _f64(wd)
    T, d = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    out = np.empty((T, d))
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k))
    h = np.empty((T * k, twoI)) if keep_intermediates else None
    a = np.empty((T * k, I)) if keep_intermediates else None
    rc = lib().moe_oracle_forward(T, d, E, k, I, _p(x), _p(lg), _p(wgu), _p(wd), _p(out), _p(idx), _p(w),
                                  _p(h) if h is not None else None, _p(a) if a is not None else None, nthreads,
                                  float(limit))
    _ok(rc, "forward")
    return dict(out=out, idx=idx, w=w, h=h, a=a)


def backward(x, logits, wgu, wd, k, gout, nthreads: int = 1, limit: float = 0.0):
    x, lg, wgu, wd, gout = _f64(x), _f32(logits), _f64(wgu), _f64(wd), _f64(gout)
    T, d = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    dx = np.empty((T, d))
    dwgu = np.empty_like(wgu)
    dwd = np.empty_like(wd)
    dscore = np.empty((T, k))
    dlogits = np.empty((T, E))
    rc = lib().moe_oracle_backward(T, d, E, k, I, _p(x), _p(lg), _p(wgu), _p(wd), _p(gout), _p(dx), _p(dwgu),
                                   _p(dwd), _p(dscore), _p(dlogits), nthreads, float(limit))
    _ok(rc, "backward")
    return dict(dx=dx, dwgu=dwgu, dwd=dwd, dscore=dscore, dlogits=dlogits)
