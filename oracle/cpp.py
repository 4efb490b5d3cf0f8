"""ctypes wrapper of the C++17 float64 oracle (``oracle/moe_oracle.cpp``) --
TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The same layer as ``oracle/moe.py``, in plain C++ with OpenMP over the rows
of each matrix-vector product.  ``build()`` compiles it with g++ into
``oracle/liboracle.so`` (on first use when the library is missing or older
than its source).  No product code is loaded or called here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
# plain IEEE arithmetic: no contraction into FMAs, no fast-math
CXXFLAGS = ["-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off"]

_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    subprocess.run(["g++", *CXXFLAGS, SRC, "-o", LIB + ".tmp"], check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        _lib.oracle_set_threads.argtypes = [i]
        _lib.oracle_set_threads.restype = i
        _lib.oracle_route.argtypes = [P, i, i, P, P, i, i, P, P, P]
        _lib.oracle_route.restype = None
        _lib.oracle_forward.argtypes = [P, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P, P, P, P]
        _lib.oracle_forward.restype = None
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        _lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        _lib.oracle_bf16_round.argtypes = [ctypes.c_double]
        _lib.oracle_bf16_round.restype = ctypes.c_uint16
    return _lib


def set_threads(n: int) -> int:
    """OpenMP threads of the following calls (n < 1: all processors)."""
    return int(lib().oracle_set_threads(int(n)))


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def route(x_bf16, router_w, bias, top_k):
    """-> (logits float32 [T][E], ids int32 [T][k], w float32 [T][k])."""
    x = np.ascontiguousarray(np.atleast_2d(x_bf16), dtype=np.uint16)
    W = np.ascontiguousarray(router_w, dtype=np.uint16)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    T, H = x.shape
    E = W.shape[0]
    logits = np.empty((T, E), np.float32)
    ids = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float32)
    lib().oracle_route(_p(x), T, H, _p(W), _p(b), E, top_k, _p(logits), _p(ids), _p(w))
    return logits, ids, w


def forward(x_bf16, ids, w, experts: dict, n_experts: int, inter: int, n_shared: int = 1):
    """The experts and the combine; ``experts`` maps expert index -> canonical
    arrays (``w13_codes``, ``w13_scales``, ``w2_codes``, ``w2_scales``).
    Returns the dict of ``oracle.moe.moe_forward`` (y, y64, xq, xs, qh, sh, h)."""
    x = np.ascontiguousarray(np.atleast_2d(x_bf16), dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    T, H = x.shape
    k = ids.shape[1]
    S = k + n_shared
    n = n_experts + n_shared
    arrs = {name: [None] * n for name in ("w13_codes", "w13_scales", "w2_codes", "w2_scales")}
    keep = []
    for e, ex in experts.items():
        for name in arrs:
            a = np.ascontiguousarray(ex[name], dtype=np.uint8)
            keep.append(a)
            arrs[name][e] = a.ctypes.data
    tabs = {name: (ctypes.c_void_p * n)(*[v or 0 for v in arrs[name]]) for name in arrs}
    y = np.empty((T, H), np.uint16)
    xq = np.empty((T, H), np.uint8)
    xs = np.empty((T,), np.float32)
    h = np.empty((T, S, inter), np.float32)
    qh = np.empty((T, S, inter), np.uint8)
    sh = np.empty((T, S), np.float32)
    y64 = np.empty((T, H), np.float64)
    lib().oracle_forward(_p(x), T, H, inter, n_experts, k, n_shared, _p(ids), _p(w),
                         ctypes.cast(tabs["w13_codes"], ctypes.c_void_p), ctypes.cast(tabs["w13_scales"], ctypes.c_void_p),
                         ctypes.cast(tabs["w2_codes"], ctypes.c_void_p), ctypes.cast(tabs["w2_scales"], ctypes.c_void_p),
                         _p(y), _p(xq), _p(xs), _p(h), _p(qh), _p(sh), _p(y64))
    del keep
    return {"y": y, "y64": y64, "xq": xq, "xs": xs, "qh": qh, "sh": sh, "h": h}


def moe_layer(x_bf16, router_w, router_bias, experts: dict, n_experts: int, top_k: int, inter: int,
              n_shared: int = 1):
    """Route, then the experts and the combine (as ``oracle.moe.moe_layer``)."""
    logits, ids, w = route(x_bf16, router_w, router_bias, top_k)
    out = forward(x_bf16, ids, w, experts, n_experts, inter, n_shared)
    out.update(logits=logits, ids=ids, w=w,
               counts=np.bincount(ids.reshape(-1), minlength=n_experts).astype(np.int32))
    return out


def e4m3_encode(v: float) -> int:
    return int(lib().oracle_e4m3_encode(float(v)))


def bf16_round(v: float) -> int:
    return int(lib().oracle_bf16_round(float(v)))
