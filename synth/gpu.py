"""Fill device buffers with the seeded inputs of synth/__init__.py on the GPU
(ctypes over synth/libsynth.so).  Used by the GPU tests and the benchmark to
create full-size weight sets without a host round trip."""
from __future__ import annotations

import ctypes
import os

from . import (LM_HEAD, LM_HEAD_SIGMA, ROUTER_SIGMA, ROUTER_W, SCALE_HI, SCALE_LO, W13_CODES, W13_SCALES,
               W2_CODES, W2_SCALES)

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsynth.so")
        if not os.path.exists(path):
            from .build import build
            build()
        L = ctypes.CDLL(path)
        u64, p, s = ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p
        L.synth_fill_expert_bytes.argtypes = [p, u64, u64, u64, u64, u64, u64, s]
        L.synth_fill_expert_ints.argtypes = [p, u64, u64, u64, u64, u64, u64, ctypes.c_uint32,
                                             ctypes.c_uint32, s]
        L.synth_fill_normals_bf16.argtypes = [p, u64, u64, u64, u64, u64, ctypes.c_double, s]
        for f in (L.synth_fill_expert_bytes, L.synth_fill_expert_ints, L.synth_fill_normals_bf16):
            f.restype = ctypes.c_int
        _LIB = L
    return _LIB


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"synth fill failed ({rc})")


def fill_layer(bufs: dict, seed: int, layer: int, n_experts: int, hidden: int, inter: int,
               n_shared: int = 1, stream: int = 0) -> None:
    """Fill ``bufs`` (torch CUDA tensors: router_w [E][H] int16/uint16,
    w13_codes [E+S][2I][H/2], w13_scales [E+S][2I][H/32], w2_codes [E+S][H][I/2],
    w2_scales [E+S][H][I/32], all uint8) with layer ``(seed, layer)``."""
    L = lib()
    n = n_experts + n_shared
    H, I = hidden, inter
    _check(L.synth_fill_normals_bf16(bufs["router_w"].data_ptr(), seed, layer, ROUTER_W, 0,
                                     n_experts * H, ROUTER_SIGMA, stream))
    _check(L.synth_fill_expert_bytes(bufs["w13_codes"].data_ptr(), seed, layer, W13_CODES, 0, n,
                                     2 * I * H // 2, stream))
    _check(L.synth_fill_expert_ints(bufs["w13_scales"].data_ptr(), seed, layer, W13_SCALES, 0, n,
                                    2 * I * H // 32, SCALE_LO, SCALE_HI, stream))
    _check(L.synth_fill_expert_bytes(bufs["w2_codes"].data_ptr(), seed, layer, W2_CODES, 0, n,
                                     H * I // 2, stream))
    _check(L.synth_fill_expert_ints(bufs["w2_scales"].data_ptr(), seed, layer, W2_SCALES, 0, n,
                                    H * I // 32, SCALE_LO, SCALE_HI, stream))


def fill_lmhead(buf, seed: int, vocab: int, hidden: int, stream: int = 0) -> None:
    """Fill ``buf`` (torch CUDA int16/uint16 [vocab][hidden]) with the output
    layer of ``synth.lmhead_weight``."""
    _check(lib().synth_fill_normals_bf16(buf.data_ptr(), seed, 0, LM_HEAD, 0, vocab * hidden, LM_HEAD_SIGMA,
                                         stream))
