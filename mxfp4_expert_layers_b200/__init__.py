"""MXFP4 mixture-of-experts decode layer for NVIDIA B200 (sm_100a).

The compute lives in ``libmxfp4moe.so`` (CUDA kernels behind the C ABI of
``include/mxfp4_moe.h``).  This package is a thin ctypes binding with the
same entry-point names: it converts arguments (torch tensors -> device
pointers, CUDA streams -> handles) and raises :class:`MoEError` on a
non-zero return code.  There is no other implementation behind it: if the
library cannot be loaded every call fails.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxfp4moe.so")

MOE_OK = 0
MOE_ERR_ARG = -1
MOE_ERR_SHAPE = -2
MOE_ERR_ALIGN = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_UNSUPPORTED = -6
MOE_ERR_DEVICE = -7
MOE_GEMV_MAX_TOKENS = 4
MOE_PREFILL_AUTO = 0
MOE_PREFILL_TCGEN05 = 1
MOE_PREFILL_EXACT = 2

EXPORTS = ("moe_create", "moe_route", "moe_forward", "moe_device_error", "moe_last_path",
           "moe_set_prefill_kernel", "moe_lmhead_quantize", "moe_lmhead_logits",
           "moe_destroy", "moe_strerror", "moe_quantize_fp8", "moe_residual_rmsnorm",
           "moe_profile_begin", "moe_profile_end", "moe_pack_weights", "moe_forward_static",
           "moe_forward_static_device_error", "moe_create_ep", "moe_decode_partial", "moe_round_bf16",
           "moe_decode", "moe_stack_create", "moe_stack_decode", "moe_stack_device_error",
           "moe_stack_profile_begin", "moe_stack_profile_end", "moe_stack_destroy")
MOE_PROFILE_KERNELS = 4
KERNEL_NAMES = ("route", "decode", "grouped_gemm", "reserved")


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} ({code})")


class moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("n_shared", ctypes.c_int32)]


class moe_mxfp4_weights(ctypes.Structure):
    _fields_ = [("w13_codes", ctypes.c_void_p), ("w13_scales", ctypes.c_void_p),
                ("w2_codes", ctypes.c_void_p), ("w2_scales", ctypes.c_void_p)]


class moe_weights(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("w13", ctypes.c_void_p), ("w2", ctypes.c_void_p)]


def w13_tile_bytes(hidden: int) -> int:
    return 272 * (hidden // 32)


def w2_tile_bytes(inter: int) -> int:
    return 272 * (inter // 32)


class moe_debug(ctypes.Structure):
    _fields_ = [("xq", ctypes.c_void_p), ("xs", ctypes.c_void_p), ("h", ctypes.c_void_p),
                ("qh", ctypes.c_void_p), ("sh", ctypes.c_void_p)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises OSError if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    L = ctypes.CDLL(path)
    p, i = ctypes.c_void_p, ctypes.c_int
    L.moe_create.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights), i,
                             ctypes.POINTER(p)]
    L.moe_route.argtypes = [p, p, i, p, p, p, p]
    L.moe_forward.argtypes = [p, p, i, p, p, p, ctypes.POINTER(moe_debug), p]
    L.moe_decode.argtypes = [p, p, i, p, p, p, p, ctypes.POINTER(moe_debug), p]
    L.moe_device_error.argtypes = [p, p]
    L.moe_last_path.argtypes = [p]
    L.moe_set_prefill_kernel.argtypes = [p, i]
    L.moe_lmhead_quantize.argtypes = [p, i, i, p, p, p]
    L.moe_lmhead_logits.argtypes = [p, p, i, i, p, i, p, p]
    L.moe_destroy.argtypes = [p]
    L.moe_stack_create.argtypes = [p, i, p]
    L.moe_stack_decode.argtypes = [p, p, p, i, ctypes.c_float, p, p, p, p]
    L.moe_stack_device_error.argtypes = [p, p]
    L.moe_stack_profile_begin.argtypes = [p, i]
    L.moe_stack_profile_end.argtypes = [p, p, p]
    L.moe_stack_destroy.argtypes = [p]
    L.moe_strerror.argtypes = [i]
    L.moe_strerror.restype = ctypes.c_char_p
    L.moe_pack_weights.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_mxfp4_weights), i, i,
                                    p, p, p]
    L.moe_forward_static.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights), p, i, p, p, p, p]
    L.moe_forward_static_device_error.argtypes = [p]
    L.moe_create_ep.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights), i, i, i, i,
                                ctypes.POINTER(p)]
    L.moe_decode_partial.argtypes = [p, p, i, p, p, p, p, p]
    L.moe_round_bf16.argtypes = [p, ctypes.c_size_t, p, p]
    L.moe_profile_begin.argtypes = [p, i]
    L.moe_profile_end.argtypes = [p, p, p]
    L.moe_quantize_fp8.argtypes = [p, i, i, p, p, p]
    L.moe_residual_rmsnorm.argtypes = [p, p, p, i, i, ctypes.c_float, p]
    for name in EXPORTS:
        if name != "moe_strerror":
            getattr(L, name).restype = i
    _lib = L
    return L


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, where: str) -> int:
    if rc != MOE_OK:
        raise MoEError(rc, where)
    return rc


def strerror(code: int) -> str:
    return load().moe_strerror(code).decode()


moe_strerror = strerror


def moe_pack_weights(hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int,
                     src: dict, expert0: int, count: int, w13_packed, w2_packed, stream=None) -> None:
    """Reorder canonical MXFP4 weights (``src``: w13_codes, w13_scales,
    w2_codes, w2_scales tensors) into the packed layout, experts
    ``expert0 .. expert0+count-1``."""
    cfg = moe_config(hidden, inter, n_experts, top_k, n_shared)
    w = moe_mxfp4_weights(*[_ptr(src.get(f)) for f, _ in moe_mxfp4_weights._fields_])
    _check(load().moe_pack_weights(ctypes.byref(cfg), ctypes.byref(w), expert0, count, _ptr(w13_packed),
                                   _ptr(w2_packed), _stream(stream)), "moe_pack_weights")


def moe_create(hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int,
               weights: dict, max_tokens: int) -> int:
    """Returns an opaque handle.  ``weights`` maps the moe_weights field names
    (router_w, router_bias, w13, w2 -- packed) to CUDA tensors
    (``router_bias`` may be None)."""
    cfg = moe_config(hidden, inter, n_experts, top_k, n_shared)
    w = moe_weights(*[_ptr(weights.get(f)) for f, _ in moe_weights._fields_])
    h = ctypes.c_void_p()
    _check(load().moe_create(ctypes.byref(cfg), ctypes.byref(w), max_tokens, ctypes.byref(h)),
           "moe_create")
    return h.value


def moe_route(handle: int, x, T: int, topk_ids, topk_w, expert_counts=None, stream=None) -> None:
    _check(load().moe_route(handle, _ptr(x), T, _ptr(topk_ids), _ptr(topk_w),
                            _ptr(expert_counts), _stream(stream)), "moe_route")


def moe_forward(handle: int, x, T: int, topk_ids, topk_w, y, dbg: dict | None = None,
                stream=None) -> None:
    d = None
    if dbg:
        d = ctypes.byref(moe_debug(*[_ptr(dbg.get(f)) for f, _ in moe_debug._fields_]))
    _check(load().moe_forward(handle, _ptr(x), T, _ptr(topk_ids), _ptr(topk_w), _ptr(y), d,
                              _stream(stream)), "moe_forward")


def moe_decode(handle: int, x, T: int, topk_ids, topk_w, y, expert_counts=None,
               dbg: dict | None = None, stream=None) -> None:
    """Routing and experts of T tokens: one fused launch for T <= MOE_GEMV_MAX_TOKENS,
    else moe_route followed by the many-token kernels; topk_ids, topk_w and
    expert_counts are outputs."""
    d = None
    if dbg:
        d = ctypes.byref(moe_debug(*[_ptr(dbg.get(f)) for f, _ in moe_debug._fields_]))
    _check(load().moe_decode(handle, _ptr(x), T, _ptr(topk_ids), _ptr(topk_w), _ptr(expert_counts),
                             _ptr(y), d, _stream(stream)), "moe_decode")


def moe_forward_static(hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int,
                       weights: dict, x, T: int, topk_ids, topk_w, y, stream=None) -> None:
    """moe_forward for callers that cannot allocate device memory: no handle,
    scratch in a fixed array of the library (see include/mxfp4_moe.h)."""
    cfg = moe_config(hidden, inter, n_experts, top_k, n_shared)
    w = moe_weights(*[_ptr(weights.get(f)) for f, _ in moe_weights._fields_])
    _check(load().moe_forward_static(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), T, _ptr(topk_ids),
                                     _ptr(topk_w), _ptr(y), _stream(stream)), "moe_forward_static")


def moe_create_ep(hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int, weights: dict,
                  max_tokens: int, expert_lo: int, expert_hi: int, with_shared: bool) -> int:
    """A handle for routed experts expert_lo .. expert_hi-1 of a layer split
    over GPUs (``weights``: the full router, and w13 / w2 holding those
    experts' packed tiles, then the shared experts when ``with_shared``)."""
    cfg = moe_config(hidden, inter, n_experts, top_k, n_shared)
    w = moe_weights(*[_ptr(weights.get(f)) for f, _ in moe_weights._fields_])
    h = ctypes.c_void_p()
    _check(load().moe_create_ep(ctypes.byref(cfg), ctypes.byref(w), max_tokens, expert_lo, expert_hi,
                                int(bool(with_shared)), ctypes.byref(h)), "moe_create_ep")
    return h.value


def moe_decode_partial(handle: int, x, T: int, topk_ids, topk_w, y_part, expert_counts=None, stream=None) -> None:
    """Routing of T tokens and this handle's float32 part of y."""
    _check(load().moe_decode_partial(handle, _ptr(x), T, _ptr(topk_ids), _ptr(topk_w), _ptr(expert_counts),
                                     _ptr(y_part), _stream(stream)), "moe_decode_partial")


def moe_round_bf16(v, n: int, out, stream=None) -> None:
    """BF16 bits of n float32 values, round to nearest even."""
    _check(load().moe_round_bf16(_ptr(v), n, _ptr(out), _stream(stream)), "moe_round_bf16")


def moe_forward_static_device_error(stream=None) -> int:
    """Device-side errors of earlier moe_forward_static calls on the current
    device; returns the code (does not raise)."""
    return load().moe_forward_static_device_error(_stream(stream))


def moe_device_error(handle: int, stream=None) -> int:
    """Returns the code (does not raise) so callers can test for errors."""
    return load().moe_device_error(handle, _stream(stream))


def moe_last_path(handle: int) -> int:
    return load().moe_last_path(handle)


def moe_lmhead_quantize(w, V: int, H: int, q, s, stream=None) -> None:
    """FP8 output layer: q [V][H] E4M3 codes and s [V] row scales of the BF16 w."""
    _check(load().moe_lmhead_quantize(_ptr(w), V, H, _ptr(q), _ptr(s), _stream(stream)), "moe_lmhead_quantize")


def moe_lmhead_logits(q, s, V: int, H: int, x, T: int, logits, stream=None) -> None:
    """logits [T][V] float32 of T <= 8 BF16 tokens x [T][H] through the FP8 output layer."""
    _check(load().moe_lmhead_logits(_ptr(q), _ptr(s), V, H, _ptr(x), T, _ptr(logits), _stream(stream)),
           "moe_lmhead_logits")


def moe_set_prefill_kernel(handle: int, kind: int) -> None:
    """Kernels of the many-token path: MOE_PREFILL_AUTO, _TCGEN05 or _EXACT."""
    _check(load().moe_set_prefill_kernel(handle, kind), "moe_set_prefill_kernel")


def moe_destroy(handle: int) -> None:
    _check(load().moe_destroy(handle), "moe_destroy")


def moe_profile_begin(handle: int, max_launches: int) -> None:
    _check(load().moe_profile_begin(handle, max_launches), "moe_profile_begin")


def moe_profile_end(handle: int) -> dict:
    """Returns ``{kernel name: (total ms, launches)}``."""
    ms = (ctypes.c_float * MOE_PROFILE_KERNELS)()
    n = (ctypes.c_int * MOE_PROFILE_KERNELS)()
    _check(load().moe_profile_end(handle, ms, n), "moe_profile_end")
    return {KERNEL_NAMES[i]: (ms[i], n[i]) for i in range(MOE_PROFILE_KERNELS)}


def moe_stack_create(handles) -> int:
    arr = (ctypes.c_void_p * len(handles))(*handles)
    st = ctypes.c_void_p()
    _check(load().moe_stack_create(arr, len(handles), ctypes.byref(st)), "moe_stack_create")
    return st.value


def moe_stack_decode(stack: int, r, x, T: int, eps: float = 1e-6, topk_ids=None, topk_w=None,
                     x_layers=None, stream=None) -> None:
    """All layers of the stack in one launch; r and x are updated in place."""
    _check(load().moe_stack_decode(stack, _ptr(r), _ptr(x), T, eps, _ptr(topk_ids), _ptr(topk_w),
                                   _ptr(x_layers), _stream(stream)), "moe_stack_decode")


def moe_stack_device_error(stack: int, stream=None) -> int:
    return load().moe_stack_device_error(stack, _stream(stream))


def moe_stack_profile_begin(stack: int, max_launches: int) -> None:
    _check(load().moe_stack_profile_begin(stack, max_launches), "moe_stack_profile_begin")


def moe_stack_profile_end(stack: int) -> dict:
    ms = (ctypes.c_float * MOE_PROFILE_KERNELS)()
    n = (ctypes.c_int * MOE_PROFILE_KERNELS)()
    _check(load().moe_stack_profile_end(stack, ms, n), "moe_stack_profile_end")
    return {KERNEL_NAMES[i]: (ms[i], n[i]) for i in range(MOE_PROFILE_KERNELS)}


def moe_stack_destroy(stack: int) -> None:
    _check(load().moe_stack_destroy(stack), "moe_stack_destroy")


def moe_quantize_fp8(v, rows: int, cols: int, q, s, stream=None) -> None:
    _check(load().moe_quantize_fp8(_ptr(v), rows, cols, _ptr(q), _ptr(s), _stream(stream)),
           "moe_quantize_fp8")


def moe_residual_rmsnorm(r, y, x_next, T: int, H: int, eps: float = 1e-6, stream=None) -> None:
    _check(load().moe_residual_rmsnorm(_ptr(r), _ptr(y), _ptr(x_next), T, H, eps, _stream(stream)),
           "moe_residual_rmsnorm")
