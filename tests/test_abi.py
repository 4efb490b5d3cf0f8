"""The C-ABI library builds, loads and exports every symbol declared in
include/*.h; host-side argument validation needs no GPU."""
import ctypes
import glob
import os
import re

import pytest

import mxfp4_expert_layers_b200 as moe
from mxfp4_expert_layers_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(path).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    B.build()
    lib = ctypes.CDLL(B.LIB)
    declared = _declared()
    assert {"moe_create", "moe_route", "moe_forward", "moe_destroy", "moe_strerror"} <= declared
    missing = [n for n in sorted(declared) if not hasattr(lib, n)]
    assert not missing, missing
    assert set(moe.EXPORTS) <= declared


def test_strerror_names_every_code():
    for c in range(0, -8, -1):
        assert "unknown" not in moe.strerror(c)
    assert "unknown" in moe.strerror(-99)


def _weights(ptr=0x1000):
    return {"router_w": ptr, "router_bias": None, "w13": ptr, "w2": ptr}


@pytest.mark.parametrize("cfg,code", [
    ((2560, 768, 512, 8, 1), None),            # valid shapes: fails later (alignment below)
    ((2561, 768, 512, 8, 1), moe.MOE_ERR_SHAPE),
    ((2560, 100, 512, 8, 1), moe.MOE_ERR_SHAPE),
    ((2560, 768, 513, 8, 1), moe.MOE_ERR_SHAPE),
    ((2560, 768, 512, 9, 1), moe.MOE_ERR_SHAPE),
    ((2560, 768, 4, 8, 1), moe.MOE_ERR_SHAPE),
    ((2560, 768, 512, 8, 3), moe.MOE_ERR_SHAPE),
])
def test_create_validates_shapes(cfg, code):
    w = _weights(0x1008)                           # misaligned on purpose (never dereferenced)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_create(*cfg, w, 4)
    assert ei.value.code == (code if code is not None else moe.MOE_ERR_ALIGN)


def test_create_rejects_null_and_bad_token_count():
    w = _weights(0x1000)
    w["w2"] = None
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_create(2560, 768, 512, 8, 1, w, 4)
    assert ei.value.code == moe.MOE_ERR_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_create(2560, 768, 512, 8, 1, _weights(0x1000), 0)
    assert ei.value.code == moe.MOE_ERR_ARG


def test_calls_on_null_handle_fail_cleanly():
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route(None, 0x1000, 1, 0x1000, 0x1000)
    assert ei.value.code == moe.MOE_ERR_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward(None, 0x1000, 1, 0x1000, 0x1000, 0x1000)
    assert ei.value.code == moe.MOE_ERR_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_quantize_fp8(None, 1, 1, 0x1000, 0x1000)
    assert ei.value.code == moe.MOE_ERR_ARG
    moe.moe_destroy(None)
    assert moe.moe_last_path(None) == 0


def test_prefill_kernel_selection_needs_a_handle():
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_set_prefill_kernel(None, moe.MOE_PREFILL_AUTO)
    assert ei.value.code == moe.MOE_ERR_ARG


@pytest.mark.parametrize("V,H,T,ptr,code", [
    (16, 128, 0, 0x1000, moe.MOE_ERR_ARG),       # no tokens
    (16, 128, 9, 0x1000, moe.MOE_ERR_ARG),       # more than 8 tokens
    (0, 128, 1, 0x1000, moe.MOE_ERR_ARG),        # empty vocabulary
    (16, 96, 1, 0x1000, moe.MOE_ERR_SHAPE),      # H not a multiple of 64
    (16, 128, 1, 0x1008, moe.MOE_ERR_ALIGN),     # misaligned (never dereferenced)
])
def test_lmhead_logits_validates_arguments(V, H, T, ptr, code):
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_lmhead_logits(ptr, ptr, V, H, ptr, T, ptr)
    assert ei.value.code == code


def test_lmhead_quantize_validates_arguments():
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_lmhead_quantize(None, 16, 128, 0x1000, 0x1000)
    assert ei.value.code == moe.MOE_ERR_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_lmhead_quantize(0x1000, 16, 100, 0x1000, 0x1000)
    assert ei.value.code == moe.MOE_ERR_SHAPE
