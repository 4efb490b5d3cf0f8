"""Number formats of the layer, written from their definitions (float64).

TEST INFRASTRUCTURE: see ``oracle/__init__.py``.

* E2M1 (FP4) element and E8M0 scale -- [OCP-MX]; the pages only say that
  MXFP4 is a blocked 4-bit float format ([devotd] section 2).
* E4M3 (FP8) -- [OCP-FP8]; the pages say activations are 8-bit ([tanhow]
  "为什么 DGX Spark 上的 MoE 解码是内存受限的？", W4A8 recipe).
* BF16 output rounding -- round to nearest, ties to even, applied once.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


# ------------------------------------------------------------------ E2M1 --

def e2m1_value(code) -> np.ndarray:
    """Value of 4-bit E2M1 codes: bit 3 sign, bits 2..1 exponent (bias 1),
    bit 0 mantissa; exponent field 0 is subnormal (0 or 0.5)."""
    c = np.asarray(code).astype(np.int64) & 0xF
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return np.where(s == 1, -mag, mag).astype(np.float64)


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    """``[..., K/2]`` bytes -> ``[..., K]`` codes.  Element ``2j`` is the low
    nibble of byte ``j`` and element ``2j+1`` the high nibble (the plain
    reading: the pages do not fix the nibble order)."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# ------------------------------------------------------------------ E8M0 --

def e8m0_value(e) -> np.ndarray:
    """E8M0 scale: ``2**(e - 127)`` for e in 0..254; 255 is NaN."""
    e = np.asarray(e).astype(np.int64)
    v = np.ldexp(np.ones(e.shape, dtype=np.float64), e - 127)
    return np.where(e == 255, np.nan, v)


def dequant_mxfp4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dequantise an MXFP4 matrix: ``W[r, k] = e2m1(code[r, k]) * 2**(E[r, k//32] - 127)``.

    ``packed`` is ``[R][K/2]`` (two codes per byte), ``scales`` ``[R][K/32]``:
    one E8M0 per 32 consecutive elements along K, the input dimension
    ([OCP-MX] block of 32).  Every value is exact in float64."""
    codes = unpack_e2m1(packed)
    R, K = codes.shape
    sc = e8m0_value(scales)
    assert sc.shape == (R, K // 32)
    return e2m1_value(codes) * np.repeat(sc, 32, axis=1)


# ------------------------------------------------------------------ E4M3 --

def e4m3_value(code) -> np.ndarray:
    """Value of E4M3 bytes: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0
    mantissa; exponent field 0 is subnormal (m/8 * 2**-6); S.1111.111 is NaN;
    there are no infinities."""
    c = np.asarray(code).astype(np.int64) & 0xFF
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e4m3_encode(v) -> np.ndarray:
    """Encode float32 values to E4M3: round to nearest, ties to even, then
    saturate to +-448 ("satfinite": anything beyond the largest finite value,
    infinities included, becomes +-448).  NaN encodes as 0x7F.

    Works on the exact value of each float32 in float64: the grid spacing
    near ``a`` is ``2**(max(floor(log2 a), -6) - 3)`` (3 mantissa bits; the
    subnormal spacing 2**-9 below 2**-6)."""
    v = np.asarray(v, dtype=np.float32)
    nan = np.isnan(v)
    neg = np.signbit(v)
    a = np.abs(v.astype(np.float64))
    a = np.where(nan, 0.0, a)
    a = np.minimum(a, 2.0 * E4M3_MAX)            # infinities -> large finite
    _, ex = np.frexp(a)                            # a = f * 2**ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)
    step = np.ldexp(1.0, E - 3)
    r = np.rint(a / step)                          # ties to even
    val = np.minimum(r * step, E4M3_MAX)           # satfinite
    # bits of the (exact) rounded value
    sub = val < 2.0 ** -6
    _, ev = np.frexp(np.where(sub, 1.0, val))
    Ev = ev - 1
    mant_n = np.rint(np.ldexp(np.where(sub, 1.0, val), -Ev) * 8.0 - 8.0).astype(np.int64)
    code_n = ((Ev + 7) << 3) | mant_n
    code_s = np.rint(val / 2.0 ** -9).astype(np.int64)
    code = np.where(sub, code_s, code_n)
    code = np.where(neg, code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


# ------------------------------------------------------------------ BF16 --

def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    """Round float64 to bfloat16 bits, nearest with ties to even, in one step
    (no intermediate float32 rounding).  Finite results beyond the largest
    bfloat16 become infinities."""
    v = np.asarray(v, dtype=np.float64)
    nan = np.isnan(v)
    neg = np.signbit(v)
    a = np.abs(np.where(nan, 0.0, v))
    a = np.minimum(a, 2.0 ** 129)
    _, ex = np.frexp(a)
    E = np.maximum(ex - 1, -126)
    step = np.ldexp(1.0, E - 7)                    # 8 significant bits
    val = np.rint(a / step) * step
    with np.errstate(over="ignore"):
        f = val.astype(np.float32)                 # exact, or inf past 2**128
    bits = (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(neg, bits | np.uint16(0x8000), bits)
    bits = np.where(nan, np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


def f64_to_f32(v) -> np.ndarray:
    """IEEE round-to-nearest-even conversion (numpy's cast)."""
    return np.asarray(v, dtype=np.float64).astype(np.float32)
