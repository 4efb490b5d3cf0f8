"""The MoE decode layer, step by step, in float64 -- TEST INFRASTRUCTURE.

See ``oracle/__init__.py`` for the sources ([tanhow], [devotd], [OCP-MX],
[OCP-FP8]).  One token goes to ``top_k`` of ``n_experts`` routed experts plus
the shared expert(s) ([tanhow] "Ling 3.0 是什么" sparse-MoE bullet: 8 of 512
plus 1 shared); every expert is a SwiGLU FFN of width ``inter`` ([tanhow]
"三项优化是什么？" item 1: width 768) at hidden ``hidden`` (2560, from the LM
head shape in item 2); weights are MXFP4 and both expert GEMMs take FP8
activations (the W4A8 recipe, [tanhow] "为什么 … 内存受限的？").

Readings taken where the pages are silent (each repeated at its function):

* scoring: softmax over float32 logits, top-k, renormalised over the k;
* logits: BF16 hidden state x BF16 router summed in float64, rounded once
  to float32, then the optional float32 bias added in float32;
* ordering: descending logit, equal logits -> lower expert index first;
* activations: FP8 E4M3, one float32 scale per token = amax/448
  (IEEE float32 division), codes = E4M3(x / scale) rounded to nearest even
  with saturation; amax == 0 gives scale 1 and all-zero codes;
* the SwiGLU output h is rounded to float32 and re-quantised to FP8 the same
  way, one scale per (token, expert), so the down GEMM is W4A8 as well;
* shared expert: same width and format, added with weight 1;
* output: the float64 sum rounded once to BF16.

Parity pins (tests/test_oracle_*.py): format tables and library
conversions, routing invariants and brute force, one-hot column extraction,
exact power-of-two scale shifts, zero codes, and an exact rational
brute-force of the whole layer on tiny shapes.  Parity unpinned: nothing
beyond those -- the pages print no worked example of the layer's output.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .formats import (E4M3_MAX, bf16_to_f64, dequant_mxfp4, e4m3_encode,
                      e4m3_value, f64_to_bf16)


@dataclass
class LayerWeights:
    """Host copy of one layer.  Expert arrays are indexed ``[expert]`` with the
    shared expert(s) after the routed ones (index ``n_experts`` ...); only the
    experts a call touches need to be present (a dict ``expert -> arrays``).

    * ``router_w``: BF16 bits ``[E][H]``; ``router_bias``: float32 ``[E]`` or None
    * per expert: ``w13_codes [2I][H/2]``, ``w13_scales [2I][H/32]`` (rows
      0..I-1 gate, I..2I-1 up), ``w2_codes [H][I/2]``, ``w2_scales [H][I/32]``.
    """
    router_w: np.ndarray
    router_bias: np.ndarray | None
    experts: dict = field(default_factory=dict)


# ------------------------------------------------------------- routing --

def router_logits(x_bf16: np.ndarray, router_w_bf16: np.ndarray,
                  bias: np.ndarray | None = None) -> np.ndarray:
    """``l[t, e] = f32( sum_k x[t,k] * W[e,k] )`` with the sum taken in float64,
    sequentially over k; then ``l += b_e`` as a float32 add.

    Routing to top-8 of 512 by these logits: [tanhow] "Ling 3.0 是什么"
    sparse-MoE bullet, [aivibenews] opening paragraph."""
    x = bf16_to_f64(x_bf16)                       # [T, H]
    W = bf16_to_f64(router_w_bf16)                # [E, H]
    T, H = x.shape
    acc = np.zeros((T, W.shape[0]), dtype=np.float64)
    for k in range(H):
        acc += x[:, k:k + 1] * W[None, :, k]
    l = acc.astype(np.float32)
    if bias is not None:
        l = (l + np.asarray(bias, dtype=np.float32)[None, :]).astype(np.float32)
    return l


def select_topk(logits: np.ndarray, k: int) -> np.ndarray:
    """Ids of the ``k`` largest logits per token, in descending order of logit;
    equal logits are ordered by the lower expert index first."""
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        order = np.lexsort((idx, -logits[t].astype(np.float64)))
        ids[t] = order[:k]
    return ids


def routing_weights(logits: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Softmax over all experts, kept for the selected ones and renormalised
    to sum 1 -- equal to a softmax over the selected logits alone:
    ``p_i = exp(l_i - l_max) / sum_j exp(l_j - l_max)`` in float64, stored
    as float32."""
    sel = np.take_along_axis(logits.astype(np.float64), ids.astype(np.int64), axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    return (z / z.sum(axis=1, keepdims=True)).astype(np.float32)


def expert_counts(ids: np.ndarray, n_experts: int) -> np.ndarray:
    """Tokens dispatched to each routed expert (token -> expert dispatch)."""
    return np.bincount(ids.reshape(-1).astype(np.int64), minlength=n_experts).astype(np.int32)


def route(x_bf16, lw: LayerWeights, top_k: int):
    l = router_logits(x_bf16, lw.router_w, lw.router_bias)
    ids = select_topk(l, top_k)
    w = routing_weights(l, ids)
    return l, ids, w, expert_counts(ids, lw.router_w.shape[0])


# --------------------------------------------------- FP8 activation quant --

def quantize_fp8(v32: np.ndarray):
    """Per-row FP8 E4M3 quantisation of float32 rows ``[R][K]``.

    ``amax = max|v|``; ``s = f32(amax) / 448`` as an IEEE float32 division
    (s = 1 when amax is 0); ``q = E4M3(f32(v / s))`` with RNE + saturation.
    Returns ``(codes uint8 [R][K], s float32 [R])``.  The 8-bit activation
    side of the W4A8 recipe ([tanhow] "为什么 … 内存受限的？",
    [devotd] section 2); the per-row amax/448 scale is the plain reading."""
    v = np.asarray(v32, dtype=np.float32)
    amax = np.max(np.abs(v), axis=-1).astype(np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s = np.where(amax == 0, np.float32(1.0), s).astype(np.float32)
    q = e4m3_encode((v / s[..., None]).astype(np.float32))
    return q, s


# ---------------------------------------------------------- expert FFN --

def mxfp4_matvec(packed: np.ndarray, scales: np.ndarray, q_codes: np.ndarray,
                 s: np.float32) -> np.ndarray:
    """``out[r] = s * sum_b 2**(E[r,b]-127) * sum_{k in b} e2m1(c[r,k]) * e4m3(q[k])``
    in float64 (dequantise, then a float64 matrix-vector product).  With the
    layer's value ranges every partial sum is exact in float64, so the
    result is the exact product rounded once by the final multiply by s."""
    W = dequant_mxfp4(packed, scales)
    a = e4m3_value(q_codes)
    return np.float64(s) * (W @ a)


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """``h = silu(g) * u = g / (1 + exp(-g)) * u`` in float64 (for very
    negative g the exponential overflows to inf and h is -0 * u, the limit)."""
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def expert_ffn(ex: dict, xq: np.ndarray, xs: np.float32, inter: int):
    """One expert on one token: gate/up GEMV, SwiGLU, FP8 re-quantisation of
    h, down GEMV.  Returns ``(d float64 [H], qh uint8 [I], sh float32, h float32 [I])``."""
    gu = mxfp4_matvec(ex["w13_codes"], ex["w13_scales"], xq, xs)
    g, u = gu[:inter], gu[inter:]
    h32 = swiglu(g, u).astype(np.float32)
    qh, sh = quantize_fp8(h32[None, :])
    d = mxfp4_matvec(ex["w2_codes"], ex["w2_scales"], qh[0], sh[0])
    return d, qh[0], sh[0], h32


def moe_forward(x_bf16: np.ndarray, ids: np.ndarray, w: np.ndarray,
                lw: LayerWeights, n_experts: int, inter: int, n_shared: int = 1):
    """``y[t] = bf16( sum_i w[t,i] * FFN_{ids[t,i]}(x_t) + sum_s FFN_shared_s(x_t) )``.

    Returns a dict with ``y`` (BF16 bits ``[T][H]``), ``y64`` (float64 before
    rounding), ``xq``/``xs`` (FP8 activations), and per (token, slot)
    ``qh [T][S][I]``, ``sh [T][S]``, ``h [T][S][I]`` where the slots are the
    routed ones in ``ids`` order followed by the shared experts."""
    x32 = bf16_to_f64(x_bf16).astype(np.float32)
    xq, xs = quantize_fp8(x32)
    T, k = ids.shape
    S = k + n_shared
    H = x32.shape[1]
    y64 = np.zeros((T, H), dtype=np.float64)
    qh = np.zeros((T, S, inter), dtype=np.uint8)
    sh = np.zeros((T, S), dtype=np.float32)
    hh = np.zeros((T, S, inter), dtype=np.float32)
    for t in range(T):
        slots = [(int(ids[t, i]), float(w[t, i])) for i in range(k)]
        slots += [(n_experts + j, 1.0) for j in range(n_shared)]
        for si, (e, we) in enumerate(slots):
            d, qh[t, si], sh[t, si], hh[t, si] = expert_ffn(lw.experts[e], xq[t], xs[t], inter)
            y64[t] += np.float64(we) * d
    return {"y": f64_to_bf16(y64), "y64": y64, "xq": xq, "xs": xs,
            "qh": qh, "sh": sh, "h": hh}


def moe_layer(x_bf16: np.ndarray, lw: LayerWeights, n_experts: int, top_k: int,
              inter: int, n_shared: int = 1):
    """Route, then run the experts and combine.  Returns the forward dict plus
    ``logits``, ``ids``, ``w``, ``counts``."""
    l, ids, w, counts = route(x_bf16, lw, top_k)
    out = moe_forward(x_bf16, ids, w, lw, n_experts, inter, n_shared)
    out.update(logits=l, ids=ids, w=w, counts=counts)
    return out


def down_replay(ex: dict, qh: np.ndarray, sh: np.float32) -> np.ndarray:
    """The down GEMV alone on given FP8 activations (used to check the down
    step in isolation from the re-quantisation of h)."""
    return mxfp4_matvec(ex["w2_codes"], ex["w2_scales"], qh, sh)


# ------------------------------------------------- chained-layer harness --

def residual_rmsnorm(r_bf16: np.ndarray, y_bf16: np.ndarray, eps: float = 1e-6):
    """Harness step between chained layers (not part of the MoE layer; the
    pages do not describe the stack's normalisation -- plain reading: residual
    add, RMS normalisation without a learned weight):
    ``r = bf16(r + y)``; ``x = bf16( r / sqrt(mean(r**2) + eps) )`` with the
    sum, mean, square root and division in float64."""
    r = f64_to_bf16(bf16_to_f64(r_bf16) + bf16_to_f64(y_bf16))
    rv = bf16_to_f64(r)
    ms = np.zeros(rv.shape[0])
    for k in range(rv.shape[1]):
        ms += rv[:, k] * rv[:, k]
    den = np.sqrt(ms / rv.shape[1] + np.float64(np.float32(eps)))
    return r, f64_to_bf16(rv / den[:, None])
