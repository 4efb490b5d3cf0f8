"""The FP8 output layer (LM head), in float64 -- TEST INFRASTRUCTURE.

The pages' second optimisation ([tanhow] "三项优化是什么？" item 2; [aivibenews]
"Online FP8 LM head"): the 157,184 x 2,560 output layer, stored in BF16 and
read in full for every generated token, is quantised to FP8 once when the
model is loaded, which halves the bytes read per token.

Readings taken where the pages are silent:

* weights: FP8 E4M3, one float32 scale per vocabulary row = amax/448 (the
  activation quantiser of the MoE layer, ``moe.quantize_fp8``, applied to the
  rows of the BF16 matrix);
* activations: the hidden state is quantised per token the same way (the
  W8A8 form of an FP8 GEMM);
* logits: ``s_w[v] * s_x[t] * sum_k e4m3(q_w[v,k]) * e4m3(q_x[t,k])``,
  returned here in float64 (every product of two E4M3 values is exact in
  float64; the sum carries float64 rounding only).

Parity pins (tests/test_oracle_lmhead.py): an exact rational brute force on
small shapes, one-hot activations extracting a dequantised column, exact
power-of-two scaling of the weights, and the row maximum mapping to the
largest E4M3 code.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64, e4m3_value
from .moe import quantize_fp8


def lmhead_quantize(w_bf16: np.ndarray):
    """BF16 bits ``[V][H]`` -> (E4M3 codes ``[V][H]`` uint8, scales float32 ``[V]``)."""
    return quantize_fp8(bf16_to_f64(w_bf16).astype(np.float32))


def lmhead_logits(q_w: np.ndarray, s_w: np.ndarray, x_bf16: np.ndarray) -> np.ndarray:
    """float64 logits ``[T][V]`` of BF16 tokens ``x [T][H]`` through the FP8
    layer ``(q_w, s_w)``; x is quantised per token first."""
    q_x, s_x = quantize_fp8(bf16_to_f64(np.atleast_2d(x_bf16)).astype(np.float32))
    W = e4m3_value(q_w).astype(np.float64)          # [V][H]
    X = e4m3_value(q_x).astype(np.float64)          # [T][H]
    return (X @ W.T) * np.asarray(s_w, np.float64)[None, :] * np.asarray(s_x, np.float64)[:, None]


def lmhead_abs_sum(q_w: np.ndarray, s_w: np.ndarray, x_bf16: np.ndarray) -> np.ndarray:
    """``s_w[v] * s_x[t] * sum_k |e4m3(q_w[v,k]) * e4m3(q_x[t,k])|``: the scale
    of any rounding error of an accumulated logit (for tolerances)."""
    q_x, s_x = quantize_fp8(bf16_to_f64(np.atleast_2d(x_bf16)).astype(np.float32))
    W = np.abs(e4m3_value(q_w).astype(np.float64))
    X = np.abs(e4m3_value(q_x).astype(np.float64))
    return (X @ W.T) * np.asarray(s_w, np.float64)[None, :] * np.asarray(s_x, np.float64)[:, None]
