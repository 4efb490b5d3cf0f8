"""Plant plausible mistakes in the oracle (CPU only) and check that the pins
catch each one.  Guards against pins that would pass a wrong oracle."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import moe as M

from oracle import lmhead as LHM

import test_oracle_formats as TF
import test_oracle_layer as TL
import test_oracle_lmhead as TLH

PINS = [
    TF.test_e2m1_table_matches_ocp,
    TF.test_unpack_nibble_order,
    TF.test_e8m0_values,
    TF.test_e4m3_decode_all_codes_vs_torch,
    TF.test_e4m3_encode_matches_torch_in_range,
    TF.test_e4m3_encode_saturates,
    TF.test_bf16_round_is_single_rounding_from_float64,
    TL.test_topk_brute_force_and_ties,
    TL.test_routing_weight_invariants,
    TL.test_quantize_fp8_properties,
    TL.test_one_hot_column_extraction,
    TL.test_scale_shift_is_exact_power_of_two,
    TL.test_matvec_brute_force_rational,
    TL.test_swiglu_matches_torch_silu,
    lambda: TL.test_layer_brute_force_tiny(False),
    TLH.test_abs_sum_exact_rational,
    TLH.test_abs_sum_equals_logits_when_every_product_is_nonnegative,
]


def _swapped_unpack(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p >> 4
    out[..., 1::2] = p & 0xF
    return out


def _swiglu_swapped(g, u):
    return u / (1.0 + np.exp(-u)) * g


def _weights_no_renorm(logits, ids):
    l = logits.astype(np.float64)
    z = np.exp(l - l.max(axis=1, keepdims=True))
    full = z / z.sum(axis=1, keepdims=True)
    return np.take_along_axis(full, ids.astype(np.int64), 1).astype(np.float32)


def _topk_ties_high_first(logits, k):
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        ids[t] = np.lexsort((-np.arange(E), -logits[t].astype(np.float64)))[:k]
    return ids


def _e8m0_off_by_one(e):
    e = np.asarray(e).astype(np.int64)
    return np.where(e == 255, np.nan, np.ldexp(1.0, e - 126))


def _e4m3_truncate(v):
    v = np.asarray(v, dtype=np.float32)
    a = np.minimum(np.abs(v.astype(np.float64)), 448.0)
    _, ex = np.frexp(a)
    step = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
    t = (np.floor(a / step) * step).astype(np.float32)
    t = np.where(np.signbit(v), -t, t).astype(np.float32)
    return F.__dict__["_orig_e4m3_encode"](t)


def _bf16_double_rounding(v):
    v32 = np.asarray(v, dtype=np.float64).astype(np.float32)
    return F.__dict__["_orig_f64_to_bf16"](v32.astype(np.float64))


def _forward_shared_half(x, ids, w, lw, n_experts, inter, n_shared=1):
    out = M.__dict__["_orig_moe_forward"](x, ids, w, lw, n_experts, inter, n_shared)
    # shared expert added with weight 0.5 instead of 1
    T = ids.shape[0]
    for t in range(T):
        d, *_ = M.expert_ffn(lw.experts[n_experts], out["xq"][t], out["xs"][t], inter)
        out["y64"][t] -= 0.5 * d
    out["y"] = F.f64_to_bf16(out["y64"])
    return out


def _matvec_no_scale(packed, scales, q, s):
    W = F.dequant_mxfp4(packed, scales)
    return W @ F.e4m3_value(q)


def _abs_sum_signed(q_w, s_w, x_bf16):
    # the magnitude sum with the absolute value dropped: the signed logit
    return LHM.lmhead_logits(q_w, s_w, x_bf16)


def _abs_sum_no_weight_scale(q_w, s_w, x_bf16):
    return LHM.__dict__["_orig_lmhead_abs_sum"](q_w, np.ones_like(s_w), x_bf16)


def _abs_sum_abs_outside(q_w, s_w, x_bf16):
    # |sum| instead of sum of |products|
    return np.abs(LHM.lmhead_logits(q_w, s_w, x_bf16))


MUTATIONS = {
    "nibble order swapped": [(F, "unpack_e2m1", _swapped_unpack)],
    "gate and up swapped": [(M, "swiglu", _swiglu_swapped)],
    "softmax not renormalised": [(M, "routing_weights", _weights_no_renorm)],
    "ties to the higher index": [(M, "select_topk", _topk_ties_high_first)],
    "E8M0 bias off by one": [(F, "e8m0_value", _e8m0_off_by_one)],
    "E4M3 truncation": [(F, "e4m3_encode", _e4m3_truncate), (M, "e4m3_encode", _e4m3_truncate)],
    "BF16 double rounding": [(F, "f64_to_bf16", _bf16_double_rounding),
                             (M, "f64_to_bf16", _bf16_double_rounding)],
    "shared expert weight 0.5": [(M, "moe_forward", _forward_shared_half)],
    "activation scale dropped": [(M, "mxfp4_matvec", _matvec_no_scale)],
    "LM-head magnitude sum without abs": [(LHM, "lmhead_abs_sum", _abs_sum_signed)],
    "LM-head magnitude sum without the row scale": [(LHM, "lmhead_abs_sum", _abs_sum_no_weight_scale)],
    "LM-head magnitude sum as |sum|": [(LHM, "lmhead_abs_sum", _abs_sum_abs_outside)],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    F._orig_e4m3_encode = F.e4m3_encode
    F._orig_f64_to_bf16 = F.f64_to_bf16
    M._orig_moe_forward = M.moe_forward
    LHM._orig_lmhead_abs_sum = LHM.lmhead_abs_sum
    for mod, attr, fn in MUTATIONS[name]:
        monkeypatch.setattr(mod, attr, fn)
    caught = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught.append(getattr(pin, "__name__", "layer"))
    assert caught, f"no pin caught mutation: {name}"
