"""Pins of the FP8 output-layer oracle (oracle/lmhead.py) against what the
definitions fix: an exact rational brute force, one-hot extraction of a
dequantised column, exact power-of-two scaling, the row maximum at the
largest E4M3 code, and tokens independent of each other."""
from fractions import Fraction

import numpy as np

import synth
from oracle import formats as OF
from oracle import lmhead as LH


def _bf16(v):
    return synth._fp32_to_bf16_bits(np.asarray(v, np.float32))


def _e4m3_fraction(code: int) -> Fraction:
    # E4M3 by its definition (OCP OFP8): sign, 4 exponent bits (bias 7), 3 mantissa bits
    s, e, m = code >> 7, (code >> 3) & 15, code & 7
    v = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if s else v


def test_brute_force_small():
    w = synth.lmhead_weight(3, 5, 64)
    x = synth.hidden_states(3, 9, 2, 64)
    q, s = LH.lmhead_quantize(w)
    got = LH.lmhead_logits(q, s, x)
    qx, sx = LH.quantize_fp8(OF.bf16_to_f64(x).astype(np.float32))
    for t in range(2):
        for v in range(5):
            acc = sum(_e4m3_fraction(int(q[v, k])) * _e4m3_fraction(int(qx[t, k])) for k in range(64))
            ref = acc * Fraction(float(s[v])) * Fraction(float(sx[t]))
            assert abs(got[t, v] - float(ref)) <= 1e-15 * max(abs(float(ref)), 1e-30)


def test_one_hot_extracts_a_dequantised_column():
    w = synth.lmhead_weight(1, 7, 128)
    q, s = LH.lmhead_quantize(w)
    for k in (0, 37, 127):
        x = np.zeros((1, 128), np.float32)
        x[0, k] = 1.75  # s_x = 1.75 / 448 = 2^-8 exactly; the code of x is 448
        got = LH.lmhead_logits(q, s, _bf16(x))[0]
        col = OF.e4m3_value(q[:, k]).astype(np.float64) * s.astype(np.float64)
        assert np.array_equal(got, col * 1.75)


def test_power_of_two_scaling_is_exact():
    w = synth.lmhead_weight(2, 6, 64)
    w2 = _bf16(OF.bf16_to_f64(w) * 4.0)
    x = synth.hidden_states(2, 1, 1, 64)
    q, s = LH.lmhead_quantize(w)
    q2, s2 = LH.lmhead_quantize(w2)
    assert np.array_equal(q, q2) and np.array_equal(s2, s * np.float32(4))
    assert np.array_equal(LH.lmhead_logits(q2, s2, x), 4.0 * LH.lmhead_logits(q, s, x))


def test_row_maximum_takes_the_largest_code():
    w = synth.lmhead_weight(4, 9, 64)
    q, s = LH.lmhead_quantize(w)
    a = np.abs(OF.bf16_to_f64(w))
    idx = np.argmax(a, axis=1)
    codes = q[np.arange(9), idx] & 0x7F
    assert np.all(codes == 0x7E)  # 448
    assert np.allclose(s, a.max(axis=1) / 448.0, rtol=1e-7)


def test_tokens_are_independent():
    w = synth.lmhead_weight(5, 11, 128)
    q, s = LH.lmhead_quantize(w)
    x = synth.hidden_states(5, 2, 3, 128)
    all3 = LH.lmhead_logits(q, s, x)
    for t in range(3):
        assert np.array_equal(all3[t], LH.lmhead_logits(q, s, x[t:t + 1])[0])
    assert np.all(LH.lmhead_abs_sum(q, s, x) >= np.abs(all3))


def test_abs_sum_exact_rational():
    """lmhead_abs_sum against an exact rational evaluation of its definition,
    s_w[v] * s_x[t] * sum_k |e4m3(q_w[v,k]) * e4m3(q_x[t,k])|, with the E4M3
    values decoded from the OCP OFP8 bit fields, on a shape with V != T so a
    transposed product cannot pass."""
    w = synth.lmhead_weight(6, 5, 64)
    x = synth.hidden_states(6, 4, 3, 64)
    q, s = LH.lmhead_quantize(w)
    got = LH.lmhead_abs_sum(q, s, x)
    assert got.shape == (3, 5)
    qx, sx = LH.quantize_fp8(OF.bf16_to_f64(x).astype(np.float32))
    for t in range(3):
        for v in range(5):
            acc = sum(abs(_e4m3_fraction(int(q[v, k])) * _e4m3_fraction(int(qx[t, k]))) for k in range(64))
            ref = acc * Fraction(float(s[v])) * Fraction(float(sx[t]))
            assert ref > 0
            assert abs(got[t, v] - float(ref)) <= 1e-15 * float(ref)


def test_abs_sum_equals_logits_when_every_product_is_nonnegative():
    """With non-negative weights and activations no product is negative, so
    the sum of magnitudes is the logit itself; flipping the sign of one
    weight row leaves the magnitude sum unchanged and negates the logit."""
    w = _bf16(np.abs(OF.bf16_to_f64(synth.lmhead_weight(7, 4, 64))).astype(np.float32))
    x = _bf16(np.abs(OF.bf16_to_f64(synth.hidden_states(7, 3, 2, 64))).astype(np.float32))
    q, s = LH.lmhead_quantize(w)
    assert np.array_equal(LH.lmhead_abs_sum(q, s, x), LH.lmhead_logits(q, s, x))
    wn = _bf16(-OF.bf16_to_f64(w).astype(np.float32))
    qn, sn = LH.lmhead_quantize(wn)
    assert np.array_equal(LH.lmhead_abs_sum(qn, sn, x), LH.lmhead_abs_sum(q, s, x))
    assert np.array_equal(LH.lmhead_logits(qn, sn, x), -LH.lmhead_logits(q, s, x))
