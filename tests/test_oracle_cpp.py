"""Pins of the C++17 float64 oracle (oracle/moe_oracle.cpp): its format
conversions against torch's and an exhaustive nearest-value search; the whole
layer against the exact rational brute force of test_oracle_layer on tiny
shapes; and bit equality with the numpy oracle on seeded full-width layers
(E = 32, T = 1..4, with and without the Zipf router bias), where every output
-- logits, ids, weights, FP8 codes and scales, h, y -- must agree exactly.
The thread count must not change any result."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import cpp as C
from oracle import formats as F
from oracle import moe as M

import test_oracle_formats as TF
import test_oracle_layer as TL


def test_e4m3_encoder_matches_torch_and_nearest_search():
    v = TF._fp32_sweep(65537)
    v = v[np.isfinite(v) & (np.abs(v) <= 464.0)]
    vals = np.unique(np.abs(F.e4m3_value(np.arange(0x7F))))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)),
                            vals.astype(np.float32)])
    v = np.concatenate([v, extra, -extra]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([C.e4m3_encode(float(x)) for x in v], dtype=np.uint8)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(ours[i]), int(ref[i])) for i in bad[:8]]
    # saturation, signed zero
    assert [C.e4m3_encode(x) for x in (464.5, 1e6, -500.0, 0.0, -0.0)] == [0x7E, 0x7E, 0xFE, 0x00, 0x80]
    # nearest finite magnitude by exhaustive search (ties to the even code)
    mags = [(c, Fraction(float(F.e4m3_value(c)))) for c in range(0x7F)]
    rng = np.random.default_rng(17)
    for x in np.concatenate([rng.standard_normal(400) * 50, rng.standard_normal(200) * 0.003]).astype(np.float32):
        fa = abs(Fraction(float(x)))
        best = min(abs(fa - m) for _, m in mags)
        cands = [c for c, m in mags if abs(fa - m) == best]
        c = cands[0] if len(cands) == 1 else [q for q in cands if q % 2 == 0][0]
        assert C.e4m3_encode(float(x)) == c | (0x80 if math.copysign(1.0, float(x)) < 0 else 0)


def test_bf16_rounding_matches_torch_and_is_single():
    v = TF._fp32_sweep(131071)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([C.bf16_round(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(ours, ref)
    # a float64 value just above a midpoint rounds up; exactly at it, to even
    lo, hi = F.bf16_to_f64(np.array([0x4000], np.uint16))[0], F.bf16_to_f64(np.array([0x4001], np.uint16))[0]
    mid = (lo + hi) / 2
    assert C.bf16_round(mid + (hi - lo) * 2.0 ** -30) == 0x4001
    assert C.bf16_round(mid) == 0x4000


@pytest.mark.parametrize("bias", [False, True])
def test_layer_matches_rational_brute_force(bias):
    H, I, E, k = 64, 32, 4, 2
    lw = M.LayerWeights(router_w=synth.router_weight(9, 0, E, H),
                        router_bias=synth.zipf_router_bias(9, 0, E) if bias else None)
    for e in range(E + 1):
        lw.experts[e] = synth.expert_weights(9, 0, e, H, I)
    x = synth.hidden_states(9, 1, 3, H)
    out = C.moe_layer(x, lw.router_w, lw.router_bias, lw.experts, E, k, I)
    ref_y, ref_ids = TL._brute_layer(x, lw, E, k, I)
    assert np.array_equal(out["ids"], ref_ids)
    assert np.array_equal(out["y"], ref_y)


@pytest.mark.parametrize("T,bias,seed", [(1, False, 0), (2, True, 1), (4, False, 2), (3, True, 3)])
def test_bit_equal_to_numpy_oracle(T, bias, seed):
    H, I, E, k, S = 2560, 768, 32, 8, 1
    lw = M.LayerWeights(router_w=synth.router_weight(seed, 0, E, H),
                        router_bias=synth.zipf_router_bias(seed, 0, E) if bias else None)
    x = synth.hidden_states(seed, 100 + T, T, H)
    _, ids, _, _ = M.route(x, lw, k)
    for e in set(ids.ravel().tolist()) | {E}:
        lw.experts[e] = synth.expert_weights(seed, 0, e, H, I)
    ref = M.moe_layer(x, lw, E, k, I, S)
    out = C.moe_layer(x, lw.router_w, lw.router_bias, lw.experts, E, k, I, S)
    for key in ("logits", "ids", "w", "counts", "xq", "xs", "h", "qh", "sh", "y64", "y"):
        assert np.array_equal(np.asarray(ref[key]), np.asarray(out[key])), key


def test_thread_count_does_not_change_results():
    H, I, E, k = 256, 128, 16, 4
    lw = M.LayerWeights(router_w=synth.router_weight(5, 0, E, H), router_bias=None)
    for e in range(E + 1):
        lw.experts[e] = synth.expert_weights(5, 0, e, H, I)
    x = synth.hidden_states(5, 3, 2, H)
    try:
        C.set_threads(1)
        one = C.moe_layer(x, lw.router_w, None, lw.experts, E, k, I)
        C.set_threads(0)
        many = C.moe_layer(x, lw.router_w, None, lw.experts, E, k, I)
    finally:
        C.set_threads(0)
    for key in ("y64", "y", "h", "qh"):
        assert np.array_equal(one[key], many[key]), key
