"""Pins of the oracle's layer arithmetic: routing invariants and brute force,
library routines (torch float64 matmul, torch SiLU), one-hot column
extraction, exact power-of-two scale shifts, zero codes, and an exact
rational brute force of the whole layer on tiny shapes.  No GPU."""
import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import moe as M

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_table():
    tab = {}
    with open(os.path.join(GOLDEN, "e2m1_ocp_mx.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                tab[int(c)] = Fraction(float(v))
    return tab


E2M1 = _e2m1_table()


def _bf16(bits):
    return struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0]


# ------------------------------------------------------------ page shapes --

def test_page_shapes_and_bytes():
    with open(os.path.join(GOLDEN, "page_shapes.json")) as f:
        p = json.load(f)
    H, I = p["lm_head_shape"][1], p["expert_width"]
    assert H == p["hidden"] == 2560 and I == 768
    per_expert = 2 * I * H // 2 + 2 * I * H // 32 + H * I // 2 + H * I // 32
    assert per_expert == 3_133_440
    touched = (p["top_k"] + p["n_shared_experts"]) * per_expert
    assert abs(touched / 1e6 - 28.2) < 0.05            # "~28 MB touched per token"
    layer = (p["n_routed_experts"] + p["n_shared_experts"]) * per_expert
    assert abs(layer / 1e9 - 1.6) < 0.01               # "~1.6 GB per layer"
    # 4 verified tokens touch at most 4 x 8 = 32 routed experts
    assert p["verify_tokens"] * p["top_k"] == p["verify_max_routed_experts"]


# --------------------------------------------------------------- routing --

def _route_case(E=64, H=256, T=5, seed=11, bias=False):
    x = synth.hidden_states(seed, 0, T, H)
    wr = synth.router_weight(seed, 0, E, H)
    b = synth.zipf_router_bias(seed, 0, E) if bias else None
    return x, wr, b


def test_router_logits_match_torch_float64_matmul():
    x, wr, b = _route_case(bias=True)
    l = M.router_logits(x, wr, b)
    xt = torch.from_numpy(F.bf16_to_f64(x))
    wt = torch.from_numpy(F.bf16_to_f64(wr))
    ref = (xt @ wt.T).to(torch.float32) + torch.from_numpy(b)
    assert np.array_equal(l, ref.numpy())


def test_topk_brute_force_and_ties():
    x, wr, b = _route_case(bias=True)
    l = M.router_logits(x, wr, b)
    ids = M.select_topk(l, 8)
    for t in range(l.shape[0]):
        ref = sorted(range(l.shape[1]), key=lambda e: (-float(l[t, e]), e))[:8]
        assert ids[t].tolist() == ref
    tie = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, -1.0]], dtype=np.float32)
    assert M.select_topk(tie, 4).tolist() == [[1, 2, 4, 3]]


def test_routing_weight_invariants():
    x, wr, b = _route_case(E=512, H=2560, T=4, seed=5)
    l = M.router_logits(x, wr, b)
    ids = M.select_topk(l, 8)
    w = M.routing_weights(l, ids)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1) <= 1e-6)
    for t in range(4):
        assert len(set(ids[t].tolist())) == 8
        assert np.all(np.diff(w[t]) <= 0)               # descending logit order
    # softmax over all experts, kept and renormalised == softmax over the 8
    full = torch.softmax(torch.from_numpy(l.astype(np.float64)), dim=1).numpy()
    sel = np.take_along_axis(full, ids.astype(np.int64), 1)
    ren = sel / sel.sum(1, keepdims=True)
    assert np.allclose(ren, w, rtol=2e-7, atol=0)
    c = M.expert_counts(ids, 512)
    assert c.sum() == 4 * 8 and c.max() <= 4


# -------------------------------------------------------- FP8 activations --

def test_quantize_fp8_properties():
    x = synth.hidden_states(2, 0, 3, 2560)
    v = F.bf16_to_f64(x).astype(np.float32)
    q, s = M.quantize_fp8(v)
    # the amax element maps to +-448 exactly
    for t in range(3):
        i = int(np.argmax(np.abs(v[t])))
        assert q[t, i] in (0x7E, 0xFE)
    # x -> 2x: identical codes, scale doubles exactly
    q2, s2 = M.quantize_fp8(v * np.float32(2))
    assert np.array_equal(q2, q) and np.array_equal(s2, 2 * s)
    # zero row: scale 1, zero codes
    qz, sz = M.quantize_fp8(np.zeros((1, 64), np.float32))
    assert sz[0] == 1.0 and not qz.any()
    # dequantised values lie within half an E4M3 step of x / s
    deq = F.e4m3_value(q) * s[:, None]
    assert np.all(np.abs(deq - v) <= np.abs(v) * 2.0 ** -4 + s[:, None] * 2.0 ** -10)


# ----------------------------------------------------------- MXFP4 GEMV --

def _rand_mx(rng, R, K, lo=120, hi=124):
    codes = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    scales = rng.integers(lo, hi + 1, (R, K // 32), dtype=np.uint8)
    return codes, scales


def test_one_hot_column_extraction():
    """x = 448 e_k gives s = 1 and q = e4m3(448), so out[r] / 448 is the
    dequantised column k: code nibble k%2 of byte k//2, scale block k//32."""
    rng = np.random.default_rng(1)
    R, K = 16, 96
    codes, scales = _rand_mx(rng, R, K)
    for k in (0, 1, 31, 32, 33, 95):
        x = np.zeros(K, np.float32)
        x[k] = 448.0
        q, s = M.quantize_fp8(x[None])
        assert s[0] == 1.0
        out = M.mxfp4_matvec(codes, scales, q[0], s[0])
        for r in range(R):
            byte = int(codes[r, k // 2])
            nib = byte & 0xF if k % 2 == 0 else byte >> 4
            want = E2M1[nib] * Fraction(2) ** (int(scales[r, k // 32]) - 127) * 448
            assert Fraction(out[r]) == want, (k, r)


def test_scale_shift_is_exact_power_of_two():
    rng = np.random.default_rng(2)
    codes, scales = _rand_mx(rng, 32, 256)
    q = F.e4m3_encode(rng.standard_normal(256).astype(np.float32) * 50)
    s = np.float32(0.37)
    a = M.mxfp4_matvec(codes, scales, q, s)
    b = M.mxfp4_matvec(codes, scales + 1, q, s)
    assert np.array_equal(b, 2 * a)
    z = M.mxfp4_matvec(np.zeros_like(codes), scales, q, s)
    assert not z.any()


def test_matvec_brute_force_rational():
    rng = np.random.default_rng(4)
    R, K = 8, 64
    codes, scales = _rand_mx(rng, R, K, 100, 140)
    q = F.e4m3_encode(rng.standard_normal(K).astype(np.float32) * 30)
    s = np.float32(0.0123)
    out = M.mxfp4_matvec(codes, scales, q, s)
    e4 = {c: Fraction(float(F.e4m3_value(c))) for c in range(256) if c not in (0x7F, 0xFF)}
    for r in range(R):
        acc = Fraction(0)
        for k in range(K):
            byte = int(codes[r, k // 2])
            nib = byte & 0xF if k % 2 == 0 else byte >> 4
            acc += E2M1[nib] * Fraction(2) ** (int(scales[r, k // 32]) - 127) * e4[int(q[k])]
        assert out[r] == float(acc * Fraction(float(s))), r


def test_swiglu_matches_torch_silu():
    g = np.linspace(-40, 40, 1001)
    u = np.cos(g) * 3
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    assert np.allclose(M.swiglu(g, u), ref, rtol=1e-15, atol=1e-300)
    assert M.swiglu(np.array([0.0]), np.array([5.0]))[0] == 0.0


# ------------------------------------------------ whole layer brute force --

def _nearest_e4m3(v32):
    fa = abs(Fraction(float(v32)))
    mags = [(c, Fraction(float(F.e4m3_value(c)))) for c in range(0x7F)]
    if fa > 448:
        c = 0x7E
    else:
        best = min(abs(fa - m) for _, m in mags)
        cands = [c for c, m in mags if abs(fa - m) == best]
        c = cands[0] if len(cands) == 1 else [x for x in cands if x % 2 == 0][0]
    return c | (0x80 if math.copysign(1.0, float(v32)) < 0 else 0)


def _quant_bf(row32):
    amax = max(abs(float(v)) for v in row32)
    s = np.float32(amax) / np.float32(448.0) if amax != 0 else np.float32(1.0)
    codes = [_nearest_e4m3(np.float32(v) / s) for v in row32]
    return codes, s


_BF16_TAB = F.bf16_to_f64(np.arange(0, 0x7F80, dtype=np.uint16))


def _nearest_bf16(y):
    a = abs(y)
    d = np.abs(_BF16_TAB - a)
    m = d.min()
    cands = np.nonzero(d == m)[0]
    c = int(cands[0]) if len(cands) == 1 else int([x for x in cands if x % 2 == 0][0])
    return c | (0x8000 if math.copysign(1.0, y) < 0 else 0)


def _brute_layer(x_bits, lw, E, k, I, n_shared=1):
    T, H = x_bits.shape
    e4 = {c: Fraction(float(F.e4m3_value(c))) for c in range(256) if c not in (0x7F, 0xFF)}
    Wr = [[Fraction(_bf16(b)) for b in row] for row in lw.router_w]

    def matvec(ex_codes, ex_scales, q, s):
        out = []
        for r in range(ex_codes.shape[0]):
            acc = Fraction(0)
            for kk in range(2 * ex_codes.shape[1]):
                byte = int(ex_codes[r, kk // 2])
                nib = byte & 0xF if kk % 2 == 0 else byte >> 4
                acc += E2M1[nib] * Fraction(2) ** (int(ex_scales[r, kk // 32]) - 127) * e4[q[kk]]
            out.append(float(acc * Fraction(float(s))))
        return out

    ys, all_ids = [], []
    for t in range(T):
        x = [Fraction(_bf16(b)) for b in x_bits[t]]
        l = []
        for e in range(E):
            v = np.float32(float(sum(a * b for a, b in zip(x, Wr[e]))))
            if lw.router_bias is not None:
                v = np.float32(v + lw.router_bias[e])
            l.append(v)
        ids = sorted(range(E), key=lambda e: (-float(l[e]), e))[:k]
        all_ids.append(ids)
        lm = max(float(l[i]) for i in ids)
        z = [math.exp(float(l[i]) - lm) for i in ids]
        p = [np.float32(zi / sum(z)) for zi in z]
        xq, xs = _quant_bf([np.float32(float(v)) for v in x])
        slots = list(zip(ids, p)) + [(E + j, np.float32(1.0)) for j in range(n_shared)]
        y = [0.0] * H
        for e, pe in slots:
            ex = lw.experts[e]
            gu = matvec(ex["w13_codes"], ex["w13_scales"], xq, xs)
            h = [np.float32(g / (1.0 + math.exp(-g)) * u) for g, u in zip(gu[:I], gu[I:])]
            qh, sh = _quant_bf(h)
            d = matvec(ex["w2_codes"], ex["w2_scales"], qh, sh)
            y = [yi + float(pe) * di for yi, di in zip(y, d)]
        ys.append([_nearest_bf16(v) for v in y])
    return np.array(ys, dtype=np.uint16), np.array(all_ids)


@pytest.mark.parametrize("bias", [False, True])
def test_layer_brute_force_tiny(bias):
    H, I, E, k = 64, 32, 4, 2
    lw = M.LayerWeights(router_w=synth.router_weight(9, 0, E, H),
                        router_bias=synth.zipf_router_bias(9, 0, E) if bias else None)
    for e in range(E + 1):
        lw.experts[e] = synth.expert_weights(9, 0, e, H, I)
    x = synth.hidden_states(9, 1, 3, H)
    out = M.moe_layer(x, lw, E, k, I)
    ref_y, ref_ids = _brute_layer(x, lw, E, k, I)
    assert np.array_equal(out["ids"], ref_ids)
    assert np.array_equal(out["y"], ref_y)


def test_four_tokens_equal_four_single_calls():
    H, I, E, k = 128, 64, 8, 2
    lw = M.LayerWeights(router_w=synth.router_weight(3, 0, E, H), router_bias=None)
    for e in range(E + 1):
        lw.experts[e] = synth.expert_weights(3, 0, e, H, I)
    x = synth.hidden_states(3, 2, 4, H)
    four = M.moe_layer(x, lw, E, k, I)
    for t in range(4):
        one = M.moe_layer(x[t:t + 1], lw, E, k, I)
        assert np.array_equal(one["y"][0], four["y"][t])
        assert np.array_equal(one["qh"][0], four["qh"][t])
