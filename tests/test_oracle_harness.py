"""Pins of the chained-layer harness step (oracle.moe.residual_rmsnorm) and
of the down-projection replay helper (oracle.moe.down_replay) against what
their definitions fix: torch's bfloat16 addition, a high-precision decimal
evaluation of the RMS normalisation, a constant vector's closed form, and the
replay equal to the down GEMV of the layer."""
from decimal import Decimal, getcontext

import numpy as np
import torch

import synth
from oracle import formats as OF
from oracle import moe as M


def test_residual_add_is_one_bf16_rounding_of_the_sum():
    r = synth.hidden_states(0, 1, 3, 256)
    y = synth.hidden_states(0, 2, 3, 256)
    rr, _ = M.residual_rmsnorm(r, y)
    tr = torch.from_numpy(r.view(np.int16)).view(torch.bfloat16)
    ty = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16)
    # torch adds bfloat16 in float32 and rounds once; every sum of two of these
    # bfloat16 values is exact in float32, so the two definitions agree
    ref = (tr.float() + ty.float()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(rr, ref)


def test_rmsnorm_against_decimal_evaluation():
    getcontext().prec = 50
    r = synth.hidden_states(3, 4, 2, 64)
    y = np.zeros_like(r)
    rr, x = M.residual_rmsnorm(r, y, eps=1e-6)
    assert np.array_equal(rr, r)  # adding zeros
    eps = Decimal(float(np.float32(1e-6)))
    for t in range(2):
        vals = [Decimal(float(v)) for v in OF.bf16_to_f64(r[t])]
        den = (sum(v * v for v in vals) / Decimal(64) + eps).sqrt()
        exact = np.array([float(v / den) for v in vals])
        # one BF16 rounding of a value within float64 error of the exact quotient
        want = OF.f64_to_bf16(exact)
        assert np.array_equal(x[t], want)


def test_rmsnorm_of_a_constant_vector():
    r = OF.f64_to_bf16(np.full((1, 128), 3.0))
    _, x = M.residual_rmsnorm(r, np.zeros_like(r), eps=1e-6)
    # 3 / sqrt(9 + 1e-6) = 1 - 5.6e-8: rounds to exactly 1 in BF16
    assert np.all(OF.bf16_to_f64(x) == 1.0)


def test_down_replay_is_the_down_gemv():
    ex = synth.expert_weights(0, 0, 3, 128, 64)
    h = np.asarray(np.random.default_rng(1).normal(size=(1, 64)), np.float32)
    qh, sh = M.quantize_fp8(h)
    got = M.down_replay(ex, qh[0], sh[0])
    W = OF.dequant_mxfp4(ex["w2_codes"], ex["w2_scales"])
    ref = (W @ OF.e4m3_value(qh[0]).astype(np.float64)) * float(sh[0])
    assert np.allclose(got, ref, rtol=1e-15, atol=0)
