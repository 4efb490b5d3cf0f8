"""GPU parity of the FP8 output layer through the C ABI against the float64
oracle (oracle/lmhead.py) on the same seeded inputs: FP8 codes and row
scales of the weights bit-exact; logits within the float32 accumulation
bound of the tensor cores; at full size (157,184 x 2,560) every logit and
the top token.

Tolerance: the tensor core sums the 32 exact products of each MMA step and
adds the step into a float32 accumulator, H/32 = 80 roundings of partial
sums bounded by the sum of |products|, at most 2^-23 each (a truncating
adder; 2^-24 when rounding to nearest); then two float32 roundings for the
scales.  So |gpu - ref| <= 80 * 2^-23 * S + 2 * 2^-24 * |ref| with S the
scaled sum of |products| (oracle.lmhead.lmhead_abs_sum); the test uses
1e-5 * S + 2e-7 * |ref|."""
import numpy as np
import pytest
import torch

import mxfp4_expert_layers_b200 as moe
import synth
import synth.gpu
from oracle import lmhead as LH

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU collection
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

H = 2560


def _layer(V, seed=0):
    w = torch.empty((V, H), dtype=torch.int16, device="cuda")
    synth.gpu.fill_lmhead(w, seed, V, H)
    q = torch.empty((V, H), dtype=torch.uint8, device="cuda")
    s = torch.empty((V,), dtype=torch.float32, device="cuda")
    moe.moe_lmhead_quantize(w, V, H, q, s)
    torch.cuda.synchronize()
    return w, q, s


def _logits(q, s, V, x_bits):
    T = x_bits.shape[0]
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    out = torch.empty((T, V), dtype=torch.float32, device="cuda")
    moe.moe_lmhead_logits(q, s, V, H, x, T, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _check(got, q, s, x_bits):
    ref = LH.lmhead_logits(q, s, x_bits)
    S = LH.lmhead_abs_sum(q, s, x_bits)
    err = np.abs(got - ref)
    assert np.all(err <= 1e-5 * S + 2e-7 * np.abs(ref)), float((err / (S + 1e-30)).max())
    return ref


def test_gpu_lmhead_fill_and_quantize_match_host():
    V = 1000
    w, q, s = _layer(V, seed=3)
    wh = synth.lmhead_weight(3, V, H)
    assert np.array_equal(w.cpu().numpy().view(np.uint16), wh)
    qr, sr = LH.lmhead_quantize(wh)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(s.cpu().numpy(), sr)


@pytest.mark.parametrize("T", [1, 3, 8])
def test_gpu_lmhead_logits_ragged_vocab(T):
    V = 4099  # not a multiple of the 16-row groups
    _, q, s = _layer(V, seed=1)
    qh, sh = q.cpu().numpy(), s.cpu().numpy()
    x = synth.hidden_states(1, 50 + T, T, H)
    _check(_logits(q, s, V, x), qh, sh, x)


def test_gpu_lmhead_full_vocab_every_logit_and_top_token():
    V = 157184
    _, q, s = _layer(V, seed=0)
    x = synth.hidden_states(0, 77, 2, H)
    got = _logits(q, s, V, x)
    qh, sh = q.cpu().numpy(), s.cpu().numpy()
    ref = np.empty_like(got)
    for r0 in range(0, V, 16384):  # the oracle in slices of the vocabulary
        ref[:, r0:r0 + 16384] = _check(got[:, r0:r0 + 16384], qh[r0:r0 + 16384], sh[r0:r0 + 16384], x)
    for t in range(2):
        top = int(np.argmax(ref[t]))
        second = np.partition(ref[t], -2)[-2]
        if ref[t, top] - second > 1e-3 * abs(ref[t, top]):  # unambiguous winner
            assert int(np.argmax(got[t])) == top


def test_gpu_lmhead_argument_errors():
    q = torch.zeros((16, 128), dtype=torch.uint8, device="cuda")
    s = torch.ones((16,), dtype=torch.float32, device="cuda")
    x = torch.zeros((9, 128), dtype=torch.int16, device="cuda")
    out = torch.empty((9, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_lmhead_logits(q, s, 16, 128, x, 9, out)
    assert ei.value.code == moe.MOE_ERR_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_lmhead_logits(q, s, 16, 96, x, 1, out)
    assert ei.value.code == moe.MOE_ERR_SHAPE
    w = torch.zeros((16, 128), dtype=torch.int16, device="cuda")
    moe.moe_lmhead_quantize(w, 16, 128, q, s)
    moe.moe_lmhead_logits(q, s, 16, 128, x, 2, out)
    torch.cuda.synchronize()
    assert torch.all(s == 1.0) and torch.all(out[:2] == 0.0)
