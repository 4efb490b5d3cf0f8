"""GPU parity of the many-token path (T > MOE_GEMV_MAX_TOKENS: dispatch and
grouped GEMMs), through the C ABI, against the float64 oracle on the same
seeded inputs, for both kernel sets:
  - tcgen05 (block-scaled MMA, float32 accumulation in tensor memory): ids
    and counts bit-exact, FP8 bytes of x bit-exact, h within the float32
    accumulation tolerance, FP8 codes of h equal up to one-step flips at
    rounding boundaries, y within the layer tolerance;
  - mma.sync with exact block sums: as above, and h bit-exact like the
    decode path's."""
import numpy as np
import pytest
import torch

import mxfp4_expert_layers_b200 as moe
import synth
from oracle import formats as OF
from oracle import moe as OM

from moe_testlib import (GpuLayer, check_forward, check_forward_tc, check_route, oracle_forward, to_dev_u16, u16,
                         H0, REL_L2, MAX_ABS)

KERNELS = {"tc": (moe.MOE_PREFILL_TCGEN05, 3), "exact": (moe.MOE_PREFILL_EXACT, 2)}

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU collection
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def _run(layer: GpuLayer, x_bits, mode="split", debug=True, path=3):
    T = x_bits.shape[0]
    xd = to_dev_u16(x_bits)
    if mode == "split":
        ids, w, counts = layer.route(xd, T)
        y, dbg = layer.forward(xd, T, ids, w, debug)
    else:
        ids, w, counts, y, dbg = layer.decode(xd, T, debug)
    torch.cuda.synchronize()
    assert moe.moe_device_error(layer.handle) == moe.MOE_OK
    assert moe.moe_last_path(layer.handle) == path
    return ids, w, counts, y, dbg


@pytest.mark.parametrize("kernel", ["tc", "exact"])
@pytest.mark.parametrize("mode", ["split", "fused"])
@pytest.mark.parametrize("n_shared", [0, 1, 2])
@pytest.mark.parametrize("T", [5, 16, 37, 200])
def test_gpu_prefill_small_shapes(T, n_shared, mode, kernel):
    """H 128 / I 64: one partial K chunk; T = 200 gives the shared experts two
    N tiles of tokens (128 + 72)."""
    E, H, I, k = 8, 128, 64, 2
    kind, path = KERNELS[kernel]
    L = GpuLayer(7, T, E, H, I, k=k, n_shared=n_shared, fill="host", max_tokens=256, prefill=kind)
    try:
        for step in range(2):
            x = synth.hidden_states(7, 100 * T + step, T, H)
            ids, w, counts, y, dbg = _run(L, x, mode, path=path)
            ref = OM.moe_layer(x, L.host, E, k, I, n_shared)
            check_route(ids, w, counts, ref)
            if kernel == "exact":
                check_forward(y, dbg, ref)
            else:
                check_forward_tc(y, dbg, ref)
    finally:
        L.close()


@pytest.mark.parametrize("kernel", ["tc", "exact"])
def test_gpu_prefill_full_width_e32(kernel):
    """40 tokens through an E = 32 layer at full width (H 2560, I 768): ten
    full K chunks for gate/up, three for down."""
    kind, path = KERNELS[kernel]
    L = GpuLayer(0, 9, 32, max_tokens=64, prefill=kind)
    try:
        x = synth.hidden_states(0, 555, 40, H0)
        ids, w, counts, y, dbg = _run(L, x, path=path)
        ref = OM.moe_layer(x, L.host, 32, 8, L.I, 1)
        check_route(ids, w, counts, ref)
        if kernel == "exact":
            st = check_forward(y, dbg, ref)
            assert st["h_exact"] == 1.0, st
        else:
            st = check_forward_tc(y, dbg, ref)
        print(kernel, st)
    finally:
        L.close()


def test_gpu_prefill_tc_equals_exact_closely():
    """Both kernel sets on the same 300-token E = 64 call: identical routing,
    y within the layer tolerance of each other."""
    T = 300
    a = GpuLayer(1, 2, 64, max_tokens=T, prefill=moe.MOE_PREFILL_TCGEN05)
    b = GpuLayer(1, 2, 64, max_tokens=T, prefill=moe.MOE_PREFILL_EXACT)
    try:
        x = synth.hidden_states(1, 77, T, H0)
        _, _, ca, ya, _ = _run(a, x, "fused", debug=False, path=3)
        _, _, cb, yb, _ = _run(b, x, "fused", debug=False, path=2)
        assert torch.equal(ca, cb)
        yg, yr = OF.bf16_to_f64(u16(ya)), OF.bf16_to_f64(u16(yb))
        rel = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
        assert rel <= REL_L2 / 4, rel
    finally:
        a.close()
        b.close()


def test_gpu_prefill_config4_sampled():
    """The chunked-prefill workload: 512 tokens through an E = 512 layer with
    the Zipf(1.1) router bias.  Routing of all tokens against the oracle;
    outputs against the oracle on 64 sampled tokens plus every token routed
    to the most popular expert (each token's output depends on its own
    routing only)."""
    T = 512
    L = GpuLayer(0, 4, 512, bias=True, max_tokens=T)
    try:
        x = synth.hidden_states(0, 7000, T, H0)
        ids, w, counts, y, _ = _run(L, x, debug=False, path=3)
        _, rids, rw, rcounts = OM.route(x, L.host, 8)
        assert np.array_equal(ids.cpu().numpy(), rids)
        assert np.array_equal(counts.cpu().numpy(), rcounts)
        assert np.allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)
        assert (rcounts > 0).sum() >= 32  # the skewed routing still touches many experts
        top = int(np.argmax(rcounts))
        rng = np.random.default_rng(3)
        sample = np.union1d(rng.choice(T, 64, replace=False), np.nonzero((rids == top).any(axis=1))[0])
        assert len(sample) >= 64 + 1 and rcounts[top] > 8, (len(sample), rcounts[top])
        ref = oracle_forward(L.host, x[sample], rids[sample], rw[sample], 512, L.I, 1)
        yg = OF.bf16_to_f64(u16(y)[sample])
        yr = OF.bf16_to_f64(ref["y"])
        rel = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
        mx = np.abs(yg - yr).max() / np.abs(yr).max()
        assert rel <= REL_L2 and mx <= MAX_ABS, (rel, mx)
        assert np.mean(u16(y)[sample] == ref["y"]) >= 0.9
    finally:
        L.close()


def test_gpu_prefill_limits():
    L = GpuLayer(0, 0, 8, 128, 64, k=2, fill="host", max_tokens=4)
    try:
        x = to_dev_u16(np.zeros((8, 128), np.uint16))
        ids = torch.zeros((8, 2), dtype=torch.int32, device="cuda")
        w = torch.zeros((8, 2), dtype=torch.float32, device="cuda")
        y = torch.empty((8, 128), dtype=torch.int16, device="cuda")
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_forward(L.handle, x, 5, ids, w, y)
        assert ei.value.code == moe.MOE_ERR_ARG  # above the handle's max_tokens
    finally:
        L.close()


def test_gpu_prefill_kernel_selection():
    L = GpuLayer(0, 0, 8, 64, 64, k=2, fill="host", max_tokens=16)
    try:
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_set_prefill_kernel(L.handle, 7)
        assert ei.value.code == moe.MOE_ERR_ARG
        # hidden 64 is not a whole number of 128-row M tiles of the down GEMM
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_set_prefill_kernel(L.handle, moe.MOE_PREFILL_TCGEN05)
        assert ei.value.code == moe.MOE_ERR_UNSUPPORTED
        moe.moe_set_prefill_kernel(L.handle, moe.MOE_PREFILL_AUTO)
        x = synth.hidden_states(0, 1, 9, 64)
        ids, w, counts, y, dbg = _run(L, x, path=2)  # AUTO falls back to the mma.sync kernels
        ref = OM.moe_layer(x, L.host, 8, 2, 64, 1)
        check_route(ids, w, counts, ref)
        check_forward(y, dbg, ref)
    finally:
        L.close()
