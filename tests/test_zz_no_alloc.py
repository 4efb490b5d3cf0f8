"""The entry point that allocates nothing (moe_forward_static) against the
handle-based moe_forward on the same inputs.

moe_forward_static serves host code that cannot allocate device memory; its
scratch lives in a fixed array inside the library that every call shares.
This file sorts last so that a run stopping at the first failure has run
everything else before it; the test also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import mxfp4_expert_layers_b200 as moe
import synth
from oracle import formats as OF

from moe_testlib import GpuLayer, to_dev_u16, u16, REL_L2, MAX_ABS

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU collection
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


@pytest.mark.parametrize("T", [1, 4])
def test_static_forward_matches_handle_forward_twice(T):
    E, H, I = 32, 2560, 768
    L = GpuLayer(11, 0, E, H, I, k=8, n_shared=1)
    try:
        for call in range(2):  # two calls in a row share the one scratch array
            x = to_dev_u16(synth.hidden_states(11, 100 + 10 * T + call, T, H))
            ids, w, _ = L.route(x, T)
            y_ref, _ = L.forward(x, T, ids, w, debug=False)
            y = torch.full((T, H), -1, dtype=torch.int16, device="cuda")
            moe.moe_forward_static(H, I, E, 8, 1, L.t, x, T, ids, w, y, torch.cuda.current_stream())
            torch.cuda.synchronize()
            a = OF.bf16_to_f64(u16(y))
            b = OF.bf16_to_f64(u16(y_ref))
            rel = np.linalg.norm(a - b) / np.linalg.norm(b)
            mx = np.abs(a - b).max() / np.abs(b).max()
            assert rel <= REL_L2 and mx <= MAX_ABS, (call, rel, mx)
    finally:
        L.close()


def test_static_forward_rejects_sizes_beyond_its_array():
    cfg = dict(hidden=2560, inter=2048, n_experts=32, top_k=8, n_shared=1)
    w = {"router_w": 0x1000, "router_bias": None, "w13": 0x1000, "w2": 0x1000}
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward_static(*cfg.values(), w, 0x1000, 1, 0x1000, 0x1000, 0x1000)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward_static(2560, 768, 32, 8, 1, w, 0x1000, 5, 0x1000, 0x1000, 0x1000)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED


def test_static_forward_reports_bad_ids():
    """An expert id outside 0..E-1 is skipped and reported by
    moe_forward_static_device_error (then cleared); the next call is clean."""
    E, H, I = 8, 128, 64
    L = GpuLayer(4, 0, E, H, I, k=2, fill="host")
    try:
        x = to_dev_u16(synth.hidden_states(4, 0, 1, H))
        y = torch.empty((1, H), dtype=torch.int16, device="cuda")
        w = torch.tensor([[0.75, 0.25]], dtype=torch.float32, device="cuda")
        bad = torch.tensor([[1, 99]], dtype=torch.int32, device="cuda")
        moe.moe_forward_static(H, I, E, 2, 1, L.t, x, 1, bad, w, y, torch.cuda.current_stream())
        assert moe.moe_forward_static_device_error() == moe.MOE_ERR_DEVICE
        assert moe.moe_forward_static_device_error() == moe.MOE_OK
        good = torch.tensor([[1, 5]], dtype=torch.int32, device="cuda")
        moe.moe_forward_static(H, I, E, 2, 1, L.t, x, 1, good, w, y, torch.cuda.current_stream())
        assert moe.moe_forward_static_device_error() == moe.MOE_OK
        y_ref, _ = L.forward(x, 1, good, w, debug=False)
        torch.cuda.synchronize()
        assert np.array_equal(u16(y), u16(y_ref))
    finally:
        L.close()
