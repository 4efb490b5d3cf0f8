"""Expert parallelism on one GPU: the parts of y that 2 and 4 ranks' handles
compute (moe_decode_partial, each holding a contiguous range of the routed
experts, rank 0 also the shared one), summed and rounded once to BF16,
against moe_decode of the whole layer.  The ranks run one after another:
nothing waits on another rank."""
import numpy as np
import pytest
import torch

import mxfp4_expert_layers_b200 as moe
from mxfp4_expert_layers_b200 import ep
import synth
from oracle import formats as OF

from moe_testlib import GpuLayer, to_dev_u16, u16, REL_L2, MAX_ABS, H0, I0

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU collection
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("T", [1, 4])
def test_gpu_ep_parts_sum_to_the_layer(world, T):
    E, k, S = 64, 8, 1
    L = GpuLayer(12, world, E, bias=True)
    layer = {"router_w": L.t["router_w"], "router_bias": L.t["router_bias"], "w13": L.t["w13"], "w2": L.t["w2"]}
    ranks = [ep.ExpertParallelLayer(H0, I0, E, k, S, layer, r, world) for r in range(world)]
    try:
        for step in range(2):
            x = to_dev_u16(synth.hidden_states(12, 50 + 10 * T + step, T, H0))
            ids_ref, w_ref, _, y_ref, _ = L.decode(x, T, debug=False)
            total = torch.zeros((T, H0), dtype=torch.float32, device="cuda")
            for rk in ranks:
                ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
                w = torch.empty((T, k), dtype=torch.float32, device="cuda")
                part = torch.full((T, H0), float("nan"), dtype=torch.float32, device="cuda")
                moe.moe_decode_partial(rk.handle, x, T, ids, w, part)
                torch.cuda.synchronize()
                assert moe.moe_device_error(rk.handle) == moe.MOE_OK
                assert torch.equal(ids, ids_ref) and torch.equal(w, w_ref)
                assert torch.isfinite(part).all()
                total += part
            y = torch.empty((T, H0), dtype=torch.int16, device="cuda")
            moe.moe_round_bf16(total, T * H0, y)
            torch.cuda.synchronize()
            a, b = OF.bf16_to_f64(u16(y)), OF.bf16_to_f64(u16(y_ref))
            rel = np.linalg.norm(a - b) / np.linalg.norm(b)
            mx = np.abs(a - b).max() / np.abs(b).max()
            assert rel <= REL_L2 / 4 and mx <= MAX_ABS, (rel, mx)
            assert np.mean(u16(y) == u16(y_ref)) >= 0.95
    finally:
        for rk in ranks:
            rk.close()
        L.close()


def test_gpu_ep_rank_without_experts_of_the_token_gives_zero():
    """A rank holding none of a token's routed experts and not the shared one
    contributes exactly zero."""
    E, k, S, world = 64, 8, 1, 4
    L = GpuLayer(13, 0, E)
    layer = {"router_w": L.t["router_w"], "router_bias": None, "w13": L.t["w13"], "w2": L.t["w2"]}
    ranks = [ep.ExpertParallelLayer(H0, I0, E, k, S, layer, r, world) for r in range(world)]
    try:
        for step in range(8):
            x = to_dev_u16(synth.hidden_states(13, step, 1, H0))
            ids, _, _, _, _ = L.decode(x, 1, debug=False)
            held = [any(rk.lo <= int(e) < rk.hi for e in ids[0].tolist()) for rk in ranks]
            for rk, h in zip(ranks[1:], held[1:]):
                if h:
                    continue
                i2 = torch.empty((1, k), dtype=torch.int32, device="cuda")
                w2 = torch.empty((1, k), dtype=torch.float32, device="cuda")
                part = torch.full((1, H0), float("nan"), dtype=torch.float32, device="cuda")
                moe.moe_decode_partial(rk.handle, x, 1, i2, w2, part)
                torch.cuda.synchronize()
                assert torch.count_nonzero(part) == 0
                return
        pytest.skip("every rank held one of the tokens' experts")
    finally:
        for rk in ranks:
            rk.close()
        L.close()


def test_gpu_ep_handle_rejects_whole_layer_calls():
    E = 16
    L = GpuLayer(14, 0, E, 128, 64, k=2, fill="host")
    layer = {"router_w": L.t["router_w"], "router_bias": None, "w13": L.t["w13"], "w2": L.t["w2"]}
    rk = ep.ExpertParallelLayer(128, 64, E, 2, 1, layer, 1, 2)
    try:
        x = to_dev_u16(synth.hidden_states(14, 0, 1, 128))
        ids = torch.empty((1, 2), dtype=torch.int32, device="cuda")
        w = torch.empty((1, 2), dtype=torch.float32, device="cuda")
        y = torch.empty((1, 128), dtype=torch.int16, device="cuda")
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_decode(rk.handle, x, 1, ids, w, y)
        assert ei.value.code == moe.MOE_ERR_UNSUPPORTED
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_create_ep(128, 64, E, 2, 1, layer, 4, 5, 3, False)
        assert ei.value.code == moe.MOE_ERR_ARG
    finally:
        rk.close()
        L.close()
