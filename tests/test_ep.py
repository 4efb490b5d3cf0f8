"""Expert parallelism, host side (CPU): the partition of the routed experts
over the ranks, and the reduction of the ranks' parts of y across a process
group -- two gloo ranks, each computing its part with the float64 oracle.
The sum of the parts, rounded once to BF16, must equal the oracle's y of the
whole layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mxfp4_expert_layers_b200 import ep


def test_expert_range_partitions_the_experts():
    for E in (8, 32, 512, 513):
        for world in (1, 2, 3, 4, 8):
            if world > E:
                continue
            ranges = [ep.expert_range(E, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == E
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        ep.expert_range(4, 8, 0)
    assert ep.holds_shared(0) and not ep.holds_shared(1)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_part(rank, world, x, layer_seed, E, H, I, k, S):
    """This rank's float64 part of y from the oracle: its routed experts'
    weighted outputs, plus the shared experts on rank 0."""
    import synth
    from oracle import moe as M
    lw = M.LayerWeights(router_w=synth.router_weight(layer_seed, 0, E, H), router_bias=None)
    _, ids, w, _ = M.route(x, lw, k)
    lo, hi = ep.expert_range(E, world, rank)
    xq, xs = M.quantize_fp8(M.bf16_to_f64(x).astype(np.float32))
    part = np.zeros((x.shape[0], H))
    for t in range(x.shape[0]):
        slots = [(int(e), float(p)) for e, p in zip(ids[t], w[t]) if lo <= e < hi]
        if ep.holds_shared(rank):
            slots += [(E + s, 1.0) for s in range(S)]
        for e, p in slots:
            d, *_ = M.expert_ffn(synth.expert_weights(layer_seed, 0, e, H, I), xq[t], xs[t], I)
            part[t] += p * d
    return part, ids


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import synth
        E, H, I, k, S = 16, 128, 64, 4, 1
        x = synth.hidden_states(21, 3, 3, H)
        part, ids = _rank_part(rank, world, x, 21, E, H, I, k, S)
        t = torch.from_numpy(part)
        ep.reduce_parts(t)
        out[rank] = (t.numpy().copy(), ids)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_parts_sum_to_the_whole_layer_over_gloo(world):
    import synth
    from oracle import formats as F
    from oracle import moe as M
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    E, H, I, k, S = 16, 128, 64, 4, 1
    x = synth.hidden_states(21, 3, 3, H)
    lw = M.LayerWeights(router_w=synth.router_weight(21, 0, E, H), router_bias=None)
    for e in range(E + S):
        lw.experts[e] = synth.expert_weights(21, 0, e, H, I)
    ref = M.moe_layer(x, lw, E, k, I, S)
    for r in range(world):
        y_sum, ids = res[r]
        assert np.array_equal(ids, ref["ids"])          # every rank routes the same
        assert np.allclose(y_sum, ref["y64"], rtol=1e-12, atol=1e-12)
        assert np.array_equal(F.f64_to_bf16(y_sum), ref["y"])
