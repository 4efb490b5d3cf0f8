"""Expert parallelism for the decode layer: the routed experts of one layer
split over the GPUs of a process group, the router replicated.

The layer shards naturally by expert: a token uses top_k of the routed
experts (8 of 512 in the layer of "NVIDIA 在单台 DGX Spark 上叠加三项优化…",
tanhow.com, section "Ling 3.0 是什么"), so each GPU holds a contiguous range
of them (plus, on one GPU, the shared experts) and computes its part of y
(``moe_decode_partial``, float32); the parts are summed across the group and
rounded once to BF16 (``moe_round_bf16``).  Every GPU computes the same
routing.  This module holds the partition, the slicing of a layer's packed
weights and the reduction; the arithmetic runs in the library's kernels and
the sum in the group's all-reduce (NCCL on GPUs).
"""
from __future__ import annotations

from . import (moe_create_ep, moe_decode_partial, moe_round_bf16)


def expert_range(n_experts: int, world: int, rank: int) -> tuple[int, int]:
    """Routed experts ``[lo, hi)`` of ``rank``: contiguous, sizes differing by
    at most one, covering 0 .. n_experts-1 once over the ranks."""
    if world < 1 or not 0 <= rank < world or n_experts < world:
        raise ValueError("need 0 <= rank < world <= n_experts")
    return rank * n_experts // world, (rank + 1) * n_experts // world


def holds_shared(rank: int) -> bool:
    """The shared experts are added by rank 0 alone."""
    return rank == 0


def local_weights(layer: dict, n_experts: int, n_shared: int, lo: int, hi: int, with_shared: bool) -> dict:
    """The handle weights of one rank from a whole layer's (``router_w``,
    ``router_bias``, packed ``w13`` / ``w2`` indexed [expert] with the shared
    experts after the routed ones): the routed experts lo..hi-1, then the
    shared ones when ``with_shared``, each a new contiguous tensor."""
    import torch
    out = {"router_w": layer["router_w"], "router_bias": layer.get("router_bias")}
    for key in ("w13", "w2"):
        parts = [layer[key][lo:hi]]
        if with_shared and n_shared:
            parts.append(layer[key][n_experts:n_experts + n_shared])
        out[key] = torch.cat(parts).contiguous()
    return out


def reduce_parts(y_part, group=None) -> None:
    """Sum the float32 parts of y over the group, in place."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(y_part, op=dist.ReduceOp.SUM, group=group)


class ExpertParallelLayer:
    """One rank's share of a layer: ``decode`` routes T <= 4 tokens, runs the
    rank's experts, sums the parts over the group and rounds to BF16."""

    def __init__(self, hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int, layer: dict,
                 rank: int, world: int, group=None, max_tokens: int = 4):
        self.H, self.E, self.k = hidden, n_experts, top_k
        self.lo, self.hi = expert_range(n_experts, world, rank)
        self.shared = holds_shared(rank)
        self.weights = local_weights(layer, n_experts, n_shared, self.lo, self.hi, self.shared)
        self.group = group
        self.handle = moe_create_ep(hidden, inter, n_experts, top_k, n_shared, self.weights, max_tokens,
                                    self.lo, self.hi, self.shared)

    def decode(self, x, T: int, stream=None):
        import torch
        ids = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        part = torch.empty((T, self.H), dtype=torch.float32, device=x.device)
        moe_decode_partial(self.handle, x, T, ids, w, part, None, stream)
        reduce_parts(part, self.group)
        y = torch.empty((T, self.H), dtype=torch.int16, device=x.device)
        moe_round_bf16(part, T * self.H, y, stream)
        return ids, w, y

    def close(self):
        from . import moe_destroy
        if self.handle:
            moe_destroy(self.handle)
            self.handle = None
