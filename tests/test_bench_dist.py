"""Host logic of bench.py's multi-rank path on CPU: two gloo ranks (the GPU
runs use NCCL with the same calls).  The timing that a multi-GPU run reports
is the maximum over the ranks, the value is the whole job's tokens over that
time, and only rank 0 runs and prints the reference arm."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's own time; every rank must get the largest
        out[rank] = bench.max_over_ranks(10.0 + 3.0 * rank, "cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 13.0, 1: 13.0}


def test_max_over_ranks_without_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(7.5, "cpu") == 7.5


def test_per_token_value_counts_every_rank():
    # 200 steps of 1 token through 64 layers in 480 ms on each of 4 ranks
    one = bench.per_token_value(480.0, 200, 64, 1, 1)
    assert one == pytest.approx(480e3 / (200 * 64))
    assert bench.per_token_value(480.0, 200, 64, 1, 4) == pytest.approx(one / 4)
    # 4-token calls: per token
    assert bench.per_token_value(480.0, 200, 64, 4, 1) == pytest.approx(one / 4)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")

    def boom(*a, **k):  # pragma: no cover - must not be reached
        raise AssertionError("rank 1 ran the oracle")

    monkeypatch.setattr(bench, "oracle_sample", boom)
    args = bench.argparse.Namespace(impl="reference", gpus=2, steps=1, warmup=0, workload="layer", layers=64,
                                    no_cpu_baseline=True, prefill_kernel="auto")
    bench.run_reference(args)
    assert capsys.readouterr().out == ""
