#!/usr/bin/env python
"""Benchmark of the MXFP4 MoE decode layer on B200.

Default workload (the metric's configuration): 512-expert layers (top-8 + 1
shared, hidden 2560, width 768, MXFP4 weights, FP8 activations), 64 distinct
seeded layers (103 GB) so the 126 MB L2 never holds a repeated layer.  A step
= one token through all 64 layers, chained by the residual + RMSNorm harness,
in one persistent launch (routing, experts and combine of every layer); the
value is microseconds per token per layer.  Prints one JSON line.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                  [--workload layer|verify4|stack42]

Under torchrun (N > 1) every rank runs its own independent layer set
(replicas: the path has no data exchange) and rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

H, I, E, K_TOP, N_SHARED = 2560, 768, 512, 8, 1
BYTES_PER_EXPERT = 2 * I * H // 2 + 2 * I * H // 32 + H * I // 2 + H * I // 32   # 3,133,440
LAYER_BYTES = (E + N_SHARED) * BYTES_PER_EXPERT + E * H * 2
METRIC = "MoE-layer decode us/token at B=1 and achieved HBM GB/s (% of B200 peak)"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="layer", choices=["layer", "verify4", "stack42", "prefill512", "lmhead"])
    p.add_argument("--layers", type=int, default=64)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--prefill-kernel", default="auto", choices=["auto", "tcgen05", "exact"],
                   help="grouped-GEMM kernels of the prefill512 workload")
    return p.parse_args()


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu --set full
# capture of each current kernel: decode_kernel on a 2-layer stack at T = 1
# (62.48 MB per launch, scaled per layer: traffic grows with the layers a
# launch runs), and tc_gemm_kernel<0> + tc_gemm_kernel<1> of one 512-token
# prefill call (Zipf routing, 103 + 1 experts touched).
NCU_DECODE_DRAM_BYTES_PER_LAYER = 62.478592e6 / 2
NCU_PREFILL_GEMM_DRAM_BYTES = 228.321024e6 + 11.817728e6 + 116.868352e6 + 3.162112e6
# lmhead_gemv_kernel, one 157,184 x 2,560 call (T = 1)
NCU_LMHEAD_DRAM_BYTES = 403.072768e6 + 3.427328e6


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------- clocks --
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.lines: list[str] = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- layers --
class Layers:
    """``n`` seeded E=512 layers resident in HBM, one library handle each."""

    def __init__(self, n, bias=False, max_tokens=4):
        import torch
        import mxfp4_expert_layers_b200 as moe
        import synth.gpu
        free, _ = torch.cuda.mem_get_info()
        fit = int((free - (6 << 30)) // LAYER_BYTES)
        self.requested = n
        self.n = max(1, min(n, fit))
        self.bufs, self.handles = [], []
        nexp = E + N_SHARED
        # canonical weights are generated into one scratch set, then packed
        canon = {"w13_codes": torch.empty((nexp, 2 * I, H // 2), dtype=torch.uint8, device="cuda"),
                 "w13_scales": torch.empty((nexp, 2 * I, H // 32), dtype=torch.uint8, device="cuda"),
                 "w2_codes": torch.empty((nexp, H, I // 2), dtype=torch.uint8, device="cuda"),
                 "w2_scales": torch.empty((nexp, H, I // 32), dtype=torch.uint8, device="cuda")}
        for layer in range(self.n):
            t = {"router_w": torch.empty((E, H), dtype=torch.int16, device="cuda"),
                 "w13": torch.empty((nexp, I // 8, moe.w13_tile_bytes(H)), dtype=torch.uint8, device="cuda"),
                 "w2": torch.empty((nexp, H // 16, moe.w2_tile_bytes(I)), dtype=torch.uint8, device="cuda")}
            canon["router_w"] = t["router_w"]
            synth.gpu.fill_layer(canon, 0, layer, E, H, I, N_SHARED)
            moe.moe_pack_weights(H, I, E, K_TOP, N_SHARED, canon, 0, nexp, t["w13"], t["w2"])
            if bias:
                import synth as S
                t["router_bias"] = torch.from_numpy(S.zipf_router_bias(0, layer, E)).cuda()
            self.bufs.append(t)
            self.handles.append(moe.moe_create(H, I, E, K_TOP, N_SHARED, t, max_tokens))
        del canon
        torch.cuda.synchronize()

    def close(self):
        import mxfp4_expert_layers_b200 as moe
        for h in self.handles:
            moe.moe_destroy(h)
        self.handles = []


def alg_bytes(T: int, distinct_routed: int):
    """Algorithmic bytes of one layer call (one decode launch): weights of the
    distinct experts touched (routed + shared), the router, x in and y out,
    and the float32 h written by gate/up and read back for the down step."""
    U = distinct_routed + N_SHARED
    w13 = U * 2 * I * (H // 2 + H // 32)
    w2 = U * H * (I // 2 + I // 32)
    router = E * H * 2
    act = T * H * 2 * 2
    hbuf = U * T * I * 4 * 2
    return {"layer": w13 + w2 + router + act + hbuf, "weights": w13 + w2 + router}


# ----------------------------------------------------------- oracle arm --
def oracle_sample(n_tokens: int, T: int = 1, budget_s: float = 20.0):
    """Time the float64 oracle on the host cores on a bounded sample of the
    same workload: ``n_tokens`` calls of T tokens through layers 0, 1, ...
    (weights regenerated outside the timed region)."""
    import synth
    from oracle import moe as OM
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        cores = 1
    times = []
    for i in range(n_tokens):
        layer = i % 64
        x = synth.hidden_states(0, 1000 + i, T, H)
        lw = OM.LayerWeights(router_w=synth.router_weight(0, layer, E, H), router_bias=None)
        _, ids, _, _ = OM.route(x, lw, K_TOP)
        for e in set(ids.ravel().tolist()) | {E}:
            lw.experts[e] = synth.expert_weights(0, layer, e, H, I)
        t0 = time.perf_counter()
        OM.moe_layer(x, lw, E, K_TOP, I, N_SHARED)
        times.append(time.perf_counter() - t0)
        if sum(times) > budget_s:
            break
    return {"us_per_token": 1e6 * sum(times) / (len(times) * T), "cores": cores,
            "sample": f"{len(times)} call(s) of {T} token(s), E=512 layers, float64 numpy oracle"}


def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def per_token_value(ms_total: float, steps: int, layers: int, tokens: int, world: int) -> float:
    """Whole-job µs per token and layer: every rank pushed steps x tokens
    tokens through the layers within the (max over ranks) time."""
    return 1e3 * ms_total / (steps * layers) / (tokens * world)


def oracle_lmhead_sample(rows: int = 8192, budget_s: float = 20.0):
    """Time the float64 FP8 LM-head oracle on the host cores on ``rows`` of
    the 157,184-row vocabulary (weights quantised outside the timed region)
    and scale to the full vocabulary: µs per token."""
    import synth
    from oracle import lmhead as LH
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        cores = 1
    V = 157184
    q, s = LH.lmhead_quantize(synth.lmhead_weight(0, V, H, 0, rows))
    times = []
    for i in range(100):
        x = synth.hidden_states(0, 3000 + i, 1, H)
        t0 = time.perf_counter()
        LH.lmhead_logits(q, s, x)
        times.append(time.perf_counter() - t0)
        if sum(times) > budget_s:
            break
    return {"us_per_token": 1e6 * (sum(times) / len(times)) * V / rows, "cores": cores,
            "sample": f"{len(times)} token(s) through {rows} of {V} rows, scaled to the full vocabulary; "
                      "float64 numpy oracle"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    T = 4 if args.workload == "verify4" else 8 if args.workload == "prefill512" else 1
    t0 = time.perf_counter()
    # each step one token (or call) of the oracle, the whole run bounded to ~2 minutes
    if args.workload == "lmhead":
        res = oracle_lmhead_sample(budget_s=min(120.0, max(5.0, 2.0 * args.steps)))
    else:
        for _ in range(min(args.warmup, 2)):
            oracle_sample(1, T, 1e9)
        t0 = time.perf_counter()
        res = oracle_sample(args.steps, T, 120.0)
    el = time.perf_counter() - t0
    # the same value and unit as this workload's own arm
    value, unit = res["us_per_token"], "us/token"
    if args.workload == "stack42":
        value, unit = value * 42, "us/token (42-layer stack)"
    elif args.workload == "prefill512":
        unit = "us/token (512-token prefill call)"
    elif args.workload == "lmhead":
        unit = "us/token (FP8 LM head, 157184 x 2560)"
    line = {"metric": METRIC, "value": value, "unit": unit, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / max(args.steps, 1), "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args, None),
            "cpu_baseline": {"value": value, "unit": unit, "cores": res["cores"],
                             "kind": "oracle", "sample": res["sample"]},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(args, layers):
    n = layers.n if layers is not None else args.layers
    if args.workload == "layer":
        w = (f"1-token decode through {n} distinct E=512 top-8 + 1 shared layers (H=2560, I=768, MXFP4 W4A8), "
             "chained by the residual + RMSNorm harness, one persistent launch per token")
    elif args.workload == "verify4":
        w = f"4-token verify call (i.i.d. tokens) through {n} chained E=512 layers, one launch per call"
    elif args.workload == "prefill512":
        w = "chunked prefill: 512 tokens per call, E=512 top-8 + 1 shared, Zipf(1.1) bias"
    elif args.workload == "lmhead":
        w = "FP8 output layer: 157,184 x 2,560 weights quantised per row, 1 token per call"
    else:
        w = "42-layer decode stack, Zipf(1.1) router bias, residual + RMSNorm chain, one launch per token"
    c = {"workload": w, "layers_resident": n, "hidden": H, "inter": I, "experts": E, "top_k": K_TOP,
         "shared": N_SHARED,
         "l2": "inputs larger than L2: every layer distinct (" +
               f"{n * LAYER_BYTES / 1e9:.1f} GB resident)"}
    if layers is not None and layers.n < layers.requested:
        c["note"] = f"only {layers.n} of {layers.requested} layers fit in free HBM"
    return c


# ------------------------------------------------------------- our arm --
def run_ours(args):
    import torch
    import torch.distributed as dist
    import mxfp4_expert_layers_b200 as moe
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    moe.load()
    hbm_peak, peak_kind = peaks()

    T = 4 if args.workload == "verify4" else 1
    n_layers = 42 if args.workload == "stack42" else args.layers
    layers = Layers(n_layers, bias=(args.workload == "stack42"), max_tokens=4)
    L = layers.n
    stack = moe.moe_stack_create(layers.handles)
    stream = torch.cuda.current_stream()
    nsteps = args.warmup + args.steps

    # fresh tokens per step, resident in HBM before timing
    xs_host = np.stack([synth.hidden_states(0, 1000 + 7919 * rank + i, T, H) for i in range(min(nsteps, 512))])
    xs = torch.from_numpy(xs_host.view(np.int16)).cuda()
    r = torch.empty((T, H), dtype=torch.int16, device="cuda")
    x = torch.empty((T, H), dtype=torch.int16, device="cuda")
    ids = torch.empty((L, T, K_TOP), dtype=torch.int32, device="cuda")
    wts = torch.empty((L, T, K_TOP), dtype=torch.float32, device="cuda")

    def step(i, s):
        # one token (or verify call) through all L layers: one launch
        x0 = xs[i % xs.shape[0]]
        r.copy_(x0)
        x.copy_(x0)
        moe.moe_stack_decode(stack, r, x, T, 1e-6, ids, wts, None, s)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(args.warmup):
        step(i, stream)
    barrier()
    assert moe.moe_stack_device_error(stack) == moe.MOE_OK

    # ---- headline: a CUDA graph of the K steps (one stack launch each)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            for i in range(args.steps):
                step(args.warmup + i, cap)
    g.replay()
    barrier()
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    ev0.record(stream)
    g.replay()
    ev1.record(stream)
    barrier()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    assert moe.moe_stack_device_error(stack) == moe.MOE_OK
    ms = max_over_ranks(ms, "cuda")

    # ---- the stack kernel's own duration: events around every launch
    moe.moe_stack_profile_begin(stack, args.steps + 2)
    barrier()
    for i in range(args.warmup, nsteps):
        step(i, stream)
    barrier()
    dk_ms, dk_n = moe.moe_stack_profile_end(stack).get("decode", (0.0, 0))
    dk_us = 1e3 * dk_ms / max(dk_n, 1)

    # ---- one launch per layer (moe_decode on each handle), CUDA graph of one pass
    y1 = torch.empty((T, H), dtype=torch.int16, device="cuda")
    ids1 = torch.empty((T, K_TOP), dtype=torch.int32, device="cuda")
    w1 = torch.empty((T, K_TOP), dtype=torch.float32, device="cuda")
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g1, stream=cap):
            for li in range(L):
                moe.moe_decode(layers.handles[li], xs[li % xs.shape[0]], T, ids1, w1, y1, None, None, cap)
    g1.replay()
    barrier()
    reps = max(1, min(20, args.steps // 10))
    ev0.record(stream)
    for _ in range(reps):
        g1.replay()
    ev1.record(stream)
    barrier()
    per_call_us = 1e3 * ev0.elapsed_time(ev1) / (reps * L)

    distinct = len(set(ids[-1].cpu().numpy().ravel().tolist()))
    ab = alg_bytes(T, distinct if T > 1 else K_TOP)
    layer_us = 1e3 * ms / (args.steps * L)
    step_us = 1e3 * ms / args.steps
    if args.workload == "stack42":
        value = step_us / world                      # us per token through the 42-layer stack
    else:
        value = per_token_value(ms, args.steps, L, T, world)
    layer_gbs = ab["layer"] / (layer_us * 1e3)
    roof = {"bound": "hbm", "kernel": "decode_kernel", "achieved": L * ab["layer"] / (dk_us * 1e3),
            "peak": hbm_peak, "unit": "GB/s", "peak_kind": f"{peak_kind} copy bandwidth (burst)",
            "frac": L * ab["layer"] / (dk_us * 1e3) / hbm_peak,
            "traffic": (NCU_DECODE_DRAM_BYTES_PER_LAYER * L if T == 1 and args.workload != "stack42" else None),
            "alg_bytes_per_launch": L * ab["layer"], "avg_launch_us": dk_us, "launches_timed": dk_n,
            "layers_per_launch": L}

    # ---- e2e through the public API with pinned host buffers
    xh = torch.from_numpy(xs_host.view(np.int16)).pin_memory()
    xo = torch.empty((T, H), dtype=torch.int16).pin_memory()
    barrier()
    ev0.record(stream)
    for i in range(args.warmup, nsteps):
        r.copy_(xh[i % xh.shape[0]], non_blocking=True)
        x.copy_(r)
        moe.moe_stack_decode(stack, r, x, T, 1e-6, None, None, None, stream)
        xo.copy_(x, non_blocking=True)
    ev1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), "cuda")
    e2e_step_us = 1e3 * e2e_ms / args.steps
    e2e_val = (e2e_step_us if args.workload == "stack42" else e2e_step_us / (L * T)) / world

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res = oracle_sample(30, T, budget_s=20.0)
        cpu = {"value": res["us_per_token"] * (L if args.workload == "stack42" else 1),
               "unit": "us/token" if args.workload != "stack42" else "us/token (42-layer stack)",
               "cores": res["cores"], "kind": "oracle", "sample": res["sample"]}

    unit = "us/token" if args.workload != "stack42" else "us/token (42-layer stack)"
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "e2m1 x e4m3 operands, f32 block sums, f64 accumulation",
            "data": "synthetic (seeded SplitMix64 weights, Irwin-Hall normals)",
            "config": workload_config(args, layers),
            "layer_us": layer_us, "layer_gbs": layer_gbs, "layer_frac_of_peak": layer_gbs / hbm_peak,
            "layer_frac_of_8tbs": layer_gbs / 8000.0, "alg_bytes_per_layer": ab["layer"],
            "per_call_us": per_call_us, "per_call_note": "one moe_decode launch per layer (CUDA graph)",
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": T * H * 2,
                    "d2h_bytes_per_step": T * H * 2},
            "gpu_launches": args.steps, "clocks": clk,
            "timing": "CUDA graph of K steps; a step = the token(s) through all resident layers in one launch"}
    if args.workload == "verify4":
        line["us_per_call"] = layer_us
        line["distinct_experts_last_call"] = distinct
    if args.workload == "stack42":
        line["stack_tokens_per_s"] = 1e6 / value
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g, g1
    moe.moe_stack_destroy(stack)
    layers.close()
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------ prefill workload --
def run_prefill(args):
    """Chunked prefill: 512 tokens per call through an E = 512 layer with the
    Zipf(1.1) router bias (routing + dispatch + grouped GEMMs + combine)."""
    import torch
    import torch.distributed as dist
    import mxfp4_expert_layers_b200 as moe
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    moe.load()
    hbm_peak, peak_kind = peaks()
    T = 512
    layers = Layers(min(args.layers, 4), bias=True, max_tokens=T)
    L = layers.n
    kind = {"auto": moe.MOE_PREFILL_AUTO, "tcgen05": moe.MOE_PREFILL_TCGEN05,
            "exact": moe.MOE_PREFILL_EXACT}[args.prefill_kernel]
    for h in layers.handles:
        moe.moe_set_prefill_kernel(h, kind)
    xs_host = np.stack([synth.hidden_states(0, 20000 + 7919 * rank + i, T, H) for i in range(4)])
    xs = torch.from_numpy(xs_host.view(np.int16)).cuda()
    ids = torch.empty((T, K_TOP), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, K_TOP), dtype=torch.float32, device="cuda")
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i, s):
        moe.moe_decode(layers.handles[i % L], xs[i % xs.shape[0]], T, ids, wts, y, counts, None, s)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(args.warmup):
        step(i, stream)
    barrier()
    assert all(moe.moe_device_error(h) == moe.MOE_OK for h in layers.handles)
    touched = int((counts.cpu().numpy() > 0).sum()) + N_SHARED
    tc = moe.moe_last_path(layers.handles[0]) == 3
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            for i in range(args.steps):
                step(args.warmup + i, cap)
    g.replay()
    barrier()
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    ev0.record(stream)
    g.replay()
    ev1.record(stream)
    barrier()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    ms = max_over_ranks(ms, "cuda")
    # grouped GEMM kernels alone (gate/up .. down), events around them
    for h in layers.handles:
        moe.moe_profile_begin(h, args.steps + 2)
    barrier()
    for i in range(args.warmup, args.warmup + args.steps):
        step(i, stream)
    barrier()
    gm_ms, gm_n = 0.0, 0
    for h in layers.handles:
        t_ms, n = moe.moe_profile_end(h).get("grouped_gemm", (0.0, 0))
        gm_ms, gm_n = gm_ms + t_ms, gm_n + n
    gemm_us = 1e3 * gm_ms / max(gm_n, 1)
    call_us = 1e3 * ms / args.steps
    flops = 2.0 * 3 * H * I * T * (K_TOP + N_SHARED)
    bytes_ = touched * BYTES_PER_EXPERT + E * H * 2 + T * H * (2 + 1 + 2)
    P = T * (K_TOP + N_SHARED)
    # the grouped GEMMs (+ requant between them): weights of the touched experts,
    # the FP8 operand panels of x and h, h written and read back (float32), and
    # the float32 combine accumulator read-modify-written once per pair
    gemm_bytes = touched * BYTES_PER_EXPERT + P * (H + I) + 2 * P * I * 4 + 2 * T * H * 4
    fp8_peak = peaks_bf16() * 2.0
    gemm_gbs = gemm_bytes / (gemm_us * 1e3)
    line = {"metric": METRIC, "value": call_us / T, "unit": "us/token (512-token prefill call)", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("e2m1 x e4m3 operands (tcgen05 block-scaled MMA), f32 accumulation" if tc else
                      "e2m1 x e4m3 operands, f32 block sums, f64 accumulation"),
            "data": "synthetic (seeded SplitMix64 weights, Irwin-Hall normals)",
            "config": {"workload": "chunked prefill: 512 tokens per call, E=512 top-8 + 1 shared, Zipf(1.1) bias",
                       "layers_resident": L, "l2": "inputs larger than L2 (touched experts ~%d MB per call)" % (bytes_ // 1e6)},
            "us_per_call": call_us, "experts_touched": touched, "flops_per_call": flops, "bytes_per_call": bytes_,
            # 54 GFLOP on ~0.36 GB: 150 FLOP/B, below the B200 ridge (fp8 ~4.5 PFLOP/s / 6.5 TB/s
            # ~ 700 FLOP/B), so the grouped GEMMs are bounded by HBM; tensor-pipe figures beside it
            "roofline": {"bound": "hbm",
                         "kernel": ("tc_gemm_kernel<0>+requant_kernel+tc_gemm_kernel<1>" if tc else
                                    "gateup_kernel+requant_kernel+down_kernel"),
                         "achieved": gemm_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "peak_kind": peak_kind + " copy bandwidth (burst)", "frac": gemm_gbs / hbm_peak,
                         "traffic": NCU_PREFILL_GEMM_DRAM_BYTES if tc else None,
                         "alg_bytes_per_launch": gemm_bytes, "avg_launch_us": gemm_us,
                         "tensor_tflops": flops / (gemm_us * 1e6), "tensor_peak_tflops": fp8_peak,
                         "tensor_peak_kind": "measured bf16 cuBLAS burst x 2 (nominal fp8/bf16 ratio)",
                         "tensor_frac": flops / (gemm_us * 1e6) / fp8_peak,
                         "hbm_gbs_of_call": bytes_ / (call_us * 1e3)},
            "cpu_baseline": None, "gpu_launches": args.steps * 9, "clocks": clk,
            "timing": "CUDA graph of K calls (route + dispatch + grouped GEMMs + combine)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g
    layers.close()
    if world > 1:
        dist.destroy_process_group()


def run_lmhead(args):
    """FP8 output layer, 157,184 x 2,560, one token per call (the decode step's
    other weight-bound operation): quantised once, then K calls timed."""
    import torch
    import torch.distributed as dist
    import mxfp4_expert_layers_b200 as moe
    import synth
    import synth.gpu

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    moe.load()
    hbm_peak, peak_kind = peaks()
    V, T = 157184, 1
    w = torch.empty((V, H), dtype=torch.int16, device="cuda")
    synth.gpu.fill_lmhead(w, 0, V, H)
    q = torch.empty((V, H), dtype=torch.uint8, device="cuda")
    sw = torch.empty((V,), dtype=torch.float32, device="cuda")
    moe.moe_lmhead_quantize(w, V, H, q, sw)
    del w
    nsteps = args.warmup + args.steps
    xs_host = np.stack([synth.hidden_states(0, 3000 + 7919 * rank + i, T, H) for i in range(min(nsteps, 256))])
    xs = torch.from_numpy(xs_host.view(np.int16)).cuda()
    out = torch.empty((T, V), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i, s):
        moe.moe_lmhead_logits(q, sw, V, H, xs[i % xs.shape[0]], T, out, s)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(args.warmup):
        step(i, stream)
    barrier()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            for i in range(args.steps):
                step(args.warmup + i, cap)
    g.replay()
    barrier()
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    ev0.record(stream)
    g.replay()
    ev1.record(stream)
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), "cuda")
    clk = clocks.stop()
    # e2e: x from pinned host memory, logits back to pinned host memory, every call
    xh = torch.from_numpy(xs_host.view(np.int16)).pin_memory()
    oh = torch.empty((T, V), dtype=torch.float32).pin_memory()
    xd = torch.empty((T, H), dtype=torch.int16, device="cuda")
    barrier()
    ev0.record(stream)
    for i in range(args.steps):
        xd.copy_(xh[i % xh.shape[0]], non_blocking=True)
        moe.moe_lmhead_logits(q, sw, V, H, xd, T, out, stream)
        oh.copy_(out, non_blocking=True)
    ev1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), "cuda")
    call_us = 1e3 * ms / args.steps
    alg = V * H + V * 4 + T * H * 2 + T * V * 4
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res = oracle_lmhead_sample()
        cpu = {"value": res["us_per_token"], "unit": "us/token (FP8 LM head, 157184 x 2560)", "cores": res["cores"],
               "kind": "oracle", "sample": res["sample"]}
    gbs = alg / (call_us * 1e3)
    line = {"metric": METRIC, "value": call_us / (T * world), "unit": "us/token (FP8 LM head, 157184 x 2560)",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 x e4m3 (mma.sync), f32 accumulation",
            "data": "synthetic (seeded SplitMix64 weights, Irwin-Hall normals)",
            "config": {"workload": "FP8 output layer: 157,184 x 2,560 weights quantised per row, 1 token per call",
                       "l2": "weights 402 MB > L2"},
            "roofline": {"bound": "hbm", "kernel": "lmhead_gemv_kernel", "achieved": gbs, "peak": hbm_peak,
                         "unit": "GB/s", "peak_kind": peak_kind + " copy bandwidth (burst)", "frac": gbs / hbm_peak,
                         "traffic": NCU_LMHEAD_DRAM_BYTES, "alg_bytes_per_launch": alg, "avg_launch_us": call_us,
                         "frac_of_8tbs": gbs / 8000.0},
            "cpu_baseline": cpu,
            "e2e": {"value": 1e3 * e2e_ms / args.steps / (T * world), "unit": "us/token (FP8 LM head, 157184 x 2560)",
                    "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * V * 4},
            "gpu_launches": args.steps, "clocks": clk,
            "timing": "CUDA graph of K calls; e2e: eager calls with host copies"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g
    if world > 1:
        dist.destroy_process_group()


def peaks_bf16():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "prefill512":
        run_prefill(args)
    elif args.workload == "lmhead":
        run_lmhead(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
