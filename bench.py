#!/usr/bin/env python
"""Benchmark of the MXFP4 MoE decode layer on B200.

Default run: the metric's configuration (512-expert layers, top-8 + 1 shared,
hidden 2560, width 768, MXFP4 weights, FP8 activations; 64 distinct seeded
layers = 103 GB, so the 126 MB L2 never holds a repeated layer).  A step =
one token through all 64 layers, chained by the residual + RMSNorm harness,
in one persistent launch (routing, experts and combine of every layer); the
value is microseconds per token per layer.  The same JSON line carries, under
"configs", the other workloads measured in the same run:

  cfg0        1 token, E = 32 layers (16 distinct, rotated past L2)
  verify4_*   4-token verify calls through the 64 layers (i.i.d. and clustered tokens)
  stack42     1 token through 42 layers with the Zipf(1.1) router bias
  prefill512  512-token chunked-prefill calls (Zipf routing, tcgen05 grouped GEMMs)
  lmhead      the FP8 output layer, 157,184 x 2,560, 1 token

Each entry has its own value, roofline and, where the oracle can be sampled,
CPU baseline (the C++ float64 oracle on the host cores, 1 thread and all).

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                  [--workload all|layer|verify4|stack42|prefill512|lmhead]

Under torchrun (N > 1) every rank runs its own independent layer set
(replicas: the path has no data exchange) and rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import hashlib
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
V_LMHEAD = 157184


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="all",
                   choices=["all", "layer", "verify4", "stack42", "prefill512", "lmhead"])
    p.add_argument("--layers", type=int, default=64)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--prefill-kernel", default="auto", choices=["auto", "tcgen05", "exact"],
                   help="grouped-GEMM kernels of the prefill workload")
    return p.parse_args()


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu
# capture of each kernel, with the SHA-256 (first 16 hex digits) of the
# source file the kernel was built from at that capture.  A source that has
# changed since makes the figure stale: the line then reports traffic null.
NCU_TRAFFIC = {
    # decode_kernel, 2-layer stack at T = 1, per layer (traffic grows with the layers a launch runs)
    "decode_kernel": {"bytes": (61.842432e6 + 0.805632e6) / 2, "per": "layer",
                      "src": "mxfp4_expert_layers_b200/csrc/decode.cu", "sha16": "94d672980f03b8a0"},
    # tc_gemm_kernel<0> + tc_gemm_kernel<1> of one 512-token prefill call (Zipf routing)
    "tc_gemm_kernel": {"bytes": 228.321024e6 + 11.817728e6 + 116.868352e6 + 3.162112e6, "per": "call",
                       "src": "mxfp4_expert_layers_b200/csrc/prefill_tc.cu", "sha16": "7eabad916cda2413"},
    # lmhead_gemv_kernel, one 157,184 x 2,560 call at T = 1
    "lmhead_gemv_kernel": {"bytes": 403.072768e6 + 3.427328e6, "per": "call",
                           "src": "mxfp4_expert_layers_b200/csrc/lmhead.cu", "sha16": "d9474f27b205c7ec"},
}


def src_sha16(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel: str, scale: float = 1.0):
    """(traffic bytes or None, provenance note)."""
    t = NCU_TRAFFIC[kernel]
    cur = src_sha16(t["src"])
    if t["bytes"] is None:
        return None, f"no ncu capture of {kernel} at source {cur}"
    if t["sha16"] != cur:
        return None, f"stale: ncu capture of {kernel} at source {t['sha16']}, current {cur}"
    return t["bytes"] * scale, f"ncu capture of {kernel} at source {cur} (per {t['per']})"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def peaks_bf16():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


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
    """``n`` seeded layers of ``n_experts`` routed experts resident in HBM,
    one library handle each (``bias``: the Zipf(1.1) router bias)."""

    def __init__(self, n, bias=False, max_tokens=4, n_experts=E, seed=0):
        import torch
        import mxfp4_expert_layers_b200 as moe
        import synth.gpu
        lb = (n_experts + N_SHARED) * BYTES_PER_EXPERT + n_experts * H * 2
        free, _ = torch.cuda.mem_get_info()
        fit = int((free - (6 << 30)) // lb)
        self.requested = n
        self.n = max(1, min(n, fit))
        self.E = n_experts
        self.bufs, self.handles = [], []
        nexp = n_experts + N_SHARED
        # canonical weights are generated into one scratch set, then packed
        canon = {"w13_codes": torch.empty((nexp, 2 * I, H // 2), dtype=torch.uint8, device="cuda"),
                 "w13_scales": torch.empty((nexp, 2 * I, H // 32), dtype=torch.uint8, device="cuda"),
                 "w2_codes": torch.empty((nexp, H, I // 2), dtype=torch.uint8, device="cuda"),
                 "w2_scales": torch.empty((nexp, H, I // 32), dtype=torch.uint8, device="cuda")}
        for layer in range(self.n):
            t = {"router_w": torch.empty((n_experts, H), dtype=torch.int16, device="cuda"),
                 "w13": torch.empty((nexp, I // 8, moe.w13_tile_bytes(H)), dtype=torch.uint8, device="cuda"),
                 "w2": torch.empty((nexp, H // 16, moe.w2_tile_bytes(I)), dtype=torch.uint8, device="cuda")}
            canon["router_w"] = t["router_w"]
            synth.gpu.fill_layer(canon, seed, layer, n_experts, H, I, N_SHARED)
            moe.moe_pack_weights(H, I, n_experts, K_TOP, N_SHARED, canon, 0, nexp, t["w13"], t["w2"])
            if bias:
                import synth as S
                t["router_bias"] = torch.from_numpy(S.zipf_router_bias(seed, layer, n_experts)).cuda()
            self.bufs.append(t)
            self.handles.append(moe.moe_create(H, I, n_experts, K_TOP, N_SHARED, t, max_tokens))
        del canon
        torch.cuda.synchronize()

    def extra_handles(self, count, bias, max_tokens, seed=0):
        """More handles over the first ``count`` layers' weights (with the
        Zipf bias of each layer, or none, and their own workspace)."""
        import torch
        import mxfp4_expert_layers_b200 as moe
        import synth as S
        hs = []
        for layer in range(min(count, self.n)):
            t = dict(self.bufs[layer])
            t["router_bias"] = torch.from_numpy(S.zipf_router_bias(seed, layer, self.E)).cuda() if bias else None
            self.bufs.append({"router_bias": t["router_bias"]})
            hs.append(moe.moe_create(H, I, self.E, K_TOP, N_SHARED, t, max_tokens))
        self.handles_extra = getattr(self, "handles_extra", []) + hs
        return hs

    def close(self):
        import mxfp4_expert_layers_b200 as moe
        for h in self.handles + getattr(self, "handles_extra", []):
            moe.moe_destroy(h)
        self.handles = []
        self.handles_extra = []


def layer_alg_bytes(T: int, distinct_routed: int, n_experts: int = E):
    """Algorithmic bytes of one layer call: weights of the distinct experts
    touched (routed + shared), the router, x in and y out, and the float32 h
    written by gate/up and read back for the down step."""
    U = distinct_routed + N_SHARED
    w13 = U * 2 * I * (H // 2 + H // 32)
    w2 = U * H * (I // 2 + I // 32)
    router = n_experts * H * 2
    act = T * H * 2 * 2
    hbuf = U * T * I * 4 * 2
    return w13 + w2 + router + act + hbuf


# ----------------------------------------------------------- timing helpers --
def barrier(world):
    import torch
    import torch.distributed as dist
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()


def time_graph(step, steps, world):
    """Capture ``steps`` calls of step(i, stream) into one CUDA graph, replay
    it once untimed, then time one replay with CUDA events.  Returns ms."""
    import torch
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            for i in range(steps):
                step(i, cap)
    g.replay()
    barrier(world)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    g.replay()
    ev1.record(stream)
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    del g
    return ms


def eager_stats(step, steps, world):
    """Per-call CUDA-event times of ``steps`` eager calls: median, p10, p90 (us)."""
    import torch
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    for i in range(steps):
        evs[i][0].record(stream)
        step(i, stream)
        evs[i][1].record(stream)
    barrier(world)
    us = np.array([1e3 * a.elapsed_time(b) for a, b in evs])
    return {"median_us": float(np.median(us)), "p10_us": float(np.percentile(us, 10)),
            "p90_us": float(np.percentile(us, 90)), "calls": steps}


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


# ----------------------------------------------------------- oracle arm --
def oracle_sample(calls: int, T: int = 1, threads: int = 0, budget_s: float = 10.0, n_experts: int = E,
                  bias: bool = False, clustered: bool = False):
    """Time the C++ float64 oracle (oracle/moe_oracle.cpp) on the host cores:
    ``calls`` layer calls of T tokens (layers 0, 1, ...), weights regenerated
    outside the timed region; stops early once ``budget_s`` of oracle time
    is spent.  threads = 0: all processors."""
    import synth
    from oracle import cpp as OC
    cores = OC.set_threads(threads)
    times = []
    try:
        for i in range(calls):
            layer = i % 64
            x = (synth.hidden_states_clustered if clustered else synth.hidden_states)(0, 1000 + i, T, H)
            wr = synth.router_weight(0, layer, n_experts, H)
            b = synth.zipf_router_bias(0, layer, n_experts) if bias else None
            t0 = time.perf_counter()
            _, ids, w = OC.route(x, wr, b, K_TOP)
            t_route = time.perf_counter() - t0
            ex = {e: synth.expert_weights(0, layer, e, H, I)
                  for e in set(ids.ravel().tolist()) | {n_experts + s for s in range(N_SHARED)}}
            t0 = time.perf_counter()
            OC.forward(x, ids, w, ex, n_experts, I, N_SHARED)
            times.append(t_route + time.perf_counter() - t0)
            if sum(times) > budget_s:
                break
    finally:
        OC.set_threads(0)
    kind = "clustered " if clustered else ""
    return {"us_per_call": 1e6 * sum(times) / len(times), "cores": cores,
            "sample": f"{len(times)} call(s) of {T} {kind}token(s) through E={n_experts} layers "
                      f"(C++ float64 oracle, {cores} thread(s))"}


def oracle_lmhead_sample(rows: int = 8192, budget_s: float = 10.0):
    """Time the float64 FP8 LM-head oracle (numpy; no C++ form) on ``rows``
    of the vocabulary, scaled to the full 157,184 rows: µs per token."""
    import synth
    from oracle import lmhead as LH
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        cores = 1
    q, s = LH.lmhead_quantize(synth.lmhead_weight(0, V_LMHEAD, H, 0, rows))
    times = []
    for i in range(100):
        x = synth.hidden_states(0, 3000 + i, 1, H)
        t0 = time.perf_counter()
        LH.lmhead_logits(q, s, x)
        times.append(time.perf_counter() - t0)
        if sum(times) > budget_s:
            break
    return {"us_per_call": 1e6 * (sum(times) / len(times)) * V_LMHEAD / rows, "cores": cores,
            "sample": f"{len(times)} token(s) through {rows} of {V_LMHEAD} rows, scaled to the full vocabulary; "
                      "float64 numpy oracle (BLAS threads)"}


def cpu_pair(unit, scale=1.0, **kw):
    """The oracle on one thread and on all host threads, same sample."""
    one = oracle_sample(threads=1, budget_s=kw.pop("budget_1", 6.0), **kw)
    allc = oracle_sample(threads=0, budget_s=kw.pop("budget_all", 6.0), **kw)
    return {"value": allc["us_per_call"] * scale, "unit": unit, "cores": allc["cores"], "kind": "oracle",
            "sample": allc["sample"], "value_1thread": one["us_per_call"] * scale,
            "sample_1thread": one["sample"]}


def run_reference(args):
    """The oracle as it stands, on the host cores, for this run's workload:
    each step one bounded sample; the whole run a few minutes at most."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = "layer" if args.workload == "all" else args.workload
    t_start = time.perf_counter()
    budget = min(150.0, max(5.0, 1.5 * args.steps))
    if wl == "lmhead":
        res = oracle_lmhead_sample(budget_s=budget)
        value, unit = res["us_per_call"], "us/token (FP8 LM head, 157184 x 2560)"
    else:
        T = 4 if wl == "verify4" else 1
        for _ in range(min(args.warmup, 1)):
            oracle_sample(1, T, budget_s=1e9)
        res = oracle_sample(args.steps, T, budget_s=budget, bias=wl in ("stack42", "prefill512"))
        value, unit = res["us_per_call"] / T, "us/token"
        if wl == "stack42":
            value, unit = value * 42, "us/token (42-layer stack)"
        elif wl == "prefill512":
            unit = "us/token (512-token prefill call)"
    el = time.perf_counter() - t_start
    line = {"metric": METRIC, "value": value, "unit": unit, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / max(args.steps, 1), "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args.layers, None),
            "cpu_baseline": {"value": value, "unit": unit, "cores": res["cores"], "kind": "oracle",
                             "sample": res["sample"]},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(wl, n, layers):
    if wl == "layer":
        w = (f"1-token decode through {n} distinct E=512 top-8 + 1 shared layers (H=2560, I=768, MXFP4 W4A8), "
             "chained by the residual + RMSNorm harness, one persistent launch per token")
    elif wl == "verify4":
        w = f"4-token verify call (i.i.d. tokens) through {n} chained E=512 layers, one launch per call"
    elif wl == "prefill512":
        w = "chunked prefill: 512 tokens per call, E=512 top-8 + 1 shared, Zipf(1.1) bias"
    elif wl == "lmhead":
        w = "FP8 output layer: 157,184 x 2,560 weights quantised per row, 1 token per call"
    else:
        w = "42-layer decode stack, Zipf(1.1) router bias, residual + RMSNorm chain, one launch per token"
    c = {"workload": w, "layers_resident": n, "hidden": H, "inter": I, "experts": E, "top_k": K_TOP,
         "shared": N_SHARED,
         "l2": "inputs larger than L2: every layer distinct (" + f"{n * LAYER_BYTES / 1e9:.1f} GB resident)"}
    if layers is not None and layers.n < layers.requested:
        c["note"] = f"only {layers.n} of {layers.requested} layers fit in free HBM"
    return c


# --------------------------------------------------------------- our arm --
class Ctx:
    def __init__(self, args):
        import torch
        import torch.distributed as dist
        import mxfp4_expert_layers_b200 as moe
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        moe.load()
        self.hbm_peak, self.peak_kind = peaks()
        self.args = args
        self.cpu = self.rank == 0 and self.world == 1 and not args.no_cpu_baseline


def stack_run(ctx, layers_handles, T, steps, warmup, xs, name, headline=False, clustered=False):
    """One token (or T-token call) through a stack of layers per step.
    Returns the timings, the ids of the last eager step and the kernel's
    per-launch duration."""
    import torch
    import mxfp4_expert_layers_b200 as moe
    L = len(layers_handles)
    stack = moe.moe_stack_create(layers_handles)
    r = torch.empty((T, H), dtype=torch.int16, device="cuda")
    x = torch.empty((T, H), dtype=torch.int16, device="cuda")
    ids = torch.empty((L, T, K_TOP), dtype=torch.int32, device="cuda")
    wts = torch.empty((L, T, K_TOP), dtype=torch.float32, device="cuda")

    def step(i, s):
        x0 = xs[i % xs.shape[0]]
        r.copy_(x0)
        x.copy_(x0)
        moe.moe_stack_decode(stack, r, x, T, 1e-6, ids, wts, None, s)

    stream = torch.cuda.current_stream()
    for i in range(warmup):
        step(i, stream)
    barrier(ctx.world)
    assert moe.moe_stack_device_error(stack) == moe.MOE_OK, name
    out = {"layers": L}
    clk = None
    if headline:
        clocks = Clocks(ctx.local)
        clocks.start()
        time.sleep(0.3)
    out["ms_graph"] = time_graph(lambda i, s: step(warmup + i, s), steps, ctx.world)
    if headline:
        clk = clocks.stop()
    assert moe.moe_stack_device_error(stack) == moe.MOE_OK, name
    out["eager"] = eager_stats(lambda i, s: step(warmup + i, s), max(10, min(steps, 100)), ctx.world)
    # the stack kernel's own duration: events around every launch
    moe.moe_stack_profile_begin(stack, steps + 2)
    barrier(ctx.world)
    for i in range(steps):
        step(warmup + i, stream)
    barrier(ctx.world)
    dk_ms, dk_n = moe.moe_stack_profile_end(stack).get("decode", (0.0, 0))
    out["kernel_us"] = 1e3 * dk_ms / max(dk_n, 1)
    out["launches_timed"] = dk_n
    idn = ids.cpu().numpy()
    out["distinct_routed"] = [len(set(idn[l].ravel().tolist())) for l in range(L)]
    out["clocks"] = clk
    out["stack"], out["r"], out["x"] = stack, r, x
    return out


def roofline_hbm(ctx, kernel, alg_bytes, launch_us, traffic, note, extra=None):
    a = alg_bytes / (launch_us * 1e3)
    d = {"bound": "hbm", "kernel": kernel, "achieved": a, "peak": ctx.hbm_peak, "unit": "GB/s",
         "peak_kind": f"{ctx.peak_kind} copy bandwidth (burst)", "frac": a / ctx.hbm_peak,
         "frac_of_8tbs": a / 8000.0, "traffic": traffic, "traffic_note": note,
         "alg_bytes_per_launch": alg_bytes, "avg_launch_us": launch_us}
    if extra:
        d.update(extra)
    return d


def run_ours(args):
    import torch
    import torch.distributed as dist
    import mxfp4_expert_layers_b200 as moe
    import synth

    ctx = Ctx(args)
    world, rank = ctx.world, ctx.rank
    wl = args.workload
    T = 4 if wl == "verify4" else 1
    n_layers = 42 if wl == "stack42" else args.layers
    layers = Layers(n_layers, bias=(wl == "stack42"), max_tokens=4)
    L = layers.n
    nsteps = args.warmup + args.steps
    xs_host = np.stack([synth.hidden_states(0, 1000 + 7919 * rank + i, T, H) for i in range(min(nsteps, 512))])
    xs = torch.from_numpy(xs_host.view(np.int16)).cuda()

    # ---- headline: the metric's workload, K steps in a CUDA graph
    res = stack_run(ctx, layers.handles, T, args.steps, args.warmup, xs, wl, headline=True)
    ms = max_over_ranks(res["ms_graph"], "cuda")
    stack, r, x = res["stack"], res["r"], res["x"]
    dk_us = res["kernel_us"]
    distinct = res["distinct_routed"]
    alg_launch = sum(layer_alg_bytes(T, d) for d in distinct)
    layer_us = 1e3 * ms / (args.steps * L)
    if wl == "stack42":
        value = 1e3 * ms / args.steps / world
    else:
        value = per_token_value(ms, args.steps, L, T, world)
    traffic, tnote = ncu_traffic("decode_kernel", L)
    if T != 1:
        traffic, tnote = None, "ncu capture is of the T = 1 stack"
    roof = roofline_hbm(ctx, "decode_kernel", alg_launch, dk_us, traffic, tnote,
                        {"launches_timed": res["launches_timed"], "layers_per_launch": L})

    # ---- e2e through the public API with pinned host buffers
    xh = torch.from_numpy(xs_host.view(np.int16)).pin_memory()
    xo = torch.empty((T, H), dtype=torch.int16).pin_memory()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    ev0.record(stream)
    for i in range(args.warmup, nsteps):
        r.copy_(xh[i % xh.shape[0]], non_blocking=True)
        x.copy_(r)
        moe.moe_stack_decode(stack, r, x, T, 1e-6, None, None, None, stream)
        xo.copy_(x, non_blocking=True)
    ev1.record(stream)
    barrier(world)
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), "cuda")
    e2e_step_us = 1e3 * e2e_ms / args.steps
    e2e_val = (e2e_step_us if wl == "stack42" else e2e_step_us / (L * T)) / world
    moe.moe_stack_destroy(stack)

    unit = "us/token" if wl != "stack42" else "us/token (42-layer stack)"
    cpu = None
    if ctx.cpu:
        cpu = cpu_pair(unit, scale=(42.0 if wl == "stack42" else 1.0 / T), calls=20, T=T,
                       bias=wl == "stack42")
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "e2m1 x e4m3 operands, f32 block sums, f64 accumulation",
            "data": "synthetic (seeded SplitMix64 weights, Irwin-Hall normals)",
            "config": workload_config("layer" if wl == "all" else wl, L, layers),
            "layer_us": layer_us, "layer_gbs": alg_launch / L / (layer_us * 1e3),
            "alg_bytes_per_layer": alg_launch / L, "eager_per_step": res["eager"],
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": T * H * 2,
                    "d2h_bytes_per_step": T * H * 2},
            "gpu_launches": args.steps, "clocks": res["clocks"],
            "timing": "CUDA graph of K steps (one stack launch each); eager_per_step: CUDA events around "
                      "each of up to 100 eager steps"}
    if wl == "verify4":
        line["distinct_experts_mean"] = float(np.mean(distinct))
    if wl == "stack42":
        line["stack_tokens_per_s"] = 1e6 / value

    if wl == "all":
        line["configs"] = measure_configs(ctx, layers)
        line["gpu_launches"] = args.steps + sum(c.get("gpu_launches", 0) for c in line["configs"].values())
    if rank == 0:
        print(json.dumps(line), flush=True)
    layers.close()
    if world > 1:
        dist.destroy_process_group()


def measure_configs(ctx, layers):
    """The other workloads of the run, each with its own value and roofline
    (and CPU baseline where the oracle can be sampled)."""
    import torch
    import synth
    cfg = {}
    steps = 20
    # ---- verify: 4 tokens per call through the 64 layers
    for kind in ("iid", "clustered"):
        gen = synth.hidden_states if kind == "iid" else synth.hidden_states_clustered
        xs = torch.from_numpy(np.stack([gen(0, 2000 + i, 4, H) for i in range(32)]).view(np.int16)).cuda()
        res = stack_run(ctx, layers.handles, 4, steps, 3, xs, "verify4")
        import mxfp4_expert_layers_b200 as moe
        moe.moe_stack_destroy(res["stack"])
        L = res["layers"]
        call_us = 1e3 * max_over_ranks(res["ms_graph"], "cuda") / (steps * L)
        alg = sum(layer_alg_bytes(4, d) for d in res["distinct_routed"])
        cfg[f"verify4_{kind}"] = {
            "value": call_us, "unit": "us/call per layer (4 tokens)", "us_per_token": call_us / 4,
            "distinct_experts_mean": float(np.mean(res["distinct_routed"])),
            "eager_per_call": {k: v / L if k.endswith("_us") else v for k, v in res["eager"].items()},
            "roofline": roofline_hbm(ctx, "decode_kernel", alg, res["kernel_us"], None, "ncu capture is of T = 1"),
            "gpu_launches": steps}
        if ctx.cpu:
            cfg[f"verify4_{kind}"]["cpu_baseline"] = cpu_pair("us/call per layer (4 tokens)", calls=6, T=4,
                                                              clustered=kind == "clustered")
    # ---- the 42-layer stack with the Zipf router bias (handles over layers 0..41)
    hs = layers.extra_handles(42, bias=True, max_tokens=4)
    xs = torch.from_numpy(np.stack([synth.hidden_states(0, 5000 + i, 1, H) for i in range(32)]).view(np.int16)).cuda()
    res = stack_run(ctx, hs, 1, steps, 3, xs, "stack42")
    import mxfp4_expert_layers_b200 as moe
    moe.moe_stack_destroy(res["stack"])
    tok_us = 1e3 * max_over_ranks(res["ms_graph"], "cuda") / steps
    alg = sum(layer_alg_bytes(1, d) for d in res["distinct_routed"])
    cfg["stack42"] = {"value": tok_us, "unit": "us/token (42-layer stack)", "tokens_per_s": 1e6 / tok_us,
                      "layers": res["layers"], "stack_gbs": alg / (tok_us * 1e3),
                      "eager_per_token": res["eager"],
                      "roofline": roofline_hbm(ctx, "decode_kernel", alg, res["kernel_us"], None,
                                               "ncu capture is of the unbiased 2-layer stack"),
                      "gpu_launches": steps}
    if ctx.cpu:
        cfg["stack42"]["cpu_baseline"] = cpu_pair("us/token (42-layer stack)", scale=42.0, calls=6, bias=True)
    # ---- config 0: E = 32, 16 distinct layers (1.6 GB) rotated past L2
    small = Layers(16, bias=False, max_tokens=4, n_experts=32, seed=0)
    xs = torch.from_numpy(np.stack([synth.hidden_states(0, i, 1, H) for i in range(32)]).view(np.int16)).cuda()
    res = stack_run(ctx, small.handles, 1, 50, 3, xs, "cfg0")
    moe.moe_stack_destroy(res["stack"])
    L = res["layers"]
    lu = 1e3 * max_over_ranks(res["ms_graph"], "cuda") / (50 * L)
    alg = sum(layer_alg_bytes(1, d, 32) for d in res["distinct_routed"])
    cfg["cfg0"] = {"value": lu, "unit": "us/token", "layers_rotated": L,
                   "l2": f"16 distinct E=32 layers ({16 * (33 * BYTES_PER_EXPERT + 32 * H * 2) / 1e9:.2f} GB) "
                         "rotated, larger than L2",
                   "eager_per_step": {k: v / L if k.endswith("_us") else v for k, v in res["eager"].items()},
                   "roofline": roofline_hbm(ctx, "decode_kernel", alg, res["kernel_us"], None, "no ncu capture of E = 32"),
                   "gpu_launches": 50}
    if ctx.cpu:
        cfg["cfg0"]["cpu_baseline"] = cpu_pair("us/token", calls=10, n_experts=32)
    small.close()
    cfg["prefill512"] = measure_prefill(ctx, layers)
    cfg["lmhead"] = measure_lmhead(ctx)
    return cfg


def measure_prefill(ctx, layers, steps=10, standalone=False):
    """Chunked prefill: 512 tokens per call through E = 512 layers with the
    Zipf(1.1) bias (routing + dispatch + grouped GEMMs + combine)."""
    import torch
    import mxfp4_expert_layers_b200 as moe
    import synth
    T = 512
    hs = layers.extra_handles(4, bias=True, max_tokens=T)
    kind = {"auto": moe.MOE_PREFILL_AUTO, "tcgen05": moe.MOE_PREFILL_TCGEN05,
            "exact": moe.MOE_PREFILL_EXACT}[ctx.args.prefill_kernel]
    for h in hs:
        moe.moe_set_prefill_kernel(h, kind)
    xs = torch.from_numpy(np.stack([synth.hidden_states(0, 20000 + 7919 * ctx.rank + i, T, H)
                                    for i in range(4)]).view(np.int16)).cuda()
    ids = torch.empty((T, K_TOP), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, K_TOP), dtype=torch.float32, device="cuda")
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    nh = len(hs)

    def step(i, s):
        moe.moe_decode(hs[i % nh], xs[i % xs.shape[0]], T, ids, wts, y, counts, None, s)

    for i in range(3):
        step(i, torch.cuda.current_stream())
    barrier(ctx.world)
    assert all(moe.moe_device_error(h) == moe.MOE_OK for h in hs)
    touched = int((counts.cpu().numpy() > 0).sum()) + N_SHARED
    tc = moe.moe_last_path(hs[0]) == 3
    ms = max_over_ranks(time_graph(lambda i, s: step(3 + i, s), steps, ctx.world), "cuda")
    eager = eager_stats(lambda i, s: step(3 + i, s), steps, ctx.world)
    for h in hs:
        moe.moe_profile_begin(h, steps + 2)
    barrier(ctx.world)
    for i in range(steps):
        step(3 + i, torch.cuda.current_stream())
    barrier(ctx.world)
    gm_ms, gm_n = 0.0, 0
    for h in hs:
        t_ms, n = moe.moe_profile_end(h).get("grouped_gemm", (0.0, 0))
        gm_ms, gm_n = gm_ms + t_ms, gm_n + n
    gemm_us = 1e3 * gm_ms / max(gm_n, 1)
    call_us = 1e3 * ms / steps
    flops = 2.0 * 3 * H * I * T * (K_TOP + N_SHARED)
    P = T * (K_TOP + N_SHARED)
    # the grouped GEMMs (+ requant between them): weights of the touched experts,
    # the FP8 operand panels of x and h, h written and read back (float32), and
    # the float32 combine accumulator read-modify-written once per pair
    gemm_bytes = touched * BYTES_PER_EXPERT + P * (H + I) + 2 * P * I * 4 + 2 * T * H * 4
    call_bytes = touched * BYTES_PER_EXPERT + E * H * 2 + T * H * (2 + 1 + 2)
    bf16_peak, bf16_kind = peaks_bf16()
    fp8_peak = bf16_peak * 2.0
    traffic, tnote = ncu_traffic("tc_gemm_kernel") if tc else (None, "mma.sync kernels: no ncu capture")
    roof = roofline_hbm(ctx, ("tc_gemm_kernel<0>+requant_kernel+tc_gemm_kernel<1>" if tc else
                              "gateup_kernel+requant_kernel+down_kernel"), gemm_bytes, gemm_us, traffic, tnote,
                        {"tensor_tflops": flops / (gemm_us * 1e6), "tensor_peak_tflops": fp8_peak,
                         "tensor_peak_kind": f"{bf16_kind} bf16 cuBLAS burst x 2 (nominal fp8/bf16 ratio)",
                         "tensor_frac": flops / (gemm_us * 1e6) / fp8_peak,
                         "hbm_gbs_of_call": call_bytes / (call_us * 1e3)})
    out = {"value": call_us, "unit": "us/call (512 tokens)", "us_per_token": call_us / T,
           "experts_touched": touched, "flops_per_call": flops, "bytes_per_call": call_bytes,
           "tflops_of_call": flops / (call_us * 1e6), "eager_per_call": eager, "roofline": roof,
           "dtype": ("e2m1 x e4m3 operands (tcgen05 block-scaled MMA), f32 accumulation" if tc else
                     "e2m1 x e4m3 operands, f32 block sums, f64 accumulation"),
           "gpu_launches": steps * 9}
    if ctx.cpu:
        # the oracle on a few tokens of the call, scaled to 512 (each token's
        # output depends on its own routing only)
        one = oracle_sample(8, 1, threads=0, budget_s=6.0, bias=True)
        out["cpu_baseline"] = {"value": one["us_per_call"] * T, "unit": "us/call (512 tokens)",
                               "cores": one["cores"], "kind": "oracle",
                               "sample": one["sample"] + "; scaled to 512 tokens"}
    return out


def measure_lmhead(ctx, steps=50):
    """FP8 output layer, 157,184 x 2,560, one token per call."""
    import torch
    import mxfp4_expert_layers_b200 as moe
    import synth
    import synth.gpu
    V, T = V_LMHEAD, 1
    w = torch.empty((V, H), dtype=torch.int16, device="cuda")
    synth.gpu.fill_lmhead(w, 0, V, H)
    q = torch.empty((V, H), dtype=torch.uint8, device="cuda")
    sw = torch.empty((V,), dtype=torch.float32, device="cuda")
    moe.moe_lmhead_quantize(w, V, H, q, sw)
    del w
    xs = torch.from_numpy(np.stack([synth.hidden_states(0, 3000 + i, T, H) for i in range(64)]).view(np.int16)).cuda()
    out = torch.empty((T, V), dtype=torch.float32, device="cuda")

    def step(i, s):
        moe.moe_lmhead_logits(q, sw, V, H, xs[i % xs.shape[0]], T, out, s)

    for i in range(3):
        step(i, torch.cuda.current_stream())
    barrier(ctx.world)
    ms = max_over_ranks(time_graph(lambda i, s: step(3 + i, s), steps, ctx.world), "cuda")
    eager = eager_stats(lambda i, s: step(3 + i, s), steps, ctx.world)
    call_us = 1e3 * ms / steps
    alg = V * H + V * 4 + T * H * 2 + T * V * 4
    traffic, tnote = ncu_traffic("lmhead_gemv_kernel")
    res = {"value": call_us, "unit": "us/token (FP8 LM head, 157184 x 2560)", "eager_per_call": eager,
           "roofline": roofline_hbm(ctx, "lmhead_gemv_kernel", alg, call_us, traffic, tnote),
           "gpu_launches": steps}
    if ctx.cpu:
        c = oracle_lmhead_sample(budget_s=6.0)
        res["cpu_baseline"] = {"value": c["us_per_call"], "unit": res["unit"], "cores": c["cores"],
                               "kind": "oracle", "sample": c["sample"]}
    return res


def run_single(args, which):
    """--workload prefill512 | lmhead on their own: the workload's own line."""
    import torch.distributed as dist
    ctx = Ctx(args)
    if which == "prefill512":
        layers = Layers(min(args.layers, 4), bias=False, max_tokens=4)
        res = measure_prefill(ctx, layers, steps=args.steps)
        layers.close()
    else:
        res = measure_lmhead(ctx, steps=args.steps)
    line = {"metric": METRIC, "value": res["value"] / ctx.world, "unit": res["unit"], "n_gpus": ctx.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["value"] / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": res.get("dtype", "e4m3 x e4m3 (mma.sync), f32 accumulation"),
            "data": "synthetic (seeded SplitMix64 weights, Irwin-Hall normals)",
            "config": workload_config(which, 4, None), "roofline": res["roofline"],
            "cpu_baseline": res.get("cpu_baseline"), "gpu_launches": res["gpu_launches"],
            "e2e": None, "detail": res}
    if ctx.rank == 0:
        print(json.dumps(line), flush=True)
    if ctx.world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload in ("prefill512", "lmhead"):
        run_single(args, args.workload)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
