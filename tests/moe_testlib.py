"""Helpers of the GPU parity tests: build a layer on the device (seeded
generator), call the library through its C ABI, and build the matching host
view for the oracle."""
from __future__ import annotations

import numpy as np
import torch

import mxfp4_expert_layers_b200 as moe
import synth
import synth.gpu
from oracle import cpp as OC
from oracle import formats as OF
from oracle import moe as OM

H0, I0 = 2560, 768
REL_L2 = 2e-3          # output tolerance of the layer (relative L2)
MAX_ABS = 1e-2         # max |delta| <= MAX_ABS * max |ref|


class LazyExperts(dict):
    """Expert arrays regenerated on the host on first use."""

    def __init__(self, seed, layer, H, I):
        super().__init__()
        self.args = (seed, layer, H, I)

    def __missing__(self, e):
        seed, layer, H, I = self.args
        v = synth.expert_weights(seed, layer, int(e), H, I)
        self[e] = v
        return v


def oracle_layer(host: OM.LayerWeights, x_bits, E, k, I, n_shared=1):
    """The C++ float64 oracle (bit-equal to oracle.moe.moe_layer, and faster
    for full-size layers): routes, regenerates the touched experts, runs the
    experts and the combine."""
    logits, ids, w = OC.route(x_bits, host.router_w, host.router_bias, k)
    return oracle_forward(host, x_bits, ids, w, E, I, n_shared, extra={"logits": logits})


def oracle_forward(host: OM.LayerWeights, x_bits, ids, w, E, I, n_shared=1, extra=None):
    """The C++ oracle's experts and combine for given routing (as
    oracle.moe.moe_forward)."""
    need = set(np.asarray(ids).ravel().tolist()) | {E + s for s in range(n_shared)}
    experts = {e: host.experts[e] for e in need}
    out = OC.forward(x_bits, ids, w, experts, E, I, n_shared)
    out.update(ids=np.asarray(ids, np.int32), w=np.asarray(w, np.float32),
               counts=np.bincount(np.asarray(ids).ravel(), minlength=E).astype(np.int32))
    if extra:
        out.update(extra)
    return out


def to_dev_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


class GpuLayer:
    def __init__(self, seed, layer, E, H=H0, I=I0, k=8, n_shared=1, bias=False, max_tokens=4,
                 fill="gpu", weights=None, prefill=None):
        self.seed, self.layer, self.E, self.H, self.I, self.k, self.S = seed, layer, E, H, I, k, n_shared
        n = E + n_shared
        dev = "cuda"
        self.canon = {}
        if weights is None:
            self.t = {
                "router_w": torch.empty((E, H), dtype=torch.int16, device=dev),
                "w13_codes": torch.empty((n, 2 * I, H // 2), dtype=torch.uint8, device=dev),
                "w13_scales": torch.empty((n, 2 * I, H // 32), dtype=torch.uint8, device=dev),
                "w2_codes": torch.empty((n, H, I // 2), dtype=torch.uint8, device=dev),
                "w2_scales": torch.empty((n, H, I // 32), dtype=torch.uint8, device=dev),
            }
            if fill == "gpu":
                synth.gpu.fill_layer(self.t, seed, layer, E, H, I, n_shared)
            else:
                lw = synth.layer_weights(seed, layer, E, H, I, n_shared)
                self.t["router_w"].copy_(to_dev_u16(lw["router_w"]))
                for key in ("w13_codes", "w13_scales", "w2_codes", "w2_scales"):
                    self.t[key].copy_(to_dev(lw[key]))
            self.host = OM.LayerWeights(router_w=synth.router_weight(seed, layer, E, H), router_bias=None,
                                        experts=LazyExperts(seed, layer, H, I))
        else:  # explicit host arrays (edge-case tests)
            self.t = {"router_w": to_dev_u16(weights["router_w"])}
            for key in ("w13_codes", "w13_scales", "w2_codes", "w2_scales"):
                self.t[key] = to_dev(weights[key])
            ex = {e: {key: weights[key][e] for key in ("w13_codes", "w13_scales", "w2_codes", "w2_scales")}
                  for e in range(n)}
            self.host = OM.LayerWeights(router_w=weights["router_w"], router_bias=None, experts=ex)
        if bias is not False:
            b = synth.zipf_router_bias(seed, layer, E) if bias is True else np.asarray(bias, np.float32)
            self.t["router_bias"] = to_dev(b)
            self.host.router_bias = b
        # packed layout the kernels read
        self.t["w13"] = torch.empty((n, I // 8, moe.w13_tile_bytes(H)), dtype=torch.uint8, device=dev)
        self.t["w2"] = torch.empty((n, H // 16, moe.w2_tile_bytes(I)), dtype=torch.uint8, device=dev)
        moe.moe_pack_weights(H, I, E, k, n_shared, self.t, 0, n, self.t["w13"], self.t["w2"])
        torch.cuda.synchronize()
        for key in ("w13_codes", "w13_scales", "w2_codes", "w2_scales"):
            self.canon = getattr(self, "canon", {})
            self.canon[key] = self.t.pop(key)
        self.handle = moe.moe_create(H, I, E, k, n_shared, self.t, max_tokens)
        if prefill is not None:
            moe.moe_set_prefill_kernel(self.handle, prefill)

    def close(self):
        if self.handle:
            moe.moe_destroy(self.handle)
            self.handle = None

    def route(self, x_dev, T):
        ids = torch.empty((T, self.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, self.k), dtype=torch.float32, device="cuda")
        counts = torch.empty((self.E,), dtype=torch.int32, device="cuda")
        moe.moe_route(self.handle, x_dev, T, ids, w, counts, torch.cuda.current_stream())
        return ids, w, counts

    def _debug_buffers(self, T):
        S = self.k + self.S
        return {"xq": torch.empty((T, self.H), dtype=torch.uint8, device="cuda"),
                "xs": torch.empty((T,), dtype=torch.float32, device="cuda"),
                "h": torch.empty((T, S, self.I), dtype=torch.float32, device="cuda"),
                "qh": torch.empty((T, S, self.I), dtype=torch.uint8, device="cuda"),
                "sh": torch.empty((T, S), dtype=torch.float32, device="cuda")}

    def forward(self, x_dev, T, ids, w, debug=True):
        y = torch.empty((T, self.H), dtype=torch.int16, device="cuda")
        dbg = self._debug_buffers(T) if debug else None
        moe.moe_forward(self.handle, x_dev, T, ids, w, y, dbg, torch.cuda.current_stream())
        return y, dbg

    def decode(self, x_dev, T, debug=True):
        """moe_decode: routing and experts in one launch."""
        ids = torch.empty((T, self.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, self.k), dtype=torch.float32, device="cuda")
        counts = torch.empty((self.E,), dtype=torch.int32, device="cuda")
        y = torch.empty((T, self.H), dtype=torch.int16, device="cuda")
        dbg = self._debug_buffers(T) if debug else None
        moe.moe_decode(self.handle, x_dev, T, ids, w, y, counts, dbg, torch.cuda.current_stream())
        return ids, w, counts, y, dbg


def check_route(g_ids, g_w, g_counts, ref):
    ids = g_ids.cpu().numpy()
    assert np.array_equal(ids, ref["ids"]), (ids, ref["ids"])
    if g_counts is not None:
        assert np.array_equal(g_counts.cpu().numpy(), ref["counts"])
    w = g_w.cpu().numpy()
    assert np.allclose(w, ref["w"], rtol=1e-6, atol=1e-7)


def legit_fp8_flip(v_ref: float, code_a: int, code_b: int) -> bool:
    """Two adjacent codes are both acceptable when the exact value sits within
    1e-6 (relative) of the midpoint between them."""
    va, vb = float(OF.e4m3_value(code_a)), float(OF.e4m3_value(code_b))
    return abs(abs(va) - abs(vb)) > 0 and abs(v_ref - (va + vb) / 2) <= 1e-6 * max(abs(v_ref), 1e-30)


def check_forward(y_dev, dbg, ref, exact_frac=0.999):
    """Tolerance of the layer, plus the stronger bit-level checks that the
    exact arithmetic of the many-token mma.sync kernels (block sums scaled and
    summed in float64) allows."""
    yg = OF.bf16_to_f64(u16(y_dev))
    yr = OF.bf16_to_f64(ref["y"])
    rel = np.linalg.norm(yg - yr) / max(np.linalg.norm(yr), 1e-300)
    mx = np.abs(yg - yr).max() / max(np.abs(yr).max(), 1e-300)
    assert rel <= REL_L2 and mx <= MAX_ABS, (rel, mx)
    stats = {"rel_l2": rel, "max_rel": mx, "y_exact": float(np.mean(u16(y_dev) == ref["y"]))}
    if dbg is not None:
        assert np.array_equal(dbg["xq"].cpu().numpy(), ref["xq"])
        assert np.array_equal(dbg["xs"].cpu().numpy(), ref["xs"])
        qg = dbg["qh"].cpu().numpy()
        bad = np.argwhere(qg != ref["qh"])
        for t, s, j in bad:
            v = float(ref["h"][t, s, j]) / float(ref["sh"][t, s])
            assert legit_fp8_flip(v, int(qg[t, s, j]), int(ref["qh"][t, s, j])), (t, s, j)
        stats["qh_flips"] = len(bad)
        stats["h_exact"] = float(np.mean(dbg["h"].cpu().numpy() == ref["h"]))
        if len(bad) == 0:
            assert np.array_equal(dbg["sh"].cpu().numpy(), ref["sh"])
    assert stats["y_exact"] >= exact_frac, stats
    return stats


# Tolerance on h of the kernels that accumulate in float32: the decode kernel
# and the tcgen05 grouped GEMMs.  Each of the K/32 block products (exact) is
# scaled and added with
# one rounding of at most 2^-24 of the running sum, so the gate and up sums
# carry a relative error of order (K/32) * 2^-24 of the sum of their block
# magnitudes -- about 5e-6 at K = 2560 for sums without cancellation, more
# where the sum cancels.  SwiGLU keeps the order (its derivative is bounded
# by about 1.1 in g).  The check bounds the error by 1e-4 of the pair's amax,
# which leaves room for cancellation and float32 SwiGLU rounding.
H_TOL_TC = 1e-4


def check_forward_tc(y_dev, dbg, ref, exact_frac=0.9):
    """Layer tolerance on y, plus the checks that float32 accumulation of
    the block products allows: exact FP8 codes of x, h within H_TOL_TC of
    each pair's amax, s_h close, and every differing FP8 code of h one step
    from the oracle's with the value near their rounding boundary."""
    yg = OF.bf16_to_f64(u16(y_dev))
    yr = OF.bf16_to_f64(ref["y"])
    rel = np.linalg.norm(yg - yr) / max(np.linalg.norm(yr), 1e-300)
    mx = np.abs(yg - yr).max() / max(np.abs(yr).max(), 1e-300)
    assert rel <= REL_L2 and mx <= MAX_ABS, (rel, mx)
    stats = {"rel_l2": rel, "max_rel": mx, "y_exact": float(np.mean(u16(y_dev) == ref["y"]))}
    if dbg is not None:
        assert np.array_equal(dbg["xq"].cpu().numpy(), ref["xq"])
        assert np.array_equal(dbg["xs"].cpu().numpy(), ref["xs"])
        hg = dbg["h"].cpu().numpy().astype(np.float64)
        hr = ref["h"].astype(np.float64)
        amax = np.abs(hr).max(axis=2, keepdims=True)
        herr = np.abs(hg - hr) / np.maximum(amax, 1e-300)
        stats["h_err"] = float(herr.max())
        assert stats["h_err"] <= H_TOL_TC, stats
        shg = dbg["sh"].cpu().numpy().astype(np.float64)
        assert np.allclose(shg, ref["sh"], rtol=H_TOL_TC, atol=0), stats
        qg = dbg["qh"].cpu().numpy()
        bad = np.argwhere(qg != ref["qh"])
        for t, s_, j in bad:
            va, vb = float(OF.e4m3_value(int(qg[t, s_, j]))), float(OF.e4m3_value(int(ref["qh"][t, s_, j])))
            v = hr[t, s_, j] / float(ref["sh"][t, s_])
            # adjacent codes, the value within the h tolerance (in code units) of their midpoint
            assert abs(abs(va) - abs(vb)) <= 2.0 ** -3 * max(abs(va), abs(vb)) + 2.0 ** -9, (t, s_, j, va, vb)
            assert abs(v - (va + vb) / 2) <= 2 * H_TOL_TC * 448 + 1e-6 * abs(v), (t, s_, j, v, va, vb)
        stats["qh_flips"] = len(bad)
        stats["qh_flip_frac"] = len(bad) / max(qg.size, 1)
        stats["h_exact"] = float(np.mean(hg == hr))
    assert stats["y_exact"] >= exact_frac, stats
    return stats
