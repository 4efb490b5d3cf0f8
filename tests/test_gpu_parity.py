"""GPU parity: the CUDA path through the C ABI against the float64 oracle on
the same seeded inputs.  Bars: expert ids and counts bit-exact, FP8
activation bytes bit-exact, BF16 outputs within relative L2 <= 2e-3 and
max |delta| <= 1e-2 * max |ref|.  The decode kernel sums the 32-element
block products in float32 (tensor core) and the scaled blocks in float32
(fused multiply-adds), so h is held to the float32-accumulation bound of
check_forward_tc: within H_TOL_TC of each pair's amax, FP8 codes of h equal
up to one-step flips at rounding boundaries, and most outputs bit-exact."""
import numpy as np
import pytest
import torch

import mxfp4_expert_layers_b200 as moe
import synth
from oracle import formats as OF
from oracle import moe as OM

from moe_testlib import (GpuLayer, check_forward_tc, check_route, to_dev, to_dev_u16, u16,
                         H0, I0, REL_L2, MAX_ABS)

check_forward = check_forward_tc  # the decode kernel accumulates in float32

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU collection
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def _oracle(layer: GpuLayer, x_bits):
    return OM.moe_layer(x_bits, layer.host, layer.E, layer.k, layer.I, layer.S)


def _run(layer: GpuLayer, x_bits, debug=True, mode="split"):
    """mode "split": moe_route then moe_forward; "fused": moe_decode."""
    T = x_bits.shape[0]
    xd = to_dev_u16(x_bits)
    if mode == "split":
        ids, w, counts = layer.route(xd, T)
        y, dbg = layer.forward(xd, T, ids, w, debug)
    else:
        ids, w, counts, y, dbg = layer.decode(xd, T, debug)
    torch.cuda.synchronize()
    assert moe.moe_device_error(layer.handle) == moe.MOE_OK
    return ids, w, counts, y, dbg


MODES = ["split", "fused"]


# ------------------------------------------------------------ generators --

def test_gpu_fill_matches_host_generator():
    E, H, I = 16, 256, 128
    L = GpuLayer(5, 3, E, H, I, k=4, fill="gpu")
    try:
        assert np.array_equal(u16(L.t["router_w"]), synth.router_weight(5, 3, E, H))
        for e in (0, 7, E):                          # includes the shared expert
            ref = synth.expert_weights(5, 3, e, H, I)
            for key in ref:
                assert np.array_equal(L.canon[key][e].cpu().numpy(), ref[key]), (e, key)
    finally:
        L.close()


def _pack_tiles_numpy(codes, scales, row_a, row_b):
    """Packed tile bytes written out from the layout's definition: per block
    b, lane L = 4g+t: bytes 16b+4t.. of rows row_a(g) and row_b(g); then per
    block the scale pairs (row_a(g), row_b(g))."""
    nb = scales.shape[1]
    out = []
    for b in range(nb):
        for L in range(32):
            g, t = L // 4, L % 4
            out.append(codes[row_a(g), 16 * b + 4 * t:16 * b + 4 * t + 4])
            out.append(codes[row_b(g), 16 * b + 4 * t:16 * b + 4 * t + 4])
    for b in range(nb):
        for g in range(8):
            out.append(np.array([scales[row_a(g), b], scales[row_b(g), b]], np.uint8))
    return np.concatenate(out)


def test_gpu_pack_layout_matches_definition():
    E, H, I = 8, 256, 128
    L = GpuLayer(6, 1, E, H, I, k=2, fill="gpu")
    try:
        w13 = L.t["w13"].cpu().numpy()
        w2 = L.t["w2"].cpu().numpy()
        for e in (0, 5, E):
            ex = synth.expert_weights(6, 1, e, H, I)
            for c in (0, 3, I // 8 - 1):
                want = _pack_tiles_numpy(ex["w13_codes"], ex["w13_scales"],
                                         lambda g: 8 * c + g, lambda g: I + 8 * c + g)
                assert np.array_equal(w13[e, c], want), (e, c)
            for pt in (0, 7, H // 16 - 1):
                want = _pack_tiles_numpy(ex["w2_codes"], ex["w2_scales"],
                                         lambda g: 16 * pt + g, lambda g: 16 * pt + 8 + g)
                assert np.array_equal(w2[e, pt], want), (e, pt)
        # a permutation: every byte accounted for
        assert w13.size == L.canon["w13_codes"].numel() + L.canon["w13_scales"].numel()
    finally:
        L.close()


# ----------------------------------------------------------------- FP8 ---

def _structured_fp32():
    hi = np.arange(1 << 16, dtype=np.uint32) << np.uint32(16)
    lows = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x1234, 0xC000], dtype=np.uint32)
    pats = (hi[:, None] | lows[None, :]).ravel()
    v = pats.view(np.float32)
    return v[np.isfinite(v) & (np.abs(v) <= 448.0)]


def test_gpu_fp8_encoder_matches_oracle():
    """Rows [v, 448]: the scale is exactly 1, so the codes are the plain
    encoder on every structured float32 pattern of magnitude <= 448 (every
    sign/exponent/top-7-mantissa combination with boundary low bits), plus
    every exact midpoint between adjacent E4M3 values and its neighbours."""
    v = _structured_fp32()
    vals = np.unique(np.abs(OF.e4m3_value(np.arange(0x7F))))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                            np.nextafter(mids, np.float32(np.inf)), vals.astype(np.float32)])
    v = np.concatenate([v, extra, -extra]).astype(np.float32)
    rows = np.stack([v, np.full_like(v, 448.0)], axis=1)
    q = torch.empty(rows.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows.shape[0], dtype=torch.float32, device="cuda")
    moe.moe_quantize_fp8(to_dev(rows), rows.shape[0], 2, q, s)
    torch.cuda.synchronize()
    assert np.all(s.cpu().numpy() == 1.0)
    got = q.cpu().numpy()[:, 0]
    ref = OF.e4m3_encode(v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(got[i]), int(ref[i])) for i in bad[:8]]


def test_gpu_quantize_rows_matches_oracle():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal((37, 1000)) * rng.uniform(1e-3, 1e3, (37, 1))).astype(np.float32)
    v[3] = 0.0
    v[5, :] = -0.0
    q = torch.empty(v.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(v.shape[0], dtype=torch.float32, device="cuda")
    moe.moe_quantize_fp8(to_dev(v), v.shape[0], v.shape[1], q, s)
    rq, rs = OM.quantize_fp8(v)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), rs)


def test_gpu_quantize_near_code_boundaries_matches_oracle():
    """The quotient v / s taken through its reciprocal: rows whose values sit
    on, and within 12 float32 ulps of, every exact midpoint between adjacent
    E4M3 values (and every E4M3 value) times a scale that is not a power of
    two, both signs; the codes equal those of the correctly rounded float32
    quotient."""
    rng = np.random.default_rng(7)
    vals = np.unique(np.abs(OF.e4m3_value(np.arange(0x7F))))
    pts = np.concatenate([(vals[1:] + vals[:-1]) / 2, vals])
    rows = []
    for amax in rng.uniform(1e-3, 1e3, 24).astype(np.float32):
        s = np.float32(amax / np.float32(448.0))
        base = (pts * np.float64(s)).astype(np.float32)
        near = (base.view(np.int32)[:, None] + np.arange(-12, 13, dtype=np.int32)[None, :]).ravel()
        v = near.view(np.float32)
        v = v[np.abs(v) < amax]
        rows.append(np.concatenate([[amax], v, -v]).astype(np.float32))
    cols = max(r.size for r in rows)
    v = np.zeros((len(rows), cols), np.float32)
    for i, r in enumerate(rows):
        v[i, :r.size] = r
    q = torch.empty(v.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(v.shape[0], dtype=torch.float32, device="cuda")
    moe.moe_quantize_fp8(to_dev(v), v.shape[0], v.shape[1], q, s)
    rq, rs = OM.quantize_fp8(v)
    assert np.array_equal(s.cpu().numpy(), rs)
    got = q.cpu().numpy()
    bad = np.argwhere(got != rq)
    assert bad.size == 0, [(float(v[i, j]), int(got[i, j]), int(rq[i, j])) for i, j in bad[:8]]


# --------------------------------------------------------------- routing --

@pytest.mark.parametrize("E,T,bias", [(32, 1, False), (512, 1, False), (512, 4, False),
                                      (512, 4, True), (512, 37, True)])
def test_gpu_route_matches_oracle(E, T, bias):
    L = GpuLayer(0, 0, E, k=8, bias=bias, max_tokens=max(T, 4))
    try:
        x = synth.hidden_states(0, 1000 + T, T, H0)
        ids, w, counts = L.route(to_dev_u16(x), T)
        l, rid, rw, rc = OM.route(x, L.host, 8)
        check_route(ids, w, counts, {"ids": rid, "w": rw, "counts": rc})
        assert np.all(np.abs(w.cpu().numpy().astype(np.float64).sum(1) - 1) <= 1e-6)
    finally:
        L.close()


def test_gpu_route_ties_go_to_lower_index():
    E, H, I = 16, 128, 64
    lw = synth.layer_weights(1, 0, E, H, I)
    lw["router_w"][9] = lw["router_w"][2]          # identical rows -> identical logits
    lw["router_w"][14] = lw["router_w"][2]
    L = GpuLayer(1, 0, E, H, I, k=4, weights=lw)
    try:
        x = synth.hidden_states(1, 0, 4, H)
        ids, w, counts = L.route(to_dev_u16(x), 4)
        l, rid, rw, rc = OM.route(x, L.host, 4)
        check_route(ids, w, counts, {"ids": rid, "w": rw, "counts": rc})
        for t in range(4):
            row = ids[t].tolist()
            for a, b in ((2, 9), (2, 14), (9, 14)):
                if a in row and b in row:
                    assert row.index(a) < row.index(b)
    finally:
        L.close()


# ------------------------------------------------------------- forward --

@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("n_shared", [0, 1, 2])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_gpu_forward_small_shapes(T, n_shared, mode):
    E, H, I, k = 8, 128, 64, 2
    L = GpuLayer(2, T, E, H, I, k=k, n_shared=n_shared, fill="host")
    try:
        for step in range(3):
            x = synth.hidden_states(2, 10 * T + step, T, H)
            ids, w, counts, y, dbg = _run(L, x, mode=mode)
            ref = _oracle(L, x)
            check_route(ids, w, counts, ref)
            check_forward(y, dbg, ref)
    finally:
        L.close()


@pytest.mark.parametrize("T", [1, 4])
def test_gpu_forward_other_shape(T):
    """A second shape set through the same kernels (the shapes are run-time
    arguments): hidden 4096, expert width 1536, E = 32 top-8 + 1 shared, at one
    and at four tokens, against the oracle."""
    H, I = 4096, 1536
    L = GpuLayer(5, 7, 32, H, I)
    try:
        for step in range(2):
            x = synth.hidden_states(5, 70 + 10 * T + step, T, H)
            ids, w, counts, y, dbg = _run(L, x, mode="fused")
            ref = _oracle(L, x)
            check_route(ids, w, counts, ref)
            check_forward(y, dbg, ref)
    finally:
        L.close()


@pytest.mark.parametrize("mode", MODES)
def test_gpu_forward_config0_single_token(mode):
    """One token, E = 32 routed top-8 + 1 shared, H 2560, I 768, seed 0."""
    L = GpuLayer(0, 0, 32)
    try:
        for step in range(4):
            x = synth.hidden_states(0, step, 1, H0)
            ids, w, counts, y, dbg = _run(L, x, mode=mode)
            ref = _oracle(L, x)
            check_route(ids, w, counts, ref)
            st = check_forward(y, dbg, ref)
            print(mode, step, st)
    finally:
        L.close()


@pytest.mark.parametrize("mode", MODES)
def test_gpu_forward_config1_full_layer(mode):
    """E = 512 (the 1.6 GB layer) at full size; tokens one at a time."""
    for layer in (0, 1):
        L = GpuLayer(0, layer, 512)
        try:
            for step in range(3):
                x = synth.hidden_states(0, 1000 + 10 * layer + step, 1, H0)
                ids, w, counts, y, dbg = _run(L, x, mode=mode)
                ref = _oracle(L, x)
                check_route(ids, w, counts, ref)
                check_forward(y, dbg, ref)
                # replay: the oracle's down + combine on the GPU's own FP8 h and
                # scales isolates the down step: the GPU's output differs from
                # it only by the float32 sums of 8-block parts
                qh, sh = dbg["qh"].cpu().numpy()[0], dbg["sh"].cpu().numpy()[0]
                slots = [(int(e), float(p)) for e, p in zip(ref["ids"][0], ref["w"][0])] + [(512, 1.0)]
                y64 = np.zeros(H0)
                for si, (e, p) in enumerate(slots):
                    y64 += p * OM.down_replay(L.host.experts[e], qh[si], sh[si])
                yg = OF.bf16_to_f64(u16(y)[0])
                assert np.abs(yg - y64).max() <= 2.0 ** -8 * np.abs(y64).max() + 1e-30
                assert np.mean(OF.f64_to_bf16(y64) == u16(y)[0]) >= 0.99
        finally:
            L.close()


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("kind", ["iid", "clustered"])
def test_gpu_forward_config2_four_tokens(kind, mode):
    """Speculative verify: 4 tokens through the E = 512 layer in one call,
    i.i.d. or 4 copies of one vector + N(0, 0.1^2) noise; also equal to 4
    single-token calls."""
    L = GpuLayer(0, 2, 512)
    try:
        if kind == "iid":
            x = synth.hidden_states(0, 2000, 4, H0)
        else:
            x = synth.hidden_states_clustered(0, 2001, 4, H0)
        ids, w, counts, y, dbg = _run(L, x, mode=mode)
        ref = _oracle(L, x)
        check_route(ids, w, counts, ref)
        check_forward(y, dbg, ref)
        distinct = len(set(ref["ids"].ravel().tolist()))
        assert distinct <= 32
        for t in range(4):
            i1, w1, c1, y1, _ = _run(L, x[t:t + 1], debug=False, mode=mode)
            assert np.array_equal(i1.cpu().numpy()[0], ids.cpu().numpy()[t])
            assert np.array_equal(u16(y1)[0], u16(y)[t])
    finally:
        L.close()


def test_gpu_fused_equals_split_and_repeats():
    """moe_decode gives the routing and output of moe_route + moe_forward, and
    the same output again on back-to-back calls (its counters and
    accumulators reset themselves)."""
    L = GpuLayer(0, 5, 512, bias=True)
    try:
        for step in range(3):
            x = synth.hidden_states(0, 3000 + step, 1 + step, H0)
            a = _run(L, x, debug=False, mode="split")
            b = _run(L, x, debug=False, mode="fused")
            c = _run(L, x, debug=False, mode="fused")
            for r in (b, c):
                assert np.array_equal(a[0].cpu().numpy(), r[0].cpu().numpy())
                assert np.array_equal(a[1].cpu().numpy(), r[1].cpu().numpy())
                assert np.array_equal(a[2].cpu().numpy(), r[2].cpu().numpy())
                assert np.array_equal(u16(a[3]), u16(r[3]))
    finally:
        L.close()


# ------------------------------------------------------------ edge cases --

def test_gpu_zero_input_and_zero_weights():
    E, H, I = 8, 128, 64
    L = GpuLayer(3, 0, E, H, I, k=2, fill="host")
    try:
        x = np.zeros((2, H), np.uint16)
        ids, w, counts, y, dbg = _run(L, x)
        assert not u16(y).any()
        assert np.all(dbg["xs"].cpu().numpy() == 1.0) and not dbg["xq"].cpu().numpy().any()
    finally:
        L.close()
    lw = synth.layer_weights(3, 0, E, H, I)
    lw["w13_codes"][:] = 0
    L = GpuLayer(3, 0, E, H, I, k=2, weights=lw)
    try:
        x = synth.hidden_states(3, 1, 1, H)
        ids, w, counts, y, dbg = _run(L, x)
        assert not (u16(y) & 0x7FFF).any()
    finally:
        L.close()


def test_gpu_block_sums_beyond_float32_span():
    """Blocks whose 32 products need more than float32's 24 significant bits:
    in every 32-element block of x, elements 0..15 are large (FP8 code 448
    after the per-token scale) and elements 16..31 tiny (E4M3 subnormal
    codes), against the largest E2M1 magnitude (6) on the large elements and
    the smallest nonzero one (0.5) on the tiny ones, signs aligned so the
    large products add up: a block sum near 16 * 6 * 448 = 43008 plus terms of
    2^-10.  The tensor core's float32 block sum may round there, so this case
    is held to the layer tolerance and the FP8 rounding-boundary rule on h,
    not to bit-exact h."""
    E, H, I, k = 4, 128, 64, 2
    lw = synth.layer_weights(6, 0, E, H, I)
    rng = np.random.default_rng(6)
    big = np.float32(28.0)                      # amax: scale 28 / 448 = 2^-4, code 448
    x32 = np.empty((2, H), np.float32)
    for t in range(2):
        for b in range(H // 32):
            x32[t, 32 * b:32 * b + 16] = big
            tiny = (1.0 + rng.integers(0, 8, 16) / 8.0) * 2.0 ** -12 * rng.choice([-1.0, 1.0], 16)
            x32[t, 32 * b + 16:32 * b + 32] = tiny.astype(np.float32)
    x = synth._fp32_to_bf16_bits(x32)
    # gate/up codes: 6 (code 7) on the large elements, +-0.5 (code 1 / 9) on the tiny ones
    codes = np.empty((E + 1, 2 * I, H), np.uint8)
    codes[:, :, :] = np.where(rng.random((E + 1, 2 * I, H)) < 0.5, 1, 9)
    for b in range(H // 32):
        codes[:, :, 32 * b:32 * b + 16] = 7
    lw["w13_codes"] = (codes[:, :, 0::2] | (codes[:, :, 1::2] << 4)).astype(np.uint8)
    L = GpuLayer(6, 0, E, H, I, k=k, weights=lw)
    try:
        for mode in MODES:
            ids, w, counts, y, dbg = _run(L, x, mode=mode)
            ref = _oracle(L, x)
            assert np.all(ref["xq"][:, 0::32] == 0x7E)          # the large elements at code 448
            sub = ref["xq"][:, 16::32] & 0x7F
            assert np.all((sub > 0) & (sub < 8))                 # the tiny ones subnormal
            check_route(ids, w, counts, ref)
            yg, yr = OF.bf16_to_f64(u16(y)), OF.bf16_to_f64(ref["y"])
            rel = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
            mx = np.abs(yg - yr).max() / np.abs(yr).max()
            assert rel <= REL_L2 and mx <= MAX_ABS, (rel, mx)
            assert np.array_equal(dbg["xq"].cpu().numpy(), ref["xq"])
            # h within float32 rounding of the block sums; s_h with it
            hg, hr = dbg["h"].cpu().numpy().astype(np.float64), ref["h"].astype(np.float64)
            amax = np.abs(hr).max(axis=2, keepdims=True)
            assert np.all(np.abs(hg - hr) <= 2.0 ** -20 * amax), float((np.abs(hg - hr) / amax).max())
            assert np.allclose(dbg["sh"].cpu().numpy(), ref["sh"], rtol=2.0 ** -20, atol=0)
            # each FP8 code of h that differs is one step away, the value near their midpoint
            qg = dbg["qh"].cpu().numpy()
            for t, s_, j in np.argwhere(qg != ref["qh"]):
                va, vb = float(OF.e4m3_value(int(qg[t, s_, j]))), float(OF.e4m3_value(int(ref["qh"][t, s_, j])))
                v = hr[t, s_, j] / float(ref["sh"][t, s_])
                assert abs(abs(va) - abs(vb)) <= 2.0 ** -3 * max(abs(va), abs(vb)) + 2.0 ** -9
                assert abs(v - (va + vb) / 2) <= 2.0 ** -19 * 448 + 1e-6 * abs(v)
            print(mode, {"rel_l2": rel, "max_rel": mx, "h_exact": float(np.mean(hg == hr)),
                         "qh_flips": int((qg != ref["qh"]).sum())})
    finally:
        L.close()


def test_gpu_bad_ids_are_reported_and_skipped():
    E, H, I = 8, 128, 64
    L = GpuLayer(4, 0, E, H, I, k=2, fill="host")
    try:
        x = synth.hidden_states(4, 0, 1, H)
        xd = to_dev_u16(x)
        ids = torch.tensor([[1, 99]], dtype=torch.int32, device="cuda")
        w = torch.tensor([[0.75, 0.25]], dtype=torch.float32, device="cuda")
        y, _ = L.forward(xd, 1, ids, w, debug=False)
        assert moe.moe_device_error(L.handle) == moe.MOE_ERR_DEVICE
        assert moe.moe_device_error(L.handle) == moe.MOE_OK      # cleared
        # the valid slot and the shared expert still count
        ref = OM.moe_forward(x, np.array([[1]], np.int32), np.array([[0.75]], np.float32),
                             L.host, E, I, 1)
        yg, yr = OF.bf16_to_f64(u16(y)), OF.bf16_to_f64(ref["y"])
        assert np.linalg.norm(yg - yr) <= 2e-3 * np.linalg.norm(yr)
    finally:
        L.close()


def test_gpu_token_count_limits():
    L = GpuLayer(0, 0, 8, 128, 64, k=2, fill="host", max_tokens=4)
    try:
        x = to_dev_u16(np.zeros((8, 128), np.uint16))
        ids = torch.zeros((8, 2), dtype=torch.int32, device="cuda")
        w = torch.zeros((8, 2), dtype=torch.float32, device="cuda")
        y = torch.empty((8, 128), dtype=torch.int16, device="cuda")
        for T in (0, 5):
            with pytest.raises(moe.MoEError) as ei:
                moe.moe_forward(L.handle, x, T, ids, w, y)
            assert ei.value.code == moe.MOE_ERR_ARG
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_route(L.handle, x.data_ptr() + 2, 1, ids, w)
        assert ei.value.code == moe.MOE_ERR_ALIGN
    finally:
        L.close()


def test_gpu_residual_rmsnorm_matches_oracle():
    T, H = 3, 2560
    r = synth.hidden_states(7, 0, T, H)
    y = synth.hidden_states(7, 1, T, H)
    rd, yd = to_dev_u16(r), to_dev_u16(y)
    xn = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe.moe_residual_rmsnorm(rd, yd, xn, T, H, 1e-6)
    rr, rx = OM.residual_rmsnorm(r, y, 1e-6)
    assert np.array_equal(u16(rd), rr)
    assert np.array_equal(u16(xn), rx)
