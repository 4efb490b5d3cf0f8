"""Seeded synthetic inputs for the MXFP4 MoE layer (host side).

This module generates inputs only: expert weight bytes, router weights,
router bias and hidden states.  It holds none of the layer's arithmetic and
is the one module that both the oracle and the CUDA path draw inputs from.
``synth/fill.cu`` implements the same generator on the GPU (for the
full-size, tens-of-GB weight sets); the two are compared byte for byte in
the tests.

Generator definition (counter based, so any element can be drawn on its
own):

* ``mix64`` is the SplitMix64 output function (Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014):
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31`` (all mod 2**64).
* A stream is named by ``(seed, layer, tensor, expert)``; its key is
  ``k0 = mix64(seed + G)``, ``k1 = mix64(k0 + (layer+1) G)``,
  ``k2 = mix64(k1 + (tensor+1) G)``, ``key = mix64(k2 + (expert+1) G)``
  with ``G = 0x9E3779B97F4A7C15``.
* Word ``i`` of a stream is ``mix64(key + (i+1) G)``.
* Random bytes: byte ``8i+j`` is byte ``j`` (little endian) of word ``i``.
  Every nibble of such a byte is uniform on 0..15, i.e. a uniform E2M1 code.
* Integers in ``[lo, hi]``: element ``i`` is ``lo + word(i) mod (hi-lo+1)``.
* Normals: element ``i`` sums the twelve 16-bit fields of words
  ``3i, 3i+1, 3i+2`` (Irwin-Hall sum of 12 uniforms, the classic
  approximation to N(0,1)); ``n = (S - 393210) / 65536`` is exact in
  binary floating point.  The stored value is ``bf16(fp32(n * sigma))``,
  each rounding to nearest even, so both implementations agree bit for bit.
"""
from __future__ import annotations

import numpy as np

G = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)

# tensor ids of the streams
ROUTER_W = 0
W13_CODES = 1
W13_SCALES = 2
W2_CODES = 3
W2_SCALES = 4
HIDDEN = 5
BIAS_PERM = 6
NOISE = 7
LM_HEAD = 8

SCALE_LO = 120   # E8M0 exponent range of the synthetic weights
SCALE_HI = 124
ROUTER_SIGMA = 0.02
LM_HEAD_SIGMA = 0.02


def mix64(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = z ^ (z >> np.uint64(30))
        z = z * M1
        z = z ^ (z >> np.uint64(27))
        z = z * M2
        z = z ^ (z >> np.uint64(31))
    return z


def _u64(v: int) -> np.ndarray:
    return np.array([v & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)


def stream_key(seed: int, layer: int, tensor: int, expert: int) -> int:
    with np.errstate(over="ignore"):
        k = mix64(_u64(seed) + G)
        k = mix64(k + _u64(layer + 1) * G)
        k = mix64(k + _u64(tensor + 1) * G)
        k = mix64(k + _u64(expert + 1) * G)
    return int(k[0])


def words(key: int, start: int, count: int) -> np.ndarray:
    """Words ``start .. start+count-1`` of the stream with this key."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(_u64(key) + idx * G)


def random_bytes(key: int, nbytes: int, start_byte: int = 0) -> np.ndarray:
    """Bytes ``start_byte .. start_byte+nbytes-1`` of the stream."""
    w0 = start_byte // 8
    w1 = (start_byte + nbytes + 7) // 8
    b = words(key, w0, w1 - w0).view(np.uint8)   # little endian host
    off = start_byte - 8 * w0
    return b[off:off + nbytes].copy()


def random_ints(key: int, n: int, lo: int, hi: int, start: int = 0) -> np.ndarray:
    w = words(key, start, n)
    return (np.uint64(lo) + w % np.uint64(hi - lo + 1)).astype(np.int64)


def _fp32_to_bf16_bits(v32: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); finite inputs."""
    b = np.asarray(v32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def normals_bf16(key: int, n: int, sigma: float, start: int = 0) -> np.ndarray:
    """``n`` approximately N(0, sigma^2) values as bfloat16 bit patterns."""
    w = words(key, 3 * start, 3 * n).reshape(n, 3)
    s = np.zeros(n, dtype=np.int64)
    for j in range(3):
        col = w[:, j]
        for f in range(4):
            s += ((col >> np.uint64(16 * f)) & np.uint64(0xFFFF)).astype(np.int64)
    z = (s - 393210).astype(np.float64) / 65536.0
    v32 = (z * np.float64(sigma)).astype(np.float32)
    return _fp32_to_bf16_bits(v32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- tensors --

def router_weight(seed: int, layer: int, n_experts: int, hidden: int) -> np.ndarray:
    """BF16 bits ``[E][H]``, ~N(0, 0.02^2)."""
    key = stream_key(seed, layer, ROUTER_W, 0)
    return normals_bf16(key, n_experts * hidden, ROUTER_SIGMA).reshape(n_experts, hidden)


def expert_codes(seed: int, layer: int, expert: int, which: str, rows: int, k: int,
                 row0: int = 0, nrows: int | None = None) -> np.ndarray:
    """Packed E2M1 codes ``[rows][k/2]`` of one expert matrix.

    ``which`` is ``"w13"`` (gate rows then up rows) or ``"w2"``."""
    tensor = W13_CODES if which == "w13" else W2_CODES
    nrows = rows if nrows is None else nrows
    key = stream_key(seed, layer, tensor, expert)
    rb = k // 2
    return random_bytes(key, nrows * rb, row0 * rb).reshape(nrows, rb)


def expert_scales(seed: int, layer: int, expert: int, which: str, rows: int, k: int,
                  row0: int = 0, nrows: int | None = None) -> np.ndarray:
    """E8M0 exponents ``[rows][k/32]``, uniform on [SCALE_LO, SCALE_HI]."""
    tensor = W13_SCALES if which == "w13" else W2_SCALES
    nrows = rows if nrows is None else nrows
    key = stream_key(seed, layer, tensor, expert)
    nb = k // 32
    v = random_ints(key, nrows * nb, SCALE_LO, SCALE_HI, row0 * nb)
    return v.astype(np.uint8).reshape(nrows, nb)


def lmhead_weight(seed: int, vocab: int, hidden: int, row0: int = 0, nrows: int | None = None) -> np.ndarray:
    """BF16 bits ``[nrows][H]`` of the output layer ``[vocab][H]``, rows
    ``row0 ..``, ~N(0, 0.02^2)."""
    n = vocab - row0 if nrows is None else nrows
    key = stream_key(seed, 0, LM_HEAD, 0)
    return normals_bf16(key, n * hidden, LM_HEAD_SIGMA, start=row0 * hidden).reshape(n, hidden)


def hidden_states(seed: int, step: int, T: int, hidden: int) -> np.ndarray:
    """BF16 bits ``[T][H]``, ~N(0,1); a fresh draw per ``(seed, step)``."""
    key = stream_key(seed, step, HIDDEN, 0)
    return normals_bf16(key, T * hidden, 1.0).reshape(T, hidden)


def hidden_states_clustered(seed: int, step: int, T: int, hidden: int,
                            noise: float = 0.1) -> np.ndarray:
    """``T`` copies of one N(0,1) vector plus N(0, noise^2), as BF16 bits.

    Each row is ``bf16(fp32(v + noise * n_t))`` with v and n_t drawn from
    the Irwin-Hall generator in float64."""
    kv = stream_key(seed, step, HIDDEN, 0)
    v = bf16_bits_to_f64(normals_bf16(kv, hidden, 1.0))
    out = np.empty((T, hidden), dtype=np.uint16)
    for t in range(T):
        kn = stream_key(seed, step, NOISE, t)
        n = bf16_bits_to_f64(normals_bf16(kn, hidden, 1.0))
        out[t] = _fp32_to_bf16_bits((v + noise * n).astype(np.float32))
    return out


def zipf_router_bias(seed: int, layer: int, n_experts: int, alpha: float = 1.1) -> np.ndarray:
    """Router bias ``b_e = -alpha * ln(rank_e)`` (float32), where ``rank`` is a
    seeded permutation of 1..E.  Larger bias = more popular expert, so the
    selection frequency falls off roughly as a Zipf law in rank."""
    key = stream_key(seed, layer, BIAS_PERM, 0)
    w = words(key, 0, n_experts)
    order = np.argsort(w, kind="stable")
    rank = np.empty(n_experts, dtype=np.int64)
    rank[order] = np.arange(1, n_experts + 1)
    return (-alpha * np.log(rank.astype(np.float64))).astype(np.float32)


def expert_weights(seed: int, layer: int, expert: int, hidden: int, inter: int) -> dict:
    """All four arrays of one expert (host, numpy)."""
    return {
        "w13_codes": expert_codes(seed, layer, expert, "w13", 2 * inter, hidden),
        "w13_scales": expert_scales(seed, layer, expert, "w13", 2 * inter, hidden),
        "w2_codes": expert_codes(seed, layer, expert, "w2", hidden, inter),
        "w2_scales": expert_scales(seed, layer, expert, "w2", hidden, inter),
    }


def layer_weights(seed: int, layer: int, n_experts: int, hidden: int, inter: int,
                  n_shared: int = 1) -> dict:
    """Every expert of one layer stacked ``[E + n_shared][...]`` (small E only)."""
    ex = [expert_weights(seed, layer, e, hidden, inter) for e in range(n_experts + n_shared)]
    out = {k: np.stack([d[k] for d in ex]) for k in ex[0]}
    out["router_w"] = router_weight(seed, layer, n_experts, hidden)
    return out
