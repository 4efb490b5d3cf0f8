"""The residual step forms x = bf16(r / den) as bf16(RN(r * RN(1 / den)))
and falls back to the division where that could round differently: when
the product lies within 8 float64 ulps of a midpoint between two bfloat16
values, or outside the normal bfloat16 range (zero excepted).  The product
is within 2 ulps of the exact quotient, so outside those cases both round
the same way.  This checks that condition in float64 numpy arithmetic (IEEE
round to nearest, like the GPU's) on quotients placed on, and a few ulps
around, bfloat16 midpoints, against the correctly rounded quotient."""
import numpy as np

from oracle import formats as OF


def _fast(r, den):
    inv = 1.0 / den
    q = r * inv
    b = q.view(np.uint64)
    low = b & np.uint64((1 << 45) - 1)
    ex = (b >> np.uint64(52)) & np.uint64(0x7FF)
    near = (low + np.uint64(8) >= np.uint64(1 << 44)) & (low <= np.uint64((1 << 44) + 8))
    safe = ((ex >= 897) & (ex < 0x47F) & ~near) | ((b << np.uint64(1)) == 0)
    return OF.f64_to_bf16(q), safe


def test_product_rounds_like_the_quotient_where_the_fast_path_is_taken():
    rng = np.random.default_rng(3)
    taken = 0
    for _ in range(40):
        den = rng.uniform(0.01, 100.0)
        k = rng.integers(-30, 30, 2000)
        mant = rng.integers(256, 512, 2000) | 1        # odd 9-bit significand: a bfloat16 midpoint
        mid = np.ldexp(mant.astype(np.float64), k - 8)
        r = mid * den
        rs = [r] + [(r.view(np.int64) + d).view(np.float64) for d in range(-12, 13) if d]
        rs += [rng.standard_normal(2000) * 10.0, np.zeros(2), -np.zeros(2)]
        rr = np.concatenate(rs)
        rr = np.concatenate([rr, -rr])
        got, safe = _fast(rr, den)
        want = OF.f64_to_bf16(rr / den)
        assert np.array_equal(got[safe], want[safe])
        taken += int(safe.sum())
    assert taken > 0
