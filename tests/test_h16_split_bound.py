"""Error bound of the fp16 S-stream's three-product form, checked on the host.

The kernel's split warps turn each scaled value v (S times its scale cS, X
times cX, both powers of two with c max|v| < 2^14) into hi = rn16(v) and
lo = rn16(v - hi); a GPU test checks those words bit for bit against the same
steps in IEEE arithmetic.  The tensor core then forms

    S_hi X_hi + S_hi X_lo + S_lo X_hi  (+ S_lo X_lo for the columns c with
                                        KP <= KP + c < N2, N2 = roundup(KP, 16))

Per operand, |hi + lo - v| <= 2^-22 |v| where lo is a normal fp16 number and
<= 2^-25 where it is not (fp16's subnormal spacing is 2^-24); the dropped
S_lo X_lo is at most 2^-22 |v_s| |v_x|.  So each entry of cS cX S X is
formed, to first order, within

    3 * 2^-22 * sum_j |s_ij| |x_jc|  +  2^-25 * sum_j (|s_ij| + |x_jc|)

(2 * 2^-22 in the first term where S_lo X_lo is formed; the second term is
at most n 2^-10 with every scaled entry below 2^14, i.e. n 2^-36 of
max|s| max|x| unless a scale sits at its cap of 2^63), before the tensor
core's fp32 accumulation.  This test emulates the split and the products in
float64 and checks that bound, and that it is reached within a small factor
(so a plausible slip in the split, such as a lost lo part, fails it).
"""
import numpy as np
import pytest


def pow2_scale(m):
    # the largest power of two c with c m < 2^14, at most 2^63; 1 for m = 0
    if not np.isfinite(m) or m <= 0:
        return 1.0
    e = np.floor(np.log2(m))
    c = 2.0 ** (13 - e)
    while c * m >= 2.0 ** 14:
        c /= 2
    while c * m * 2 < 2.0 ** 14:
        c *= 2
    return min(c, 2.0 ** 63)


def split(v32):
    """hi = rn16(v), lo = rn16(v - hi), the difference taken in float32."""
    hi = v32.astype(np.float16)
    lo = (v32 - hi.astype(np.float32)).astype(np.float32).astype(np.float16)
    return hi.astype(np.float64), lo.astype(np.float64)


def three_products(S, X, KP):
    cs = pow2_scale(float(np.abs(S).max()))
    cx = pow2_scale(float(np.abs(X).max()))
    s = (S * np.float32(cs)).astype(np.float32)
    x = (X * np.float32(cx)).astype(np.float32)
    sh, sl = split(s)
    xh, xl = split(x)
    P = sh @ xh + sh @ xl + sl @ xh
    n2 = (KP + 15) // 16 * 16
    both = [c for c in range(X.shape[1]) if KP + c < n2]
    if both:
        P[:, both] += sl @ xl[:, both]
    return P, s.astype(np.float64), x.astype(np.float64), both


def spread(rng, shape, binades):
    # magnitudes over many binades, some exact zeros and entries far below the largest
    a = rng.random(shape) * np.exp2(-rng.random(shape) * binades)
    a[rng.random(shape) < 0.02] = 0.0
    return a


@pytest.mark.parametrize("k", [24, 16, 8, 5])
@pytest.mark.parametrize("scale_s,scale_x", [(1.0, 1.0), (2.0 ** -60, 2.0 ** -55), (3.0e4, 7.0e-3),
                                              (2.0 ** 40, 2.0 ** 20)])
def test_three_product_error_within_the_stated_bound(k, scale_s, scale_x):
    rng = np.random.default_rng(k * 7 + int(np.log2(scale_s) + 100))
    n = 384
    KP = (k + 7) // 8 * 8
    S = (spread(rng, (n, n), 30) * scale_s).astype(np.float32)
    X = (spread(rng, (n, k), 30) * scale_x).astype(np.float32)
    P, s, x, both = three_products(S, X, KP)
    exact = s @ x
    absprod = np.abs(s) @ np.abs(x)
    rel = np.full(k, 3 * 2.0 ** -22)
    rel[both] = 2 * 2.0 ** -22
    small = np.abs(s).sum(axis=1)[:, None] + np.abs(x).sum(axis=0)[None, :]
    bound = (absprod * rel + 2.0 ** -25 * small) * (1 + 2.0 ** -10)
    assert np.all(2.0 ** -25 * small <= n * 2.0 ** -10)
    if np.abs(s).max() >= 2.0 ** 13 and np.abs(x).max() >= 2.0 ** 13:   # neither scale capped
        assert np.all(2.0 ** -25 * small <= n * 2.0 ** -36 * np.abs(s).max() * np.abs(x).max())
    err = np.abs(P - exact)
    assert np.all(err <= bound), float(np.max(err / bound))


def test_split_error_reaches_its_bound_and_no_further():
    # per operand: |hi + lo - v| <= 2^-22 |v| + 2^-25; the relative part comes
    # within a factor of about two where lo is a normal fp16 number (both
    # roundings cannot be at their worst at once)
    rng = np.random.default_rng(5)
    v = (rng.random(1 << 18) * 2.0 ** 14).astype(np.float32)
    v = np.concatenate([v, np.exp2(rng.uniform(-30, 14, 1 << 16)).astype(np.float32)])
    hi, lo = split(v)
    v64 = v.astype(np.float64)
    err = np.abs(hi + lo - v64)
    assert np.all(err <= 2.0 ** -22 * v64 + 2.0 ** -25)
    big = v64 >= 2.0
    assert (err[big] / v64[big]).max() >= 0.4 * 2.0 ** -22


def test_bound_is_nearly_reached_and_a_lost_lo_part_breaks_it():
    # inner dimension 1 (no cancellation across j): the product error comes
    # within a factor of four of the bound, and dropping X_lo exceeds it
    rng = np.random.default_rng(6)
    m, k = 4096, 24
    S = rng.random((m, 1)).astype(np.float32) + np.float32(0.5)
    X = rng.random((1, k)).astype(np.float32) + np.float32(0.5)
    P, s, x, both = three_products(S, X, 24)
    exact = s @ x
    absprod = np.abs(s) @ np.abs(x)
    rel = np.full(k, 3 * 2.0 ** -22)
    rel[both] = 2 * 2.0 ** -22
    ratio = np.abs(P - exact) / (absprod * rel)
    assert ratio.max() <= 1.0 + 2.0 ** -10
    assert ratio.max() >= 0.25
    # a split that lost X_lo (the products S_hi X_hi + S_lo X_hi alone)
    sh, sl = split(s.astype(np.float32))
    xh, _ = split(x.astype(np.float32))
    bad = sh @ xh + sl @ xh
    assert np.any(np.abs(bad - exact) > absprod * rel * (1 + 2.0 ** -10))
