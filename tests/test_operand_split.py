"""The scoring's operand: each value x of a plane (and of a query) enters the
tensor cores as two fp16 terms, t0 = x rounded to fp16 and t1 = (x - t0)
rounded to fp16. These CPU tests pin the bounds the kernels and the design
state for that split, with numpy's round-to-nearest-even conversions standing
for the device's:

  * the remainder x - t0 is exact in fp32 (t0 is within a factor of two of x);
  * |x - t0 - t1| <= max(2^-22 |x|, 2^-25) for every |x| <= 65504: relative
    where the remainder is a normal fp16 number, absolute (half the fp16
    subnormal spacing) below;
  * from |x| >= 65520 on, t0 overflows to infinity, which makes the products
    non-finite -- the condition on which the kernel recomputes a row in fp32.
"""

import numpy as np


def _split(x32):
    with np.errstate(over="ignore", invalid="ignore"):   # overflow is one of the cases
        t0 = x32.astype(np.float16)
        r = x32 - t0.astype(np.float32)
        t1 = r.astype(np.float16)
    return t0, r, t1


def _values(rng, n):
    # magnitudes spread evenly in log2 over the fp16 range, both signs, plus
    # fp16 boundary values and their fp32 neighbours
    mag = np.exp2(rng.uniform(-30.0, np.log2(65504.0), n))
    x = (mag * rng.choice([-1.0, 1.0], n)).astype(np.float32)
    edges = np.array([65504.0, 65519.0, 2.0 ** -14, 2.0 ** -24, 2.0 ** -3, 1.0, 1.0 + 2.0 ** -11,
                      1.0 + 2.0 ** -12 + 2.0 ** -23, 3.0 * 2.0 ** -12], dtype=np.float32)
    edges = np.concatenate([edges, np.nextafter(edges, np.float32(np.inf)),
                            np.nextafter(edges, np.float32(0.0))])
    return np.concatenate([x, edges, -edges])


def test_remainder_is_exact_in_fp32():
    x = _values(np.random.default_rng(1), 200_000)
    t0, r, _ = _split(x)
    exact = x.astype(np.float64) - t0.astype(np.float64)
    assert np.array_equal(r.astype(np.float64), exact)


def test_two_terms_bound():
    x = _values(np.random.default_rng(2), 200_000)
    t0, _, t1 = _split(x)
    err = np.abs(x.astype(np.float64) - t0.astype(np.float64) - t1.astype(np.float64))
    bound = np.maximum(2.0 ** -22 * np.abs(x.astype(np.float64)), 2.0 ** -25)
    assert np.all(err <= bound)
    # the relative bound alone holds once the remainder is a normal fp16 number
    big = np.abs(x) >= 2.0 ** -2
    assert np.all(err[big] <= 2.0 ** -22 * np.abs(x[big].astype(np.float64)))
    # and it is attained to within a factor of two somewhere (the bound is not loose)
    assert np.max(err[big] / np.abs(x[big].astype(np.float64))) > 2.0 ** -24


def test_overflow_starts_at_65520():
    below = np.float32(65519.996)
    t0, _, t1 = _split(np.array([below, -below], dtype=np.float32))
    assert np.all(np.isfinite(t0)) and np.all(np.isfinite(t1))
    t0, _, t1 = _split(np.array([65520.0, -65520.0, 7.0e4], dtype=np.float32))
    assert np.all(np.isinf(t0))
    # the terms' products with a nonzero query term do not sum to a finite value
    q = np.float32(0.5)
    with np.errstate(invalid="ignore"):
        prod = t0.astype(np.float32) * q + t1.astype(np.float32) * q
    assert not np.any(np.isfinite(prod))
