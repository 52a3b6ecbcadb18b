"""The two identities the selection's floating-point count rests on, checked in fp32 on
the CPU (the kernel's counts are compared with the oracle on the GPU elsewhere):

1. for an order key c of a finite float (c above the smallest) and scores s that are never
   -0 (the kernel adds +0 to each), key(s) >= c exactly when s > f, where f is the float
   whose key is c - 1, stepped one key further down where that float is -0 (it compares
   equal to the score +0);
2. (s - f) * inf saturated to [0, 1] is 1 exactly when s > f (it is +inf above, -inf
   below and NaN at equality; saturation sends NaN to 0), for every finite s and f, with
   s = -inf (a non-candidate) giving 0.
"""
import numpy as np


def order_key(x: np.ndarray) -> np.ndarray:
    u = x.astype(np.float32).view(np.uint32)
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def key_float(k: np.ndarray) -> np.ndarray:
    k = k.astype(np.uint32)
    u = np.where(k & 0x80000000, k & 0x7FFFFFFF, ~k).astype(np.uint32)
    return u.view(np.float32)


def float_below_key(c: np.ndarray) -> np.ndarray:
    k = (c.astype(np.uint32) - np.uint32(1)).astype(np.uint32)
    return key_float(np.where(k == 0x7FFFFFFF, k - np.uint32(1), k).astype(np.uint32))


def saturate(x: np.ndarray) -> np.ndarray:
    return np.where(np.isnan(x), np.float32(0), np.clip(x, 0, 1)).astype(np.float32)


def _floats(n, seed):
    rng = np.random.default_rng(seed)
    x = np.concatenate([  # normal, tiny, huge, and the special finite values
        rng.standard_normal(n).astype(np.float32),
        (rng.standard_normal(n) * 1e-30).astype(np.float32),
        (rng.standard_normal(n) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, np.finfo(np.float32).tiny, -np.finfo(np.float32).tiny,
                  np.finfo(np.float32).max, -np.finfo(np.float32).max, 1e-45, -1e-45], dtype=np.float32),
    ])
    # and each value's neighbours in float order
    with np.errstate(over="ignore"):
        up = np.nextafter(x, np.float32(np.inf)).astype(np.float32)
        dn = np.nextafter(x, np.float32(-np.inf)).astype(np.float32)
    keep = np.isfinite(up) & np.isfinite(dn)
    x, up, dn = x[keep], up[keep], dn[keep]
    return np.concatenate([x, up, dn])


def test_key_round_trip_and_order():
    x = _floats(2000, 0)
    assert np.array_equal(key_float(order_key(x)).view(np.uint32), x.view(np.uint32))
    # strictly increasing keys for strictly increasing floats (-0 and +0 compare equal as
    # floats and are two keys, -0 below +0)
    xs = np.sort(x)
    ks = order_key(xs).astype(np.int64)
    strict = xs[1:] > xs[:-1]
    assert np.all(np.diff(ks)[strict] > 0)
    assert order_key(np.array([-0.0], dtype=np.float32))[0] + 1 == order_key(np.array([0.0], dtype=np.float32))[0]


def test_key_threshold_equals_strict_float_compare():
    s = (_floats(3000, 1) + np.float32(0)).astype(np.float32)  # -0 becomes +0, as in the kernel
    assert not np.any((s == 0) & np.signbit(s))
    c = order_key(_floats(300, 2))
    c = np.concatenate([c, order_key(np.array([0.0, -0.0], dtype=np.float32))])  # the thresholds at the zeros
    c = c[c > order_key(np.array([-np.finfo(np.float32).max], dtype=np.float32))[0]]  # c - 1 stays finite
    f = float_below_key(c)
    assert np.all(np.isfinite(f))
    lhs = order_key(s)[:, None] >= c[None, :]
    rhs = s[:, None] > f[None, :]
    assert np.array_equal(lhs, rhs)
    # without the step past -0 the threshold at +0's key would miss the score +0
    k0 = order_key(np.array([0.0], dtype=np.float32))
    assert not (np.float32(0.0) > key_float(k0 - np.uint32(1))[0])


def test_saturated_product_is_the_strict_compare():
    s = np.concatenate([_floats(1500, 3), np.array([-np.inf], dtype=np.float32)])
    f = _floats(200, 4)
    with np.errstate(invalid="ignore", over="ignore"):
        ind = saturate((s[:, None] - f[None, :]).astype(np.float32) * np.float32(np.inf))
    assert np.array_equal(ind == 1, s[:, None] > f[None, :])
    assert np.all((ind == 0) | (ind == 1))
