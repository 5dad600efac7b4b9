"""Host checks of arithmetic tricks compiled into the kernels, emulated in
float32 with numpy.  CPU only.

* The attention producer's division by a run-time sub-box count (a float
  reciprocal quotient corrected by one step): exact over every argument the
  kernel can see, which the configuration check bounds (fewer than 2^22
  sub-boxes per context, at most 8,192 pool or recent slots).
* The selection's radix top-k ranks float scores by an unsigned key: the key
  order must be the float order, with -0 and +0 equal."""

import numpy as np


def _div_small(a, b, inv_b):
    """floor(a / b) the kernel's way: q = trunc(float(a) * inv_b) in float32,
    then one correction step on the remainder."""
    q = np.trunc(a.astype(np.float32) * np.float32(inv_b)).astype(np.int64)
    r = a - q * b
    return np.where(r < 0, q - 1, np.where(r >= b, q + 1, q))


def _inverses(b):
    # 1.f / b as compiled (IEEE division, correctly rounded), and one ulp either
    # side, so that the result does not hang on the last bit of the reciprocal
    inv = np.float32(1.0) / np.float32(b)
    return [inv, np.nextafter(inv, np.float32(0)), np.nextafter(inv, np.float32(1))]


def test_division_by_sub_box_counts_is_exact():
    A_MAX, SLOTS = 1 << 22, 8192
    # every numerator for small divisors (sub-boxes per compressed block: 6 at
    # the pages' scale)
    for b in range(1, 65):
        a = np.arange(min(A_MAX, SLOTS * b), dtype=np.int64)
        for inv in _inverses(b):
            assert np.array_equal(_div_small(a, b, inv), a // b), b
    # larger divisors (sub-boxes per full block: 195 at the pages' scale, up to
    # 2^19): each quotient's first and last numerator, and its neighbours
    rng = np.random.default_rng(0)
    bs = sorted({65, 100, 127, 128, 129, 195, 390, 1000, 4093, 4096, 6240, 65521, 65536, 99991,
                 (1 << 19) - 1, 1 << 19} | set(rng.integers(65, 1 << 19, 40).tolist()))
    for b in bs:
        q = np.arange(min(SLOTS, A_MAX // b + 1), dtype=np.int64)
        a = np.concatenate([q * b, q * b + b - 1, q * b + 1, np.maximum(q * b - 1, 0),
                            rng.integers(0, min(A_MAX, SLOTS * b), 4096)])
        a = a[a < min(A_MAX, SLOTS * b)]
        for inv in _inverses(b):
            assert np.array_equal(_div_small(a, b, inv), a // b), b


def _order_key(f):
    """The selection's key: -0 made +0, then negative floats bit-inverted and
    non-negative ones given the top bit."""
    u = (f.astype(np.float32) + np.float32(0.0)).view(np.uint32)
    return np.where(u & np.uint32(0x80000000), ~u, u | np.uint32(0x80000000))


def test_order_key_sorts_like_the_scores():
    rng = np.random.default_rng(1)
    tiny = np.finfo(np.float32).tiny
    special = np.array([0.0, -0.0, tiny, -tiny, tiny / 8, -tiny / 8, 1.0, -1.0,
                        np.finfo(np.float32).max, -np.finfo(np.float32).max, np.inf, -np.inf], dtype=np.float32)
    f = np.concatenate([special, rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(5000) * 1e-30).astype(np.float32),
                        rng.integers(0, 2**32, 5000, dtype=np.uint64).astype(np.uint32).view(np.float32)])
    f = f[~np.isnan(f)]
    k = _order_key(f)
    i, j = rng.integers(0, len(f), (2, 200000))
    assert np.array_equal(f[i] < f[j], k[i] < k[j])
    assert np.array_equal(f[i] == f[j], k[i] == k[j])             # -0 == +0 on both sides
    assert _order_key(np.array([-0.0], np.float32))[0] == _order_key(np.array([0.0], np.float32))[0]
