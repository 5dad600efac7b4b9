"""Host checks of constants and arithmetic tricks compiled into the kernels,
emulated in float32 with numpy.  CPU only.

* The cubic that the attention softmax can use for part of its exponentials
  (an option of the attention kernel): the coefficients in ptx.cuh must be
  the ones the fitting script produces, and the whole evaluation (round to
  integer by the 1.5 * 2^23 trick, cubic on the fraction, exponent bits
  added) must stay within the stated relative error.
* The attention producer's division by a run-time sub-box count (a float
  reciprocal quotient corrected by one step): exact over every argument the
  kernel can see, which the configuration check bounds (fewer than 2^22
  sub-boxes per context, at most 8,192 pool or recent slots).
* The selection's radix top-k ranks float scores by an unsigned key: the key
  order must be the float order, with -0 and +0 equal."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "packed_kv_cache_b200", "csrc", "ptx.cuh")


def _fit():
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(ROOT, "tests", "fit_exp2.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.remez_relative()


def _source_coefficients(func):
    src = open(PTX).read()
    body = src[src.index(f"{func}("):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]
    return sorted(set(vals))


def _ex2_poly_f32(x, c):
    """The kernel's steps in float32 (separate rounding for multiply and add
    where the kernel fuses them: at most one ulp apart)."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    f = (x - (t - magic)).astype(f32)
    c0, c1, c2, c3 = (f32(v) for v in c)
    p = (c3 * f + c2).astype(f32)
    p = (p * f + c1).astype(f32)
    p = (p * f + c0).astype(f32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(f32)


def test_coefficients_are_the_fitted_ones():
    c, err = _fit()
    assert 5e-5 < err < 1e-4                                   # the level the comment states (7.5e-5)
    got = _source_coefficients("ex2_poly")
    assert len(got) == 4
    assert np.allclose(sorted(c), got, rtol=1e-8, atol=0)
    # the paired form uses the same four numbers
    assert _source_coefficients("ex2_poly_x2") == got


def test_evaluation_error_over_the_softmax_range():
    c, _ = _fit()
    # softmax arguments are <= 0 after the running max is subtracted (base 2);
    # the lazy rescale lets them reach +8 before the max moves
    x = np.concatenate([np.linspace(-125.0, 8.0, 400_001), np.arange(-125, 9, dtype=np.float64)])
    y = _ex2_poly_f32(x, c).astype(np.float64)
    rel = np.abs(y - np.exp2(x)) / np.exp2(x)
    assert rel.max() < 1.2e-4, rel.max()
    # below the clamp every result is the clamp's value, about 2^-126 (the cubic
    # is just under 1 there, so the encoding is subnormal): never 0, NaN or large
    low = _ex2_poly_f32(np.array([-126.0, -200.0, -1e4, -1e30]), c).astype(np.float64)
    assert np.all(low == low[0]) and abs(low[0] / 2.0 ** -126 - 1) < 2e-4


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
