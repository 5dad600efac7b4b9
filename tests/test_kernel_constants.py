"""Host checks of constants compiled into the kernels: the cubic that the
attention softmax can use for part of its exponentials (an option of the
attention kernel).  The coefficients in ptx.cuh must be the ones the fitting
script produces, and the whole evaluation (round-to-integer by the 1.5 * 2^23
trick, cubic on the fraction, exponent bits added) must stay within the
stated relative error.  CPU only."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "packed_kv_cache_b200", "csrc", "ptx.cuh")


def _fit():
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(ROOT, "packed_kv_cache_b200", "fit_exp2.py"))
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
