"""The FMA-pipe exp2 of the kernel (csrc/tfa_ptx.cuh, exp2_poly2), replayed in
float32 with the same operations, against float64 exp2 and against the Remez
fit that produced its constants."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "sliding_window_gqa_tfa_b200", "csrc", "tfa_ptx.cuh")
sys.path.insert(0, os.path.join(ROOT, "sliding_window_gqa_tfa_b200", "csrc"))


def _coeffs():
    text = open(PTX).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1)))
            for i in range(4)]


def _exp2_poly(x):
    """float32 replay: clamp, round-by-magic, reduce, Horner (fma), scale by 2^n."""
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)  # fma(n, -1, x) is exact here
    p = (np.float64(c3) * f + c2).astype(np.float32)          # fma: one rounding
    p = (p.astype(np.float64) * f + c1).astype(np.float32)
    p = (p.astype(np.float64) * f + c0).astype(np.float32)
    tbits = t.view(np.uint32)
    scale = ((tbits << np.uint32(23)) + np.uint32(0x3F800000)).astype(np.uint32).view(np.float32)
    return (p * scale).astype(np.float32)


def test_relative_error_over_the_kernel_range():
    x = np.linspace(-120.0, 8.0, 2_000_001).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()


def test_masked_scores_give_exact_zero_and_integers_are_exact_powers():
    x = np.array([-np.inf, -1e30, -127.0, -126.6], dtype=np.float32)
    assert np.all(_exp2_poly(x) == 0.0)
    k = np.arange(-100, 9, dtype=np.float32)
    got = _exp2_poly(k)
    assert np.allclose(got, np.exp2(k.astype(np.float64)), rtol=1e-4, atol=0)


def test_constants_match_the_remez_fit():
    import gen_exp2_poly

    coef, err = gen_exp2_poly.remez_exp2(3)
    assert err < 8e-5
    for c, k in zip(coef, _coeffs()):
        assert abs(np.float32(c) - k) <= 1e-7 * max(1.0, abs(float(k)))
