"""The FMA-pipe exp2 of the attention kernel, pinned against fp64 exp2.

The kernel evaluates part of its exponentials as 2^x = 2^n * p(f) with x = n + f,
n = rint(x), |f| <= 1/2, a degree-3 polynomial p fitted for minimax relative error, and 2^n
applied by an integer add to the exponent field (x clamped to [-125, 126]).  This test reads
the coefficients and the clamp from the kernel source, replays that float32 evaluation (range
reduction by the 1.5 * 2^23 rounding trick, Horner with fused multiply-adds, the exponent
add) on a dense sweep of x in [-125, 126], and checks the relative error against fp64 exp2
stays within the fit's bound (7.5e-5), the bound the attention's bf16 and e4m3 rounding of P
absorbs.  Above the clamp the value must stay huge and positive: the speculative softmax
relies on it to notice a tile whose scores rose far above the running max."""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "long_sequence_attention_b200", "csrc", "attn_fwd.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("void exp2_fma2("):]
    body = body[:body.index("\n}\n")]
    consts = re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)
    vals = [float(c) for c in consts if float(c) != 12582912.0]
    assert len(vals) == 4, vals
    assert "fminf(fmaxf(x0, -125.0f), 126.0f)" in body and "fminf(fmaxf(x1, -125.0f), 126.0f)" in body
    return [np.float32(v) for v in vals]          # c3, c2, c1, c0 in Horner order


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_kernel(x):
    c3, c2, c1, c0 = _coefficients()
    x = np.minimum(np.maximum(x.astype(np.float32), np.float32(-125.0)), np.float32(126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_exp2_polynomial_within_fit_bound():
    x = np.concatenate([np.linspace(-125.0, 126.0, 4_000_001, dtype=np.float64),
                        np.arange(-125, 126, dtype=np.float64) + 0.5, np.arange(-125, 127, dtype=np.float64)])
    x32 = x.astype(np.float32)
    got = _exp2_kernel(x32).astype(np.float64)
    ref = np.exp2(x32.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= 7.6e-5, rel.max()
    assert rel.max() > 1e-5                      # the bound is the polynomial's, not a float32 rounding


def test_exp2_polynomial_clamps_below_minus_125():
    got = _exp2_kernel(np.array([-125.0, -126.5, -300.0, -1e30], dtype=np.float32)).astype(np.float64)
    assert np.all(np.abs(got / 2.0 ** -125 - 1.0) <= 7.6e-5) and np.all(got > 0)


def test_exp2_polynomial_stays_huge_above_126():
    """Without the upper clamp, n >= 128 would carry into the sign bit and return a tiny
    negative number, which a row sum would accept: the key would silently be dropped."""
    x = np.array([126.0, 126.4, 127.0, 128.0, 130.0, 200.0, 1e6, 1e30], dtype=np.float32)
    got = _exp2_kernel(x).astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(got >= 2.0 ** 125.9)
    # one such value already exceeds the largest row-sum bound the kernel accepts (2^8)
    assert np.all(got > 2.0 ** 8)
