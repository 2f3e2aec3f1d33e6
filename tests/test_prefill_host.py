"""Host-side checks of the prefill kernel's exp2 on the FMA pipe (exp2_poly2 in
csrc/prefill.cu), against the mathematics: the cubic's coefficients are read
from the kernel source, evaluated in fp32 the way the kernel does (Horner with
fused multiply-adds), and the Cody-Waite reconstruction (rint by adding
1.5 * 2^23, 2^j by adding j << 23 to the exponent bits) is replayed in fp32
bit arithmetic.  The stated bound is a relative error below 8e-5 over the
whole range the softmax feeds it (x <= 16, clamped at -125)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "int4_kivi_quantized_s4kv_b200", "csrc", "prefill.cu")


def _poly_source():
    text = open(SRC).read()
    body = text[text.index("float2 exp2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    return body


def _coefficients():
    body = _poly_source()
    # the Horner steps: q = c3 * f + c2, then q * f + c1, then q * f + c0
    consts = [float(c) for c in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    assert len(consts) == 4, consts
    c3, c2, c1, c0 = consts
    rnd = float(re.search(r"kRound = ([0-9.]+)f", body).group(1))
    clamp = float(re.search(r"fmaxf\(x\.x, (-[0-9.]+)f\)", body).group(1))
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3), np.float32(rnd), np.float32(clamp)


def _fma32(a, b, c):
    # fp32 fused multiply-add: the exact product-sum rounded once (float64
    # holds the product of two fp32 numbers exactly)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x):
    c0, c1, c2, c3, rnd, clamp = _coefficients()
    x = np.asarray(x, np.float32)
    xc = np.maximum(x, clamp)
    t = (xc + rnd).astype(np.float32)
    f = (xc - (t - rnd).astype(np.float32)).astype(np.float32)
    q = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.full_like(f, c0))
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_coefficients_are_read_from_the_kernel():
    c0, c1, c2, c3, rnd, clamp = _coefficients()
    assert rnd == np.float32(1.5 * 2 ** 23)
    assert clamp == np.float32(-125.0)
    # a cubic close to the Taylor series of 2^f = e^(f ln 2) (a minimax fit moves
    # the coefficients by up to about 1 %)
    ln2 = np.log(2.0)
    for c, ref in zip((c0, c1, c2, c3), (1.0, ln2, ln2 ** 2 / 2, ln2 ** 3 / 6)):
        assert abs(float(c) - ref) < 0.03 * ref


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-125.0, 16.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 8e-5, rel.max()


def test_reduction_at_integers_and_half_integers():
    # x = j exactly: f = 0, the result is p(0) * 2^j; at j + 1/2 the
    # reduction rounds to even, f = +-1/2, the ends of the fitted interval
    j = np.arange(-125, 17, dtype=np.float32)
    for x in (j, j + np.float32(0.5), j - np.float32(0.5)):
        x = x[x >= -125]
        got = _exp2_poly(x).astype(np.float64)
        rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
        assert rel.max() < 8e-5, rel.max()


def test_below_the_clamp_the_weight_is_negligible():
    # masked logits (-inf) and anything below -125 give 2^-125 (times the
    # cubic at f = 0): zero after the fp16 rounding of P, nothing to the sum
    got = _exp2_poly(np.array([-np.inf, -1e30, -300.0, -126.0], np.float32)).astype(np.float64)
    assert np.all(got > 0) and np.all(got <= 2.0 ** -124)
    assert np.all(got.astype(np.float16) == 0)
