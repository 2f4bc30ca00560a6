"""The decoders compute an outlier record's value q / 127 (R15: the fp32 IEEE
quotient) without a division instruction: x0 = RN(q * r) with r = RN(1/127),
res = RN(q - 127 x0) (one fused multiply-add), x = RN(x0 + res * r) (another).
This checks that scheme against the exactly rounded quotient for every q the
8-bit record can hold, in exact rational arithmetic (no GPU needed).  The GPU
parity tests then check the kernels against the oracle's IEEE division."""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def rn32(x: Fraction) -> np.float32:
    """Round a rational to the nearest fp32, ties to even."""
    f = np.float32(float(x))
    best = None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        d = abs(Fraction(float(c)) - x)
        even = (np.array([c], dtype=np.float32).view(np.uint32)[0] & 1) == 0
        if best is None or d < best[0] or (d == best[0] and even):
            best = (d, c)
    return np.float32(best[1])


def test_reciprocal_constant_is_the_rounded_reciprocal():
    r = rn32(Fraction(1, 127))
    assert np.array([r], dtype=np.float32).view(np.uint32)[0] == 0x3C010204


def test_corrected_quotient_is_exactly_rounded_for_every_record_value():
    r = Fraction(float(rn32(Fraction(1, 127))))
    for q in range(-128, 128):
        x0 = Fraction(float(rn32(q * r)))
        exact_res = q - 127 * x0
        res = Fraction(float(rn32(exact_res)))
        assert res == exact_res, q  # the residual is representable: the first FMA is exact
        x = rn32(res * r + x0)
        assert x == rn32(Fraction(q, 127)), q
