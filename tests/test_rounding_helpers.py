"""The tests' FP64 -> BF16 rounding helper (the reference side of every bit-exact BF16 comparison)
against round-to-nearest-even worked out in exact rational arithmetic: normal values, midpoints of
both parities, BF16 subnormals (a fixed grid of 2^-133), the step into the normal range, overflow to
infinity and signed zeros.  Every copy of the helper (the GPU tests and the host-emulation scripts
each carry one) must agree."""
import os
import sys
from fractions import Fraction

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "host_emulation"))


def bf16_rne_exact(v: float) -> int:
    """BF16 bits of v by the definition: the nearest value of the form m * 2^(e-7), 128 <= m < 256
    (normal) or m * 2^-133, m < 128 (subnormal), ties to even m; infinity from 2^128 - 2^119 up."""
    sign = 0x8000 if np.signbit(v) else 0
    a = Fraction(abs(v))
    if a == 0:
        return sign
    e = -126
    while a >= Fraction(2) ** (e + 1):
        e += 1
    q = a / Fraction(2) ** (e - 7)
    m = q.numerator // q.denominator
    rem = q - m
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
        m += 1
    if m == 256:
        m, e = 128, e + 1
    if e > 127:
        return sign | 0x7F80
    if m < 128:  # subnormal: exponent field 0
        return sign | m
    return sign | ((e + 127) << 7) | (m - 128)


VALUES = [1.0, -1.0, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40, 3.1415926, -2.0 ** -126,
          2.0 ** -126 * (1 - 2.0 ** -9), 2.0 ** -127, 3 * 2.0 ** -134, 5 * 2.0 ** -134, 2.0 ** -134 + 2.0 ** -160,
          2.0 ** -135, 1.7e-40, -1.7e-40, 0.0, -0.0, 3.3895e38, 3.3896e38, 3.3961e38, 3.4e38, 1e39, -1e39]


def _copies():
    import cases
    import library_cases
    import test_gpu_bwd
    import test_gpu_neighbors
    return [test_gpu_bwd.f64_to_bf16_bits, test_gpu_neighbors.f64_to_bf16_bits, cases.f64_to_bf16_bits,
            library_cases.f64_to_bf16_bits]


@pytest.mark.parametrize("which", range(4))
def test_f64_to_bf16_helper_matches_exact_rounding(which):
    f = _copies()[which]
    got = f(np.array(VALUES))
    want = np.array([bf16_rne_exact(v) for v in VALUES], dtype=np.uint16)
    assert got.tolist() == want.tolist()
    rng = np.random.default_rng(3)
    x = np.ldexp(rng.uniform(-2, 2, 4000), rng.integers(-140, 130, 4000))
    assert f(x).tolist() == [bf16_rne_exact(v) for v in x]
