"""The division-free quotient the quantise-append kernels use for every code decision
(`quotient_rn` in the CUDA sources): q0 = RN(a * y), r = RN(a - q0 * b) by one fused
multiply-add, q = RN(q0 + r * y) by another, with y = RN(1/b). The kernels rely on q
being exactly RN(a / b) whenever b has at most 11 significant bits (an fp16 scale, or
the constants 15 and 127). This file checks that claim on the arithmetic itself, with
every rounding done exactly (rational arithmetic, round-to-nearest-even to binary32),
on random operands over many binades and on operands built to sit on or next to
rounding midpoints and code-decision ties. CPU only; it does not run the kernels (the
GPU parity tests compare their codes with the oracle's IEEE divisions)."""
from fractions import Fraction

import numpy as np


def rn32(x: Fraction) -> np.float32:
    """x rounded to binary32, nearest-even (normal range)."""
    f = np.float32(float(x))  # within one ulp; pick the nearest neighbour exactly
    best, best_err = None, None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        err = abs(Fraction(float(c)) - x)
        if best is None or err < best_err or (
                err == best_err and (int(c.view(np.uint32)) & 1) == 0):
            best, best_err = c, err
    return best


def fma32(a, b, c) -> np.float32:
    return rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def quotient_rn(a, b, y):
    q0 = rn32(Fraction(float(a)) * Fraction(float(y)))
    r = fma32(-q0, b, a)
    return fma32(r, y, q0)


def exact(a, b):
    return rn32(Fraction(float(a)) / Fraction(float(b)))


def divisors(rng, n):
    """Positive divisors with at most 11 significant bits: fp16 values over the fp16
    normal and subnormal range, plus 15 and 127."""
    bits = rng.integers(1, 0x7C00, n).astype(np.uint16)  # positive finite fp16 patterns
    b = bits.view(np.float16).astype(np.float32)
    return np.concatenate([b, np.float32([15.0, 127.0])])


def test_random_operands_over_many_binades():
    rng = np.random.default_rng(1)
    bs = divisors(rng, 1500)
    for b in bs:
        y = rn32(Fraction(1) / Fraction(float(b)))
        for _ in range(3):
            # numerators whose quotient spans |a/b| in [2^-20, 2^10] (codes live below 2^8)
            q_target = np.float32(rng.choice([-1, 1]) * 2.0 ** rng.uniform(-20, 10))
            a = np.float32(q_target * b)
            if not np.isfinite(a) or a == 0 or abs(float(a)) < 2.0 ** -120:
                continue
            assert quotient_rn(a, b, y) == exact(a, b), (a, b)


def test_ties_and_their_neighbours():
    """Quotients that are exact half-integers (the code-decision ties bf16 inputs hit
    often) and numerators one ulp either side of them."""
    rng = np.random.default_rng(2)
    bs = divisors(rng, 400)
    checked = 0
    for b in bs:
        y = rn32(Fraction(1) / Fraction(float(b)))
        for k in rng.integers(0, 255, 4):
            a = np.float32((float(k) + 0.5) * float(b))
            if not np.isfinite(a) or a == 0 or abs(float(a)) < 2.0 ** -120:
                continue
            for cand in (np.nextafter(a, np.float32(-np.inf)), a,
                         np.nextafter(a, np.float32(np.inf))):
                assert quotient_rn(cand, b, y) == exact(cand, b), (cand, b)
                checked += 1
    assert checked > 3000


def test_plain_reciprocal_product_is_not_enough():
    """Without the correction step the product alone misses RN(a/b) on some operands,
    which is why the kernels take the second fma."""
    rng = np.random.default_rng(3)
    misses = 0
    for b in divisors(rng, 300):
        y = rn32(Fraction(1) / Fraction(float(b)))
        for _ in range(5):
            a = np.float32(rng.uniform(1, 2) * 2.0 ** rng.integers(-5, 6) * float(b))
            if not np.isfinite(a) or a == 0:
                continue
            if rn32(Fraction(float(a)) * Fraction(float(y))) != exact(a, b):
                misses += 1
    assert misses > 0


def test_rounding_by_the_magic_add_and_the_code_extraction():
    """The kernels round a quotient q to the nearest-even integer by one binary32 add,
    y = q + 1.5*2^23 (the add itself rounds to an integer for |q| < 2^22), and read the
    code from y's bits: the low nibble is the INT4 code for results in [0, 15], the low
    byte the int8 code (two's complement) for results in [-127, 127]; two INT4 codes
    pack into a byte as y_even + (y_odd << 4)."""
    rng = np.random.default_rng(4)
    magic = np.float32(12582912.0)
    q = np.concatenate([rng.uniform(-200, 200, 20000),
                        np.arange(-255, 256) / 2.0]).astype(np.float32)  # includes ties
    y = (q + magic).astype(np.float32)
    assert np.array_equal(y - magic, np.rint(q))             # nearest-even integer
    bits = y.view(np.uint32)
    r = np.rint(q).astype(np.int64)
    m4 = (r >= 0) & (r <= 15)
    assert np.array_equal(bits[m4] & 0xF, r[m4])
    m8 = (r >= -127) & (r <= 127)
    low = (bits[m8] & 0xFF).astype(np.uint8).view(np.int8)
    assert np.array_equal(low, r[m8].astype(np.int8))
    ce, co = rng.integers(0, 16, 1000), rng.integers(0, 16, 1000)
    ye = (ce.astype(np.float32) + magic).view(np.uint32).astype(np.uint64)
    yo = (co.astype(np.float32) + magic).view(np.uint32).astype(np.uint64)
    assert np.array_equal((ye + (yo << 4)) & 0xFF, ce | (co << 4))
