"""IEEE identities the attention kernels rely on to feed codes to the fp16 tensor cores
without conversions, checked on every code value with numpy's binary16 (CPU only):

* a half whose exponent field is 0 and whose low nibble is a code c (the rest zero) is
  exactly c * 2^-24; a code in bits 4-7 gives exactly 16c * 2^-24 (V codes as
  subnormals; the kernels undo 2^24 and 2^20 once per output row);
* an int8 code b placed, offset by 128, in the low byte of a half with high byte 0x64
  is 1024 + (b + 128); subtracting 1152 gives b exactly (INT8 codes by one byte permute
  and one half subtraction);
* P' = p * scale rounded once to fp16 and multiplied by a subnormal code is exact in
  fp32 (the tensor-core product of two halves needs at most 22 significant bits).
"""
import numpy as np


def halves(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16)


def test_nibble_codes_as_subnormal_halves():
    c = np.arange(16, dtype=np.uint16)
    assert np.array_equal(halves(c).astype(np.float64), c * 2.0 ** -24)
    assert np.array_equal(halves(c << 4).astype(np.float64), 16 * c * 2.0 ** -24)
    # the pair masks of one 32-bit word: (t0, t1) dims 0 and 1 of a transposed V word
    rng = np.random.default_rng(0)
    w = rng.integers(0, 2 ** 32, 1000, dtype=np.uint64).astype(np.uint32)
    lo = (w & 0x000F000F).astype(np.uint32).view(np.uint16).reshape(-1, 2)
    assert np.array_equal(halves(lo).astype(np.float64),
                          np.stack([w & 0xF, (w >> 16) & 0xF], 1) * 2.0 ** -24)


def test_int8_codes_by_byte_permute_and_one_subtraction():
    b = np.arange(-128, 128, dtype=np.int64)
    h = (0x6400 | ((b + 128) & 0xFF)).astype(np.uint16)
    v = halves(h).astype(np.float32)
    assert np.array_equal(v, 1024.0 + (b + 128))
    d = (halves(h) - np.float16(1152.0))  # fp16 subtraction, exact here
    assert np.array_equal(d.astype(np.int64), b)
    assert np.float16(1152.0).view(np.uint16) == 0x6480


def test_fp16_products_with_subnormal_codes_are_exact_in_fp32():
    rng = np.random.default_rng(1)
    p = rng.uniform(0, 1, 5000).astype(np.float16)  # P' rounded once to fp16
    c = rng.integers(0, 16, 5000)
    code = halves(c.astype(np.uint16))              # c * 2^-24
    prod32 = p.astype(np.float32) * code.astype(np.float32)
    assert np.array_equal(prod32.astype(np.float64),
                          p.astype(np.float64) * c * 2.0 ** -24)


def test_fixed_point_query_split():
    """The query in 15-bit fixed point (the integer QK^T): with 2^e the step such that
    max|q| < 2^(e+14), each element is rounded to n = rint(q / 2^e), |n| <= 2^14, split
    into a signed high byte and an unsigned low byte, n = 256 hi + lo; the rounding is
    at most 2^-14 max|q|, and elements of magnitude at least 2^7 steps (a power of two
    between max|q|/128 and max|q|/64: their 8 significant bf16 bits then lie on the
    step grid) are exact."""
    rng = np.random.default_rng(2)
    for scale in (1e-30, 1e-3, 1.0, 7.5, 2e6):
        q = (rng.standard_normal(128) * scale).astype(np.float32)
        q = (q.view(np.uint32) & 0xFFFF0000).view(np.float32)  # bf16 values
        amax = float(np.abs(q).max())
        _, ex = np.frexp(amax)  # amax < 2^ex
        step = 2.0 ** (int(ex) - 14)
        n = np.rint(q.astype(np.float64) / step).astype(np.int64)
        assert np.abs(n).max() <= 2 ** 14
        lo, hi = n & 0xFF, n >> 8
        assert np.all((hi >= -128) & (hi <= 127)) and np.all((lo >= 0) & (lo <= 255))
        assert np.array_equal(256 * hi + lo, n)
        err = np.abs(n * step - q.astype(np.float64))
        assert err.max() <= 2.0 ** -14 * amax
        big = np.abs(q) >= 128 * step
        assert np.all(err[big] == 0)
        assert 128 * step > amax / 128 and 128 * step <= amax / 64
