"""IEEE identities the attention kernels rely on to feed codes to the fp16 tensor cores
without conversions, checked on every code value with numpy's binary16 (CPU only):

* a half whose exponent field is 0 and whose low nibble is a code c (the rest zero) is
  exactly c * 2^-24; a code in bits 4-7 gives exactly 16c * 2^-24 (V codes as
  subnormals; the kernels undo 2^24 and 2^20 once per output row);
* an int8 code b placed, offset by 128, in the low byte of a half with high byte 0x64
  is 1024 + (b + 128); subtracting 1152 gives b exactly (INT8 codes by one byte permute
  and one half subtraction);
* P' = p * scale rounded once to fp16 and multiplied by a subnormal code is exact in
  fp32 (the tensor-core product of two halves needs at most 22 significant bits);
* the one rounding that remains, P' to fp16, keeps the attention output within the 2e-3
  tolerance for V magnitudes down to ~3e-3 and not below ~1e-4 (a model of that
  arithmetic, below).
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


def _lift(scales16):
    """The kernels' power-of-two lift (log2 units) for weights whose largest V scale is
    the largest of scales16 (fp16 values): E with max * 2^E < 1, 0 <= E <= 24."""
    smax = float(np.max(scales16))
    if smax == 0:
        return 0
    return int(min(24, max(0, -1 - int(np.floor(np.log2(smax))))))


def _pv_relative_error(rng, sigma, L, int4, lifted=False):
    """Model of the kernels' PV arithmetic for one output row: p = e^(s - max s) in
    (0, 1] with logits s ~ N(0, 1); V ~ N(0, sigma^2) quantised by the oracle's
    quantisers; P' = RN16(p * scale) times the exact codes, plus sum p * min (INT4) taken
    exactly; normalised by sum p. With `lifted`, the weights are formed as the kernels do
    for small V scales (last page's lift >= 6): P' = RN16(p * 2^E * scale) with E from the
    first page (16 positions), the factor 2^E cancelling in the normalisation.
    Returns max |O_model - O_exact| / max |O_exact|."""
    from oracle import kv4_oracle as O
    v = (rng.normal(0, 1, (L, 128)) * sigma).astype(np.float32)
    s = rng.normal(0, 1, L)
    p = np.exp(s - s.max())
    if int4:
        c, sc, mn = O.quantize_int4(v)
        scale = np.repeat(sc.astype(np.float64), 32, axis=1)
        minv = (p[:, None] * np.repeat(mn.astype(np.float64), 32, axis=1)).sum(0)
    else:
        c, sc = O.quantize_int8(v)
        scale = np.broadcast_to(sc.astype(np.float64)[:, None], c.shape)
        minv = 0.0
    exact = ((p[:, None] * scale * c).sum(0) + minv) / p.sum()
    E = _lift(scale[:16]) if lifted and _lift(scale[-16:]) >= 6 else 0
    p16 = (p[:, None] * 2.0 ** E * scale).astype(np.float16).astype(np.float64)
    model = ((p16 * c).sum(0) / 2.0 ** E + minv) / p.sum()
    return np.abs(model - exact).max() / np.abs(exact).max()


def test_fp16_probability_weights_cover_the_tolerance_range():
    """P' leaves the fp16 normal range when V is small (below 2^-14 it keeps 2^-25 of
    absolute precision). Over 2000 INT4 positions and 144 INT8 ones (worst of 5 draws):
    without the lift, the modelled error stays below 1e-3 of the output scale for V
    standard deviations from 1 down to 3e-3 (INT4) and 1e-2 (INT8), and exceeds the 2e-3
    tolerance at 1e-4; with the lift the kernels apply when the V scales are small, it
    stays below 1e-3 down to 1e-6 for INT4 (where the fp16 scales are subnormal) and 1e-5
    for INT8 (at 1e-6 the INT8 scale max|x| / 127 ~ 2e-8 underflows fp16 to 0 or its
    smallest subnormal: the quantiser itself, not the weights, is then the limit)."""
    rng = np.random.default_rng(20)
    worst = lambda sigma, L, int4, lifted: max(_pv_relative_error(rng, sigma, L, int4, lifted)
                                               for _ in range(5))
    for sigma in (1.0, 0.1, 0.01, 0.003):
        assert worst(sigma, 2000, True, False) < 1e-3, sigma
    for sigma in (1.0, 0.1, 0.01):
        assert worst(sigma, 144, False, False) < 1e-3, sigma
    assert worst(1e-4, 2000, True, False) > 2e-3
    assert worst(1e-4, 144, False, False) > 2e-3
    for sigma in (1.0, 0.01, 1e-3, 1e-4, 1e-5, 1e-6):
        assert worst(sigma, 2000, True, True) < 1e-3, sigma
    for sigma in (1.0, 0.01, 1e-3, 1e-4, 1e-5):
        assert worst(sigma, 144, False, True) < 1e-3, sigma
