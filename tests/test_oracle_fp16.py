"""Pin the oracle's binary16 encoder/decoder to numpy's IEEE conversions.

The oracle writes its own round-to-nearest-even binary16 encoder from the
format definition; numpy's float32 -> float16 cast is an independent library
implementation of the same IEEE operation.
"""
import numpy as np


def test_decoder_all_patterns(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.fp16_to_float_array(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _check_patterns(orc, u):
    f = u.view(np.float32)
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    got = orc.fp16_from_float_array(f)
    nan = np.isnan(f)
    assert np.count_nonzero(got[~nan] != ref[~nan]) == 0
    g = got[nan]
    assert np.all(((g & 0x7C00) == 0x7C00) & ((g & 0x3FF) != 0))


def test_encoder_boundary_exponents_exhaustive(orc):
    """Every positive binary32 pattern whose exponent sits at a binary16 boundary:
    flush to zero and the whole binary16 subnormal range (2^-26..2^-14), overflow (2^15..2^16),
    plus the infinities and NaNs."""
    for be in (*range(101, 114), 142, 143, 255):
        u = (np.uint32(be) << np.uint32(23)) + np.arange(1 << 23, dtype=np.uint32)
        _check_patterns(orc, u)


def test_encoder_all_ties_every_exponent(orc):
    """For every exponent, every 10-bit kept mantissa with the dropped 13 bits equal to
    just below, exactly at and just above one half (the rounding decisions)."""
    hi = np.arange(1 << 10, dtype=np.uint32) << np.uint32(13)
    low = np.array([0x0FFF, 0x1000, 0x1001, 0x0000, 0x1FFF], dtype=np.uint32)
    mant = (hi[:, None] | low[None, :]).ravel()
    for be in range(256):
        _check_patterns(orc, (np.uint32(be) << np.uint32(23)) | mant)


def test_encoder_random_sample(orc):
    rng = np.random.default_rng(11)
    _check_patterns(orc, rng.integers(0, 1 << 31, size=1 << 23, dtype=np.uint32))


def test_encoder_sign_symmetry_sample(orc):
    rng = np.random.default_rng(7)
    u = rng.integers(0, 1 << 31, size=1 << 22, dtype=np.uint32)
    f = u.view(np.float32)
    pos = orc.fp16_from_float_array(f)
    neg = orc.fp16_from_float_array(-f)
    keep = ~np.isnan(f)
    assert np.array_equal(neg[keep], pos[keep] | 0x8000)


def test_encoder_boundaries(orc):
    # largest finite, the overflow midpoint (ties to even -> inf), smallest subnormal ties
    assert orc.fp16_from_float(65504.0) == 0x7BFF
    assert orc.fp16_from_float(65519.99609375) == 0x7BFF
    assert orc.fp16_from_float(65520.0) == 0x7C00
    assert orc.fp16_from_float(2.0 ** -24) == 0x0001
    assert orc.fp16_from_float(2.0 ** -25) == 0x0000          # tie -> even (0)
    assert orc.fp16_from_float(3 * 2.0 ** -25) == 0x0002      # tie -> even (2)
    assert orc.fp16_from_float(2.0 ** -14) == 0x0400
    assert orc.fp16_from_float(-0.0) == 0x8000
