"""Pins of the oracle's Q4_0 x Q8_K_128 dot product (matrix-vector form).

[Q8] = "ik_llama.cpp 量化精度修复实录：用 Q8_K_128 替代 Q8_1 根治 IQ1_S_R4 / IQ1_M_R4 的 fp16 溢出"
       (www.hnwysp.cn/news/39281).  修复前的数值隐患: the consumer multiplies unsigned
       weight codes by the int8 activation codes and corrects with the block sum;
       修复方案: the sums are int16 per 32 values, not multiplied by d.

The oracle computes the plain definition, the dot product of the two dequantized
vectors with exact binary64 products.  These tests pin it against (a) a closed form
with constant codes, (b) the offset-and-block-sum route the page describes, done in
exact integer / rational arithmetic from the stored bsums, (c) numpy's binary64 matmul
of the separately pinned dequantized operands, and (d) exact symmetries.
"""
from fractions import Fraction

import numpy as np
import pytest

U53 = 2.0 ** -53


def _q4_0_bytes(d16: int, codes):
    """One 18-byte Q4_0 block: d16 little endian, qs[i] = (l_i + 8) | (l_{i+16} + 8) << 4."""
    n = [int(c) + 8 for c in codes]
    return bytes([d16 & 0xFF, d16 >> 8] + [n[i] | (n[i + 16] << 4) for i in range(16)])


def _q8_bytes(d8: float, q):
    """One 140-byte Q8_K_128 block: float d | int8 q[128] | int16 bsums[4]."""
    q = np.asarray(q, np.int64)
    bs = [int(q[32 * i:32 * i + 32].sum()) for i in range(4)]
    return (np.float32(d8).tobytes() + q.astype(np.int8).tobytes()
            + np.array(bs, np.int16).tobytes())


def _rand_q4_0(rng, rows, k):
    d = rng.integers(0x1000, 0x2C00, rows * (k // 32))           # finite positive scales
    d |= rng.integers(0, 2, d.size) << 15                          # random signs
    codes = rng.integers(-8, 8, (rows * (k // 32), 32))
    return np.frombuffer(b"".join(_q4_0_bytes(int(h), c) for h, c in zip(d, codes)),
                         np.uint8).reshape(rows, -1)


def _rand_q8(rng, tok, k):
    out = []
    for _ in range(tok * (k // 128)):
        q = rng.integers(-127, 128, 128)
        q[rng.integers(0, 128)] = 127 * rng.choice([-1, 1])
        out.append(_q8_bytes(float(np.float32(rng.uniform(1e-4, 3.0))), q))
    return np.frombuffer(b"".join(out), np.uint8).reshape(tok, -1)


def test_constant_codes_closed_form(orc):
    """Every weight code c and one scale d0: y = d0 * c * sum_g d8_g * (sum of the
    group's activation codes), exactly (all values are small dyadic rationals)."""
    k = 512
    d0 = 2.0 ** -6
    h = int(np.float16(d0).view(np.uint16))
    q_all = (np.arange(k) % 255) - 127                             # -127..127 ramp
    d8s = [0.5, 0.25, 2.0 ** -10, 3.0]
    a = np.frombuffer(b"".join(_q8_bytes(d8s[g], q_all[128 * g:128 * g + 128])
                               for g in range(k // 128)), np.uint8).reshape(1, -1)
    for c in (-8, -3, 0, 1, 7):
        w = np.frombuffer(b"".join(_q4_0_bytes(h, [c] * 32) for _ in range(k // 32)),
                          np.uint8).reshape(1, -1)
        y, s = orc.dot_q4_0_q8_k128(w, a, 1, k, 1)
        expect = sum(Fraction(d0) * c * Fraction(d8s[g]) * int(q_all[128 * g:128 * g + 128].sum())
                     for g in range(k // 128))
        assert Fraction(float(y[0, 0])) == expect
        expect_abs = sum(Fraction(d0) * abs(c) * Fraction(d8s[g]) * int(np.abs(q_all[128 * g:128 * g + 128]).sum())
                         for g in range(k // 128))
        assert Fraction(float(s[0, 0])) == expect_abs


def test_matches_offset_and_block_sum_route(orc):
    """[Q8] 修复前的数值隐患: sum_j l_j q_j = sum_j u_j q_j - 8 * bsum with unsigned
    codes u = l + 8 and the stored unscaled int16 sums.  That route, in exact integers
    per 32-value block and exact rationals for the scales, equals the oracle's value
    within its stated summation bound K * 2^-53 * sum |products|."""
    rng = np.random.default_rng(7)
    rows, tok, k = 5, 3, 384
    w = _rand_q4_0(rng, rows, k)
    a = _rand_q8(rng, tok, k)
    y, s = orc.dot_q4_0_q8_k128(w, a, rows, k, tok)
    wb = w.reshape(rows, k // 32, 18)
    ab = a.reshape(tok, k // 128, 140)
    for t in range(tok):
        for r in range(rows):
            total = Fraction(0)
            for b in range(k // 32):
                d4 = Fraction(float(wb[r, b, 0:2].copy().view(np.float16)[0]))
                qs = wb[r, b, 2:18].astype(np.int64)
                u = np.concatenate([qs & 15, qs >> 4])             # unsigned codes 0..15
                g, i = divmod(b, 4)
                d8 = Fraction(float(ab[t, g, 0:4].copy().view(np.float32)[0]))
                q = ab[t, g, 4 + 32 * i:4 + 32 * i + 32].view(np.int8).astype(np.int64)
                bsum = int(ab[t, g, 132 + 2 * i:134 + 2 * i].copy().view(np.int16)[0])
                total += d4 * d8 * (int(np.dot(u, q)) - 8 * bsum)
            assert abs(Fraction(float(y[t, r])) - total) <= Fraction(k * U53) * Fraction(float(s[t, r]))


def test_matches_library_matmul_of_dequantized_operands(orc):
    """The dequantized operands (oracle.dequant_q4_0 is pinned on its own; the Q8_K_128
    values d * q are read straight from the bytes) through numpy's binary64 matmul, a
    different summation order: agreement within 2 K 2^-53 sum |products|."""
    rng = np.random.default_rng(8)
    rows, tok, k = 48, 4, 1024
    x = (rng.standard_normal((rows, k)) * 0.02).astype(np.float32)
    act = rng.standard_normal((tok, k)).astype(np.float32)
    w, _ = orc.quantize_q4_0_w(x, np.exp(rng.standard_normal(k)).astype(np.float32))
    a, _ = orc.quantize_q8_k128(act)
    y, s = orc.dot_q4_0_q8_k128(w, a, rows, k, tok)
    wd = orc.dequant_q4_0(w, rows, k).astype(np.float64)
    d8, q8, _ = orc.decode_q8_k128(a, tok, k)
    ad = (np.repeat(d8.astype(np.float64), 128, axis=1) * q8.astype(np.float64))
    ref = ad @ wd.T
    assert np.all(np.abs(y - ref) <= 2 * k * U53 * s)
    assert np.allclose(s, np.abs(ad) @ np.abs(wd).T, rtol=4 * k * U53)
    # and it approximates the float product (4-bit weights: about 9% here)
    f = act.astype(np.float64) @ x.T.astype(np.float64)
    assert np.linalg.norm(y - f) <= 0.15 * np.linalg.norm(f)


def test_exact_symmetries(orc):
    """Flipping every weight scale's sign negates y; doubling every activation scale
    doubles it; permuting tokens permutes the output rows -- all bit for bit."""
    rng = np.random.default_rng(9)
    rows, tok, k = 7, 3, 256
    w = _rand_q4_0(rng, rows, k)
    a = _rand_q8(rng, tok, k)
    y, _ = orc.dot_q4_0_q8_k128(w, a, rows, k, tok)
    wn = w.reshape(rows, -1, 18).copy()
    wn[:, :, 1] ^= 0x80
    yn, _ = orc.dot_q4_0_q8_k128(wn.reshape(rows, -1), a, rows, k, tok)
    assert np.array_equal(yn, -y)
    a2 = a.reshape(tok, -1, 140).copy()
    d = a2[:, :, 0:4].copy().view(np.float32) * np.float32(2.0)
    a2[:, :, 0:4] = d.view(np.uint8).reshape(tok, -1, 4)
    y2, _ = orc.dot_q4_0_q8_k128(w, a2.reshape(tok, -1), rows, k, tok)
    assert np.array_equal(y2, 2.0 * y)
    perm = [2, 0, 1]
    yp, _ = orc.dot_q4_0_q8_k128(w, a[perm], rows, k, tok)
    assert np.array_equal(yp, y[perm])


def test_zero_and_empty(orc):
    rng = np.random.default_rng(10)
    w = _rand_q4_0(rng, 3, 128)
    a = np.frombuffer(_q8_bytes(0.0, np.zeros(128, np.int64)), np.uint8).reshape(1, -1)
    y, s = orc.dot_q4_0_q8_k128(w, a, 3, 128, 1)
    assert np.all(y == 0) and np.all(s == 0)
    y, s = orc.dot_q4_0_q8_k128(w, a, 0, 128, 1)
    assert y.shape == (1, 0)
    with pytest.raises(ValueError):
        orc.dot_q4_0_q8_k128(w, a, 3, 96, 1)
