"""Pins of the oracle's Q8_K_128 activation quantizer.

[Q8] = "ik_llama.cpp 量化精度修复实录：用 Q8_K_128 替代 Q8_1 根治 IQ1_S_R4 / IQ1_M_R4 的 fp16 溢出"
       (www.hnwysp.cn/news/39281).  修复前的数值隐患: Q8_1 keeps d = x_max/127 and
       s = d * sum(q) in fp16, and s can overflow although d fits; 修复方案: Q8_K_128 keeps a
       binary32 d per 128 values and int16 sums per 32 values that are not multiplied by d.
"""
from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden


def _rne_int(fr: Fraction) -> int:
    """Round a rational to the nearest integer, ties to even (exact)."""
    fl = fr.numerator // fr.denominator
    rem = fr - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl


def _golden_case(name):
    recs = {r["case"]: r for r in read_golden("q8_k128_cases.txt")}
    assert name in recs
    j = np.arange(128)
    if name == "ramp":
        return (j - 64).astype(np.float32)
    if name == "zeros":
        return np.zeros(128, np.float32)
    x = np.where(j % 2 == 0, 0.5, -0.5).astype(np.float32)
    x[3] = 1.5e5
    return x


def test_page_constants_match_layout(orc):
    c = {r["name"]: int(r["value"]) for r in read_golden("page_constants.txt")}
    # 140 bytes = binary32 scale + 128 int8 codes + (128/32) int16 sums
    assert orc.Q8_K128_BYTES == c["q8_k128_scale_bits"] // 8 + c["q8_k128_block_values"] + \
        (c["q8_k128_block_values"] // c["q8_k128_sum_group"]) * c["q8_k128_sum_bits"] // 8
    assert orc.lib().oracle_q8_k128_block_bytes() == orc.Q8_K128_BYTES
    # 18 bytes = binary16 scale + 32 four-bit codes; nmax 8 -> codes in [-8, 7]
    assert orc.lib().oracle_q4_0_block_bytes() == 2 + 32 * 4 // 8
    assert orc.fp16_to_float(0x7BFF) == c["fp16_max"]


def test_ramp_closed_form(orc):
    x = _golden_case("ramp")
    out, flags = orc.quantize_q8_k128(x.reshape(1, 128))
    d, qs, bs = orc.decode_q8_k128(out, 1, 128)
    assert flags == 0
    assert d[0, 0] == np.float32(64.0) / np.float32(127.0)
    expect = [_rne_int(Fraction(int(v)) * Fraction(127, 64)) for v in x]
    assert qs[0].tolist() == expect
    assert bs[0, 0].tolist() == [sum(expect[32 * i:32 * i + 32]) for i in range(4)]


def test_zero_block(orc):
    out, flags = orc.quantize_q8_k128(_golden_case("zeros").reshape(1, 128))
    assert flags == 0 and not out.any()


def test_spike_beyond_fp16_stays_finite(orc):
    x = _golden_case("spike_beyond_fp16")
    out, flags = orc.quantize_q8_k128(x.reshape(1, 128))
    d, qs, bs = orc.decode_q8_k128(out, 1, 128)
    assert flags == 0
    assert d[0, 0] == np.float32(1.5e5) / np.float32(127.0) and np.isfinite(d[0, 0])
    assert qs[0, 3] == 127 and np.count_nonzero(qs[0]) == 1
    assert bs[0, 0].tolist() == [127, 0, 0, 0]


def test_q8_1_contrast_overflows_where_q8_k128_does_not(orc):
    """[Q8] 修复前的数值隐患: a block whose x_max fits fp16 can still overflow the fp16 sum
    s = d * sum(q); the Q8_K_128 sums are integers and its scale is binary32."""
    x = np.full(128, 60000.0, np.float32)
    assert np.isfinite(np.float16(x.max()))
    d_q81 = np.float16(np.float32(60000.0) / np.float32(127.0))
    assert np.isfinite(d_q81)
    with np.errstate(over="ignore"):
        s_q81 = np.float16(np.float32(d_q81) * np.float32(32 * 127))
    assert np.isinf(s_q81)
    out, flags = orc.quantize_q8_k128(x.reshape(1, 128))
    d, qs, bs = orc.decode_q8_k128(out, 1, 128)
    assert flags == 0 and np.isfinite(d).all()
    assert bs[0, 0].tolist() == [32 * 127] * 4


def test_invariants_on_activation_like_data(orc):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((64, 1024)).astype(np.float32)
    m = rng.random(x.shape) < 1e-3
    x[m] = (rng.uniform(6e4, 2e5, m.sum()) * rng.choice([-1, 1], m.sum())).astype(np.float32)
    out, flags = orc.quantize_q8_k128(x)
    assert flags == 0
    d, qs, bs = orc.decode_q8_k128(out, 64, 1024)
    xb = x.reshape(64, 8, 128)
    qb = qs.reshape(64, 8, 128).astype(np.int64)
    amax = np.abs(xb).max(axis=2)
    assert np.array_equal(d, amax / np.float32(127.0))                # IEEE binary32 division
    assert np.abs(qb).max() <= 127
    assert np.all(np.abs(qb).max(axis=2) == 127)                      # the extreme maps to +-127
    assert np.array_equal(bs.astype(np.int64), qb.reshape(64, 8, 4, 32).sum(axis=3))
    err = np.abs(xb.astype(np.float64) - d[:, :, None].astype(np.float64) * qb)
    assert np.all(err <= 0.5001 * d[:, :, None])


def test_sign_symmetry_and_power_of_two_scaling(orc):
    rng = np.random.default_rng(13)
    x = rng.standard_normal((8, 512)).astype(np.float32)
    a, _ = orc.quantize_q8_k128(x)
    b, _ = orc.quantize_q8_k128(-x)
    c, _ = orc.quantize_q8_k128(x * np.float32(2.0 ** 7))
    da, qa, ba = orc.decode_q8_k128(a, 8, 512)
    db, qb, bb = orc.decode_q8_k128(b, 8, 512)
    dc, qc, bc = orc.decode_q8_k128(c, 8, 512)
    assert np.array_equal(da, db) and np.array_equal(qa, -qb) and np.array_equal(ba, -bb)
    assert np.array_equal(qa, qc) and np.array_equal(da * np.float32(128.0), dc)


def test_nonfinite_flag_and_shape_error(orc):
    x = np.zeros((1, 256), np.float32)
    x[0, 200] = np.inf
    assert orc.quantize_q8_k128(x)[1] & 1
    with pytest.raises(ValueError):
        orc.quantize_q8_k128(np.zeros((1, 96), np.float32))


# ------------------------------------------------------------------ Q8_1 (the overflowing format)

def test_q8_1_invariants_and_overflow_count(orc):
    """[Q8] 修复前的数值隐患: Q8_1 keeps d = x_max/127 and s = d*sum(q) as fp16 per 32
    values; s overflows on blocks whose d still fits."""
    rng = np.random.default_rng(31)
    x = rng.standard_normal((16, 1024)).astype(np.float32)
    m = rng.random(x.shape) < 2e-3
    x[m] = (rng.uniform(6e4, 2e5, m.sum()) * rng.choice([-1, 1], m.sum())).astype(np.float32)
    out, n_over = orc.quantize_q8_1(x)
    d16, s16, qs = orc.decode_q8_1(out, 16, 1024)
    xb = x.reshape(16, 32, 32)
    amax = np.abs(xb).max(axis=2)
    d = amax / np.float32(127.0)
    assert np.array_equal(d16, d.astype(np.float16).view(np.uint16))
    q = qs.reshape(16, 32, 32).astype(np.int64)
    assert np.abs(q).max() <= 127 and np.all(np.abs(q).max(axis=2) == 127)
    with np.errstate(over="ignore"):
        s_ref = (d * q.sum(axis=2).astype(np.float32)).astype(np.float16)
    assert np.array_equal(s16, s_ref.view(np.uint16))
    assert n_over == int(np.count_nonzero(np.isinf(s_ref) & np.isfinite(d.astype(np.float16))))
    assert n_over > 0
    err = np.abs(xb.astype(np.float64) - d[:, :, None].astype(np.float64) * q)
    assert np.all(err <= 0.5001 * d[:, :, None])
    # the same values quantized to Q8_K_128 stay finite
    k_out, flags = orc.quantize_q8_k128(x)
    kd, _, kbs = orc.decode_q8_k128(k_out, 16, 1024)
    assert flags == 0 and np.isfinite(kd).all()
