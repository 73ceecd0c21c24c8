"""Pins of the oracle's weighted Q5_0 / Q6_0 / Q8_0 quantizers: the same search as
Q4_0 with nmax = 16, 32, 128 and codes in [-nmax, nmax-1].

[W] = "ik_llama.cpp 量化权重之谜：weight[j] = qw[j] * sqrtf(sigma2 + xb[j]*xb[j])的由来与原理"
      (www.dpshk.com/news/4810665), §一: the same weighting appears in
      quantize_row_q5_0_impl, quantize_row_q6_0_impl, ... (and make_qx_quants takes nmax).
Byte layouts (reading; the pages do not print them), biased code n = l + nmax:
  Q5_0 22 B: d16 | qh u32 (bit j = n_j >> 4 & 1) | qs[16] (low nibbles, j and j+16 paired)
  Q6_0 26 B: d16 | qh u64 (bits 2j, 2j+1 = n_j >> 4) | qs[16]
  Q8_0 34 B: d16 | int8 l[32]
"""
import itertools

import numpy as np
import pytest

BITS = (5, 6, 8)


def _pack(bits, d, codes, orc):
    nmax = orc.NMAX[bits]
    h = int(np.float16(d).view(np.uint16))
    head = [h & 0xFF, h >> 8]
    if bits == 8:
        return bytes(head + [c & 0xFF for c in codes])
    n = [c + nmax for c in codes]
    if bits == 4:
        return bytes(head + [n[i] | (n[i + 16] << 4) for i in range(16)])
    if bits == 5:
        qh = sum(((v >> 4) & 1) << j for j, v in enumerate(n))
        hb = qh.to_bytes(4, "little")
    else:
        qh = sum(((v >> 4) & 3) << (2 * j) for j, v in enumerate(n))
        hb = qh.to_bytes(8, "little")
    qs = [(n[i] & 15) | ((n[i + 16] & 15) << 4) for i in range(16)]
    return bytes(head) + hb + bytes(qs)


def _err(x, w, l):
    x, w, l = (a.astype(np.float64) for a in (x, w, l))
    b = np.sum(w * l * l)
    d = np.sum(w * x * l) / b
    return float(np.sum(w * (x - d * l) ** 2))


def test_block_sizes(orc):
    assert [orc.qx_block_bytes(b) for b in (4, 5, 6, 8)] == [18, 22, 26, 34]


@pytest.mark.parametrize("bits", BITS)
def test_exact_blocks_and_layout(orc, bits):
    """x = d0 * n with integer codes n spanning [-nmax, nmax-1], the extreme -nmax
    unique: the search returns codes n and d0 exactly (weights 1), and the bytes follow
    the layout reading."""
    nmax = orc.NMAX[bits]
    rng = np.random.default_rng(bits)
    for d0 in (2.0 ** -7, -0.25, 3.0):
        codes = rng.integers(-nmax + 1, nmax, 32)
        codes[5] = -nmax
        codes[9] = 1                        # no common factor
        x = (np.float32(d0) * codes.astype(np.float32)).reshape(1, 32)
        out, flags = orc.quantize_qx_0_w(bits, x, np.ones(32, np.float32), weight_mode=1)
        assert flags == 0
        assert bytes(out[0]) == _pack(bits, d0, codes.tolist(), orc)
        y = orc.dequant_qx_0(bits, out, 1, 32)
        assert np.array_equal(y, x)


@pytest.mark.parametrize("bits", BITS)
def test_dequant_is_the_exact_product(orc, bits):
    nmax = orc.NMAX[bits]
    rng = np.random.default_rng(10 + bits)
    blocks, expect = [], []
    for _ in range(200):
        h = np.uint16(rng.integers(0, 0x7C00)) | np.uint16(rng.integers(0, 2) << 15)
        d = h.view(np.float16)
        codes = rng.integers(-nmax, nmax, 32)
        blocks.append(np.frombuffer(_pack(bits, d, codes.tolist(), orc), np.uint8))
        expect.append(np.float64(d) * codes)
    y = orc.dequant_qx_0(bits, np.stack(blocks), 200, 32)
    assert np.array_equal(y.astype(np.float64), np.stack(expect))


@pytest.mark.parametrize("bits", BITS)
def test_symmetries(orc, bits):
    rng = np.random.default_rng(20 + bits)
    x = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(256)).astype(np.float32)
    a, _ = orc.quantize_qx_0_w(bits, x, qw)
    b, _ = orc.quantize_qx_0_w(bits, -x, qw)
    c, _ = orc.quantize_qx_0_w(bits, x * np.float32(8.0), qw)
    ya, yb, yc = (orc.dequant_qx_0(bits, t, 16, 256) for t in (a, b, c))
    assert np.array_equal(ya, -yb)
    assert np.array_equal(ya * np.float32(8.0), yc)


@pytest.mark.parametrize("bits", BITS)
def test_search_never_worse_than_candidates_and_locally_optimal(orc, bits):
    """As for Q4_0: the result is at least as good as every candidate's rounding and no
    single +-1 move improves it beyond the binary32 resolution of the score."""
    nmax = orc.NMAX[bits]
    rng = np.random.default_rng(30 + bits)
    u = 2.0 ** -24
    for _ in range(300):
        x = (rng.standard_normal(32) * 0.02).astype(np.float32)
        w = np.exp(rng.standard_normal(32)).astype(np.float32)
        d, L, Ls, info = orc.qx_block_search(x, w, nmax)
        L = L.astype(np.int64)                      # int8 codes would wrap at +-128
        energy = float(np.sum(w.astype(np.float64) * x.astype(np.float64) ** 2))
        tol = (18 * 32 + 2) * u * energy
        ef = _err(x, w, L)
        xmax = x[int(np.argmax(np.abs(x)))]
        for k in range(-9, 10):
            c = np.float32(nmax * (80 + k)) / np.float32(80.0)
            iscale = np.float32(-c) / xmax
            cand = np.clip(np.rint(np.float32(iscale) * x), -nmax, nmax - 1)
            assert ef <= _err(x, w, cand) + tol
        if info[1] < 5:
            for j in range(32):
                for s in (-1, 1):
                    if -nmax <= L[j] + s <= nmax - 1:
                        M = L.copy()
                        M[j] += s
                        assert _err(x, w, M) >= ef - tol


def test_brute_force_three_values_q5(orc):
    """3-value toy blocks with nmax = 16: every one of the 32^3 code vectors bounds
    the search from below."""
    rng = np.random.default_rng(40)
    codes = np.array(list(itertools.product(range(-16, 16), repeat=3)), np.float64)
    hits = 0
    for _ in range(200):
        x = rng.standard_normal(3).astype(np.float32)
        w = np.exp(rng.standard_normal(3)).astype(np.float32)
        d, L, Ls, info = orc.qx_block_search(x, w, 16)
        xd, wd = x.astype(np.float64), w.astype(np.float64)
        A = codes @ (wd * xd)
        B = (codes * codes) @ wd
        ok = B > 0
        E = np.full(len(codes), np.sum(wd * xd * xd))
        E[ok] -= A[ok] ** 2 / B[ok]
        eg = max(float(E.min()), 0.0)
        eo = _err(x, w, L)
        assert eg <= eo * (1 + 1e-9) + 1e-12
        hits += eo - eg <= 1e-9 * max(eo, 1e-30)
    assert hits > 100


def test_more_bits_less_error(orc):
    rng = np.random.default_rng(50)
    x = (rng.standard_normal((32, 512)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(512)).astype(np.float32)
    errs = []
    for bits in (4, 5, 6, 8):
        out, _ = orc.quantize_qx_0_w(bits, x, qw)
        y = orc.dequant_qx_0(bits, out, 32, 512)
        errs.append(float(np.sum(qw * (x - y).astype(np.float64) ** 2)))
    assert errs[0] > errs[1] > errs[2] > errs[3]


def test_weighted_rmse_closed_form(orc):
    """Hand-built blocks of every format with x = y + delta, delta exactly representable:
    the accumulator equals the exact sums of qw e^2, qw, e^2 and max |e|; bits = 4 is the
    separately pinned Q4_0 reduction."""
    from fractions import Fraction
    rng = np.random.default_rng(60)
    for bits in (4, 5, 6, 8):
        nmax = orc.NMAX[bits]
        d0 = 2.0 ** -5
        codes = rng.integers(-nmax, nmax, (3, 32))
        blk = np.stack([np.frombuffer(_pack(bits, d0, c.tolist(), orc), np.uint8) for c in codes])
        delta = (rng.integers(-64, 65, (3, 32)) * 2.0 ** -12).astype(np.float32)
        x = (codes * np.float32(d0)).astype(np.float32) + delta     # exact in binary32
        qw = (rng.integers(1, 9, 32) * 0.25).astype(np.float32)
        acc = orc.weighted_rmse_qx(bits, x.reshape(1, 96), blk.reshape(1, -1), np.tile(qw, 3))
        e = [Fraction(float(v)) for v in delta.reshape(-1)]
        q = [Fraction(float(v)) for v in np.tile(qw, 3)]
        assert Fraction(acc[0]) == sum(qi * ei * ei for qi, ei in zip(q, e))
        assert Fraction(acc[1]) == sum(q)
        assert Fraction(acc[2]) == sum(ei * ei for ei in e)
        assert acc[3] == float(np.abs(delta).max())
        if bits == 4:
            ref = orc.weighted_rmse(x.reshape(1, 96), blk.reshape(1, -1), np.tile(qw, 3))
            assert np.array_equal(acc, ref)


def test_weighted_rmse_stacked_imatrix(orc):
    """One imatrix row per rows_per_qw rows: with constant rows 1, 2, 3 the weight sum is
    the closed form n * sum_r qw[r // rows_per_qw], for every format."""
    rng = np.random.default_rng(61)
    rows, n = 6, 64
    x = rng.standard_normal((rows, n)).astype(np.float32)
    for bits in (4, 5, 6, 8):
        for rpq, nq in ((1, 6), (2, 3), (4, 2), (0, 1)):
            qw = np.stack([np.full(n, float(i + 1), np.float32) for i in range(nq)])
            out, _ = orc.quantize_qx_0_w(bits, x, qw if rpq else qw[0], rpq)
            acc = orc.weighted_rmse_qx(bits, x, out, qw if rpq else qw[0], rpq)
            expect = n * sum((r // rpq if rpq else 0) + 1 for r in range(rows))
            assert acc[1] == expect, (bits, rpq, acc[1], expect)
            e = (x - orc.dequant_qx_0(bits, out, rows, n)).astype(np.float64)
            qfull = np.array([[(r // rpq if rpq else 0) + 1.0] * n for r in range(rows)])
            assert abs(acc[0] - float(np.sum(qfull * e * e))) <= 1e-12 * acc[0]


@pytest.mark.parametrize("bits", (4, 5, 6, 8))
def test_stacked_imatrix_selects_row(orc, bits):
    """One imatrix row per rows_per_qw rows (the experts' stacked imatrix): the stacked call
    equals quantizing each group of rows with its own imatrix row, for every format, and
    the rows do matter (one row for all gives other blocks)."""
    rng = np.random.default_rng(70 + bits)
    x = (rng.standard_normal((12, 128)) * 0.02).astype(np.float32)
    qw = np.exp(2.0 * rng.standard_normal((4, 128))).astype(np.float32)
    stacked, _ = orc.quantize_qx_0_w(bits, x, qw, rows_per_qw=3)
    for g in range(4):
        part, _ = orc.quantize_qx_0_w(bits, x[3 * g:3 * g + 3], qw[g])
        assert np.array_equal(stacked[3 * g:3 * g + 3], part), g
    one, _ = orc.quantize_qx_0_w(bits, x, qw[0])
    assert not np.array_equal(one[3:], stacked[3:])


@pytest.mark.parametrize("bits", (4, 5, 8))
def test_fudge_factor_special_cases(orc, bits):
    """[W] §四's fudge factor, read as scaling the sigma2 term of the importance: fudge = 1
    is the plain quantizer; fudge = 0 removes sigma2, so qw*sqrt(sigma2 + x^2) becomes
    qw*|x| (sqrt of the rounded x^2 rounds back to |x| for normal x), qw*(sigma2 + x^2)
    becomes qw*x^2 and qw*(sqrt(sigma2) + |x|) becomes qw*|x| -- bit for bit; and a
    power-of-two fudge scales sigma2 exactly, so it equals quantizing with that sigma2."""
    rng = np.random.default_rng(70 + bits)
    x = (rng.standard_normal((12, 256)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(256)).astype(np.float32)
    plain, _ = orc.quantize_qx_0_w(bits, x, qw, 0, 0)
    assert np.array_equal(orc.quantize_qx_0_w(bits, x, qw, 0, 0, fudge=1.0)[0], plain)
    m3, _ = orc.quantize_qx_0_w(bits, x, qw, 0, 3)
    m2, _ = orc.quantize_qx_0_w(bits, x, qw, 0, 2)
    assert np.array_equal(orc.quantize_qx_0_w(bits, x, qw, 0, 0, fudge=0.0)[0], m3)
    assert np.array_equal(orc.quantize_qx_0_w(bits, x, qw, 0, 4, fudge=0.0)[0], m2)
    assert np.array_equal(orc.quantize_qx_0_w(bits, x, qw, 0, 5, fudge=0.0)[0], m3)
    # modes without sigma2 ignore it
    for mode in (1, 2, 3):
        assert np.array_equal(orc.quantize_qx_0_w(bits, x, qw, 0, mode, fudge=7.0)[0],
                              orc.quantize_qx_0_w(bits, x, qw, 0, mode)[0])
    # fudge 4 on a row equals the block search with sigma2 * 4, through the block functions
    f4, _ = orc.quantize_qx_0_w(bits, x[:1], qw, 0, 0, fudge=4.0)
    s2 = np.float32(4.0) * np.float32(orc.row_sigma2(x[0]))
    for b in range(0, 256, 32):
        w = orc.block_weights(x[0, b:b + 32], qw[b:b + 32], float(s2), 0)
        d, L, _, _ = orc.qx_block_search(x[0, b:b + 32], w, orc.NMAX[bits])
        blk = _pack(bits, np.float32(d), L.astype(np.int64).tolist(), orc)
        assert bytes(f4[0, (b // 32) * len(blk):(b // 32 + 1) * len(blk)]) == blk
