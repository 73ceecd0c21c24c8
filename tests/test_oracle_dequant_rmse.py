"""Pins of the oracle's Q4_0 dequantization and round-trip weighted-RMSE reduction.

[SVD] = "量化方法论实证：为什么 LQER/L²QER 难以改进 ik_llama.cpp 的 k-quants 与 i-quants"
        (www.0539edu.com/news/4792009), §3.2: quantize-stats reports
        rmse = sqrt(total_error / num_samples) and maxerr.
"""
import numpy as np


def _pack(d, codes):
    """Block bytes from the layout reading: binary16 d (LE), byte 2+i = lo code i | hi code i+16."""
    h = int(np.float16(d).view(np.uint16))
    qs = [(codes[i] + 8) | ((codes[i + 16] + 8) << 4) for i in range(16)]
    return np.array([h & 0xFF, h >> 8] + qs, np.uint8)


def test_dequant_layout(orc):
    codes = list(range(-8, 8)) + list(range(7, -9, -1))
    blk = _pack(0.5, codes)
    y = orc.dequant_q4_0(blk.reshape(1, 18), 1, 32)
    assert y[0].tolist() == [0.5 * c for c in codes]


def test_dequant_is_exact_product(orc):
    rng = np.random.default_rng(14)
    h = rng.integers(0, 0x7C00, size=500).astype(np.uint16)        # every finite positive d16
    h[::2] |= 0x8000
    codes = rng.integers(-8, 8, size=(500, 32))
    blocks = np.stack([_pack(np.uint16(hh).view(np.float16), c) for hh, c in zip(h, codes)])
    y = orc.dequant_q4_0(blocks, 500, 32)
    d = h.view(np.float16).astype(np.float64)
    assert np.array_equal(y.astype(np.float64), d[:, None] * codes)


def test_roundtrip_consistency(orc):
    rng = np.random.default_rng(15)
    x = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(256)).astype(np.float32)
    blocks, _ = orc.quantize_q4_0_w(x, qw)
    y = orc.dequant_q4_0(blocks, 16, 256)
    d16, codes = orc.decode_q4_0(blocks, 16, 256)
    assert np.array_equal(y, np.repeat(d16.view(np.float16).astype(np.float32), 32, axis=1) * codes)
    acc = orc.weighted_rmse(x, blocks, qw)
    e = (x - y).astype(np.float64)                                 # binary32 difference
    assert abs(acc[0] - np.sum(qw.astype(np.float64) * e * e)) <= 1e-12 * acc[0]
    assert abs(acc[1] - 16 * np.sum(qw.astype(np.float64))) <= 1e-12 * acc[1]
    assert abs(acc[2] - np.sum(e * e)) <= 1e-12 * acc[2]
    assert acc[3] == np.max(np.abs(e))


def test_rmse_closed_form(orc):
    """Values exactly a quarter off the grid d = 1: every error is +-0.25, so
    sum e^2 = n/16, sum qw e^2 = sum qw / 16 and maxerr = 0.25."""
    rng = np.random.default_rng(16)
    codes = rng.integers(-7, 7, size=(4, 64))
    blocks = np.stack([np.concatenate([_pack(1.0, r[:32]), _pack(1.0, r[32:])]) for r in codes])
    delta = np.where(rng.random((4, 64)) < 0.5, -0.25, 0.25)
    x = (codes + delta).astype(np.float32)
    qw = np.exp(rng.standard_normal(64)).astype(np.float32)
    acc = orc.weighted_rmse(x, blocks, qw)
    sq = float(np.sum(qw.astype(np.float64)))
    assert acc[2] == 256 / 16 and acc[3] == 0.25
    assert abs(acc[0] - 4 * sq / 16) <= 1e-14 * acc[0] and abs(acc[1] - 4 * sq) <= 1e-14 * acc[1]


def test_rmse_accumulates_and_uses_stacked_imatrix(orc):
    rng = np.random.default_rng(17)
    x = (rng.standard_normal((6, 64)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal((2, 64))).astype(np.float32)
    blocks, _ = orc.quantize_q4_0_w(x, qw, rows_per_qw=3)
    whole = orc.weighted_rmse(x, blocks, qw, rows_per_qw=3)
    acc = np.zeros(4)
    orc.weighted_rmse(x[:3], blocks[:3], qw[0], acc=acc)
    orc.weighted_rmse(x[3:], blocks[3:], qw[1], acc=acc)
    assert np.allclose(whole, acc, rtol=1e-13, atol=0)
