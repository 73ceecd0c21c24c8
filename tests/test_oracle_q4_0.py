"""Pins of the oracle's imatrix-weighted Q4_0 quantizer against what the pages and
the mathematics fix, independently of the oracle's own code.

[W] = "ik_llama.cpp 量化权重之谜：weight[j] = qw[j] * sqrtf(sigma2 + xb[j]*xb[j])的由来与原理"
      (www.dpshk.com/news/4810665), §一 (formula, make_qx_quants sums, greedy gradient),
      §三 (asymptotes of sqrt(sigma^2 + x^2)).
"""
import itertools
import math

import numpy as np
import pytest

from conftest import read_golden


def _err(x, w, l):
    """fp64 weighted error sum w (x - d l)^2 at the optimal d = sum wxl / sum wl^2."""
    x = x.astype(np.float64)
    w = w.astype(np.float64)
    l = l.astype(np.float64)
    b = np.sum(w * l * l)
    if b <= 0:
        return float(np.sum(w * x * x))
    d = np.sum(w * x * l) / b
    return float(np.sum(w * (x - d * l) ** 2))


def _blocks(n_blocks, seed, n=32, outliers=True):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((n_blocks, n)) * 0.02).astype(np.float32)
    if outliers:
        m = rng.random((n_blocks, n)) < 0.01
        x[m] = (0.2 * rng.standard_t(3, size=m.sum())).astype(np.float32)
    qw = np.exp(rng.standard_normal((n_blocks, n))).astype(np.float32)
    return x, qw


# ------------------------------------------------------------------ sigma2 and weights

def test_sigma2_equals_correctly_rounded_mean_square(orc):
    rng = np.random.default_rng(1)
    for r in range(200):
        n = int(rng.choice([32, 96, 4096, 11008]))
        x = (rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 2)).astype(np.float32)
        exact = math.fsum(float(v) * float(v) for v in x.astype(np.float64))
        assert orc.row_sigma2(x) == np.float32(exact / n)


def test_sigma2_closed_form(orc):
    x = np.array([0.5, -0.5] * 64, np.float32)
    assert orc.row_sigma2(x) == np.float32(0.25)
    x = np.zeros(32, np.float32)
    x[0] = 4.0
    assert orc.row_sigma2(x) == np.float32(0.5)


def test_weights_closed_form_and_asymptotes(orc):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(32) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(32)).astype(np.float32)
    s2 = np.float32(4e-4)
    w = orc.block_weights(x, qw, float(s2), 0)
    ref = qw.astype(np.float64) * np.sqrt(np.float64(s2) + x.astype(np.float64) ** 2)
    assert np.all(np.abs(w - ref) <= 3 * 2.0 ** -24 * ref)
    # |x| >> sigma: weight -> qw |x| ;  |x| << sigma: weight -> qw sigma   ([W] §三)
    big = np.full(32, 1000 * 0.02, np.float32)
    wb = orc.block_weights(big, qw, float(s2), 0)
    assert np.allclose(wb, qw * 20.0, rtol=1e-6)
    small = np.full(32, 1e-3 * 0.02, np.float32)
    ws = orc.block_weights(small, qw, float(s2), 0)
    assert np.allclose(ws, qw * 0.02, rtol=1e-6)
    # weight = qw variant, and qw absent means qw = 1
    assert np.array_equal(orc.block_weights(x, qw, float(s2), 1), qw)
    assert np.array_equal(orc.block_weights(x, None, float(s2), 1), np.ones(32, np.float32))
    assert np.allclose(orc.block_weights(x, None, float(s2), 0),
                       np.sqrt(np.float64(s2) + x.astype(np.float64) ** 2), rtol=3e-7)


def test_magnitude_weight_forms(orc):
    """[W] §二: the importance forms tried before imatrix existed -- x^2, |x|,
    sigma^2 + x^2, sigma + |x| (weight modes 2..5), times qw when given."""
    rng = np.random.default_rng(21)
    x = (rng.standard_normal(32) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(32)).astype(np.float32)
    s2 = np.float32(4e-4)
    xd, qd, sd = x.astype(np.float64), qw.astype(np.float64), float(s2)
    refs = {2: xd * xd, 3: np.abs(xd), 4: sd + xd * xd, 5: np.sqrt(sd) + np.abs(xd)}
    for mode, ref in refs.items():
        w = orc.block_weights(x, qw, float(s2), mode)
        assert np.all(np.abs(w - qd * ref) <= 3 * 2.0 ** -24 * qd * ref), mode
        w1 = orc.block_weights(x, None, float(s2), mode)
        assert np.all(np.abs(w1 - ref) <= 2 * 2.0 ** -24 * ref), mode
    with pytest.raises(ValueError):
        orc.quantize_q4_0_w(x.reshape(1, 32), qw, weight_mode=6)


@pytest.mark.parametrize("mode", [2, 3, 4, 5])
def test_magnitude_forms_keep_the_symmetries(orc, mode):
    """Every form is even in x and homogeneous in a power-of-two scale of x, so the
    codes survive x -> -x and x -> 2^k x, and d follows the sign and the scale."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(256)).astype(np.float32)
    a, _ = orc.quantize_q4_0_w(x, qw, weight_mode=mode)
    b, _ = orc.quantize_q4_0_w(-x, qw, weight_mode=mode)
    c, _ = orc.quantize_q4_0_w(x * np.float32(4.0), qw, weight_mode=mode)
    da, ca = orc.decode_q4_0(a, 16, 256)
    db, cb = orc.decode_q4_0(b, 16, 256)
    dc, cc = orc.decode_q4_0(c, 16, 256)
    assert np.array_equal(ca, cb) and np.array_equal(da ^ 0x8000, db)
    assert np.array_equal(ca, cc)
    assert np.array_equal(da.view(np.float16).astype(np.float32) * np.float32(4.0),
                          dc.view(np.float16).astype(np.float32))


# ------------------------------------------------------------------ exact blocks (golden)

def _expected_block_bytes(d0, n):
    h = np.float16(d0).view(np.uint16)
    qs = [(n[i] + 8) | ((n[i + 16] + 8) << 4) for i in range(16)]
    return bytes([int(h) & 0xFF, int(h) >> 8] + qs)


@pytest.mark.parametrize("mode", [1, 0])
def test_exactly_representable_blocks(orc, mode):
    for rec in read_golden("q4_0_exact_blocks.txt"):
        d0 = float(rec["d0"])
        n = [int(v) for v in rec["n"].split()]
        assert len(n) == 32
        x = (np.float32(d0) * np.array(n, np.float32)).reshape(1, 32)
        qw = np.ones(32, np.float32)
        out, flags = orc.quantize_q4_0_w(x, qw, weight_mode=mode)
        assert flags == 0
        assert bytes(out[0]) == _expected_block_bytes(d0, n)
        if mode == 1:
            w = np.ones(32, np.float32)
            d, L, _, info = orc.block_search(x[0], w)
            assert d == np.float32(d0) and info[1] == 1


# ------------------------------------------------------------------ invariances

def test_sign_flip_symmetry(orc):
    """x -> -x leaves sigma2 and the weights unchanged and negates xmax, so the codes
    are identical and only the sign bit of d flips."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(256)).astype(np.float32)
    for mode in (0, 1):
        a, _ = orc.quantize_q4_0_w(x, qw, weight_mode=mode)
        b, _ = orc.quantize_q4_0_w(-x, qw, weight_mode=mode)
        a = a.reshape(-1, 18)
        b = b.reshape(-1, 18)
        assert np.array_equal(a[:, 2:], b[:, 2:])
        assert np.array_equal(a[:, 1] ^ 0x80, b[:, 1]) and np.array_equal(a[:, 0], b[:, 0])


@pytest.mark.parametrize("k", [-3, 5])
def test_power_of_two_scaling(orc, k):
    """x -> 2^k x scales every weight (mode 0) and every sum by exact powers of two, so
    the codes are unchanged and d scales by 2^k exactly."""
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((32, 512)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(512)).astype(np.float32)
    s = np.float32(2.0 ** k)
    a, _ = orc.quantize_q4_0_w(x, qw)
    b, _ = orc.quantize_q4_0_w(x * s, qw)
    da, ca = orc.decode_q4_0(a, 32, 512)
    db, cb = orc.decode_q4_0(b, 32, 512)
    assert np.array_equal(ca, cb)
    fa = da.view(np.float16).astype(np.float32)
    fb = db.view(np.float16).astype(np.float32)
    assert np.array_equal(fa * s, fb)


def test_imatrix_scaling(orc):
    """qw -> 2^k qw scales sumlx and suml2 alike: codes and d are unchanged."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((32, 512)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(512)).astype(np.float32)
    a, _ = orc.quantize_q4_0_w(x, qw)
    b, _ = orc.quantize_q4_0_w(x, qw * np.float32(64.0))
    assert np.array_equal(a, b)


def test_rows_per_qw_selects_imatrix_row(orc):
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((12, 128)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal((3, 128))).astype(np.float32)
    stacked, _ = orc.quantize_q4_0_w(x, qw, rows_per_qw=4)
    for g in range(3):
        part, _ = orc.quantize_q4_0_w(x[4 * g:4 * g + 4], qw[g])
        assert np.array_equal(stacked[4 * g:4 * g + 4], part)


# ------------------------------------------------------------------ scale, sweep, greedy

def test_scale_is_weighted_least_squares_optimum(orc):
    """[W] §一: d = sumlx/suml2 minimises sum w (x - d l)^2 for fixed codes.  A dense sweep
    of d in fp64 finds nothing lower, and the oracle's binary32 d is that optimum up to
    the rounding of its binary32 sums."""
    x, qw = _blocks(200, 7)
    for i in range(200):
        w = orc.block_weights(x[i], qw[i], float(np.mean(x[i].astype(np.float64) ** 2)), 0)
        d, L, _, _ = orc.block_search(x[i], w)
        xd, wd, ld = x[i].astype(np.float64), w.astype(np.float64), L.astype(np.float64)
        dstar = np.sum(wd * xd * ld) / np.sum(wd * ld * ld)
        # binary32 sums of 32 same-signed terms: relative error <= (2n + 3) u, u = 2^-24
        assert abs(float(d) - dstar) <= (2 * 32 + 3) * 2.0 ** -24 * abs(dstar)
        grid = dstar * (1.0 + np.linspace(-2e-2, 2e-2, 4001))
        e = np.sum(wd[None, :] * (xd[None, :] - grid[:, None] * ld[None, :]) ** 2, axis=1)
        e0 = np.sum(wd * (xd - dstar * ld) ** 2)
        assert np.all(e >= e0 * (1 - 1e-12))
        # score <-> error identity: E(d*) = sum w x^2 - sumlx^2 / suml2
        ident = np.sum(wd * xd * xd) - np.sum(wd * xd * ld) ** 2 / np.sum(wd * ld * ld)
        assert abs(ident - e0) <= 1e-9 * np.sum(wd * xd * xd)


def _candidate_codes(xb):
    a = np.abs(xb)
    xmax = xb[int(np.argmax(a))]
    out = []
    for k in range(-9, 10):
        c = np.float32(80 + k) / np.float32(10.0)
        iscale = np.float32(-c) / xmax
        out.append(np.clip(np.rint(np.float32(iscale) * xb), -8, 7).astype(np.int8))
    return out


def test_sweep_picks_lowest_error_candidate_lowest_k_on_ties(orc):
    x, qw = _blocks(400, 8)
    for i in range(400):
        w = orc.block_weights(x[i], qw[i], 4e-4, 0)
        d, L, Ls, info = orc.block_search(x[i], w)
        cands = _candidate_codes(x[i])
        errs = [_err(x[i], w, c) for c in cands]
        assert _err(x[i], w, Ls) <= min(errs) * (1 + 1e-5) + 1e-30
        # the chosen k is the first candidate producing the chosen codes
        k = int(info[0])
        assert np.array_equal(cands[k + 9], Ls)
        first = next(j for j, c in enumerate(cands) if np.array_equal(c, Ls))
        assert first == k + 9


def test_greedy_pass_limit_is_reached_and_kept(orc):
    """The greedy refinement runs at most 5 passes (a pass with no accepted move ends it
    and is counted).  On a seeded 256x4096 tensor the counts fall off geometrically and
    the bound is reached by a few blocks, never exceeded."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((256, 4096)) * 0.02).astype(np.float32)
    qw = np.exp(rng.standard_normal(4096)).astype(np.float32)
    _, _, passes = orc.quantize_q4_0_w(x, qw, want_passes=True)
    counts = np.bincount(passes.ravel(), minlength=7)
    assert counts[0] == 0 and counts[6:].sum() == 0, counts
    assert counts[5] >= 3, counts
    assert all(counts[p] > counts[p + 1] for p in range(1, 5)), counts


def test_greedy_never_worse_and_locally_optimal(orc):
    """The greedy stage never ends above the sweep's error, and when it stops early no
    single +-1 code move lowers the fp64 error by more than the binary32 resolution of
    the score it compares.  That score sumlx^2/suml2 (= sum w x^2 - error) is built from
    running binary32 sums that absorb at most n + 5n roundings each, so its relative
    error is below (2*6n + 6n + 2) u, u = 2^-24; a move whose gain is smaller than that
    fraction of sum w x^2 may be invisible to the search."""
    x, qw = _blocks(1500, 9)
    passes = []
    u = 2.0 ** -24
    for i in range(1500):
        w = orc.block_weights(x[i], qw[i], 4e-4, 0)
        d, L, Ls, info = orc.block_search(x[i], w)
        ef, es = _err(x[i], w, L), _err(x[i], w, Ls)
        energy = float(np.sum(w.astype(np.float64) * x[i].astype(np.float64) ** 2))
        tol = (18 * 32 + 2) * u * energy
        assert ef <= es + tol
        passes.append(int(info[1]))
        if info[1] < 5:
            for j in range(32):
                for s in (-1, 1):
                    if -8 <= L[j] + s <= 7:
                        M = L.copy()
                        M[j] += s
                        assert _err(x[i], w, M) >= ef - tol
    assert 1 <= min(passes) and max(passes) <= 5


def test_brute_force_toy_blocks(orc):
    """4-element blocks: the exhaustive optimum over all 16^4 code vectors bounds the
    search from below, and the search never ends above its own candidate sweep."""
    rng = np.random.default_rng(10)
    codes = np.array(list(itertools.product(range(-8, 8), repeat=4)), np.float64)
    gaps = []
    for _ in range(300):
        x = rng.standard_normal(4).astype(np.float32)
        w = np.exp(rng.standard_normal(4)).astype(np.float32)
        d, L, Ls, info = orc.block_search(x, w)
        xd, wd = x.astype(np.float64), w.astype(np.float64)
        A = codes @ (wd * xd)
        B = (codes * codes) @ wd
        ok = B > 0
        E = np.full(len(codes), np.sum(wd * xd * xd))
        E[ok] -= A[ok] ** 2 / B[ok]
        eg = max(float(E.min()), 0.0)
        eo, es = _err(x, w, L), _err(x, w, Ls)
        assert eg <= eo * (1 + 1e-9) + 1e-12
        assert eo <= es * (1 + 1e-6) + 1e-12
        gaps.append(eo - eg)
    # the heuristic reaches the exhaustive optimum on most toy blocks
    assert np.mean(np.array(gaps) <= 1e-9) > 0.5


# ------------------------------------------------------------------ degenerate cases, flags

def test_zero_block_and_zero_weight_block(orc):
    x = np.zeros((1, 64), np.float32)
    x[0, 32:] = np.linspace(-1, 1, 32, dtype=np.float32)
    qw = np.ones(64, np.float32)
    qw[32:] = 0.0
    out, flags = orc.quantize_q4_0_w(x, qw)
    blk = out.reshape(2, 18)
    assert bytes(blk[0]) == bytes([0, 0] + [0x88] * 16)            # all-zero block
    d, L, _, info = orc.block_search(x[0, 32:], np.zeros(32, np.float32))
    assert info[2] == 1 and info[1] == 0                            # fallback, no greedy
    xmax = np.float32(-1.0)  # first element of largest |x|
    iscale0 = np.float32(np.float32(-8.0) / xmax)
    assert d == np.float32(np.float32(1.0) / iscale0)
    assert np.array_equal(L, np.clip(np.rint(iscale0 * x[0, 32:]), -8, 7).astype(np.int8))


def test_constant_block(orc):
    x = np.full(32, 0.02, np.float32)
    w = np.ones(32, np.float32)
    d, L, _, _ = orc.block_search(x, w)
    assert len(set(L.tolist())) == 1 and L[0] in (-7, -8)
    # d is a binary32 sum of 32 equal terms over an exact sum: relative error <= (32 + 2) u
    assert abs(float(d) * float(L[0]) - float(np.float32(0.02))) <= 34 * 2.0 ** -24 * 0.02


def test_flags(orc):
    x = (np.random.default_rng(11).standard_normal((2, 64)) * 0.02).astype(np.float32)
    qw = np.ones(64, np.float32)
    assert orc.quantize_q4_0_w(x, qw)[1] == 0
    xn = x.copy()
    xn[1, 5] = np.nan
    assert orc.quantize_q4_0_w(xn, qw)[1] & 1
    qn = qw.copy()
    qn[7] = -1.0
    assert orc.quantize_q4_0_w(x, qn)[1] & 2
    assert orc.quantize_q4_0_w(x * np.float32(2.0e7), qw)[1] & 4   # d beyond 65504
    with pytest.raises(ValueError):
        orc.quantize_q4_0_w(np.zeros((1, 40), np.float32))
