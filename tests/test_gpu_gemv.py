"""Q4_0 x Q8_K_128 matrix-vector product on the GPU (through the C ABI) against the
oracle's binary64 dot product of the dequantized vectors.

Bound (derived, not tuned): every block term d8 * d4 * isum is exact in binary64 on the
GPU, so its result differs from the exact dot product only by binary64 summation
(at most K/32 + 16 roundings on any path) and the final rounding to binary32; the oracle
sums K exact products in binary64.  Hence
    |y_gpu - y_oracle| <= 2^-24 |y_oracle| + 2^-149 + (K + K/32 + 16) 2^-53 sum|products|.
Nearly every output is also the correctly rounded binary32 of the oracle's value.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def iqq():
    import post_weight_quantization_rowwise_b200 as m
    return m


@pytest.fixture(scope="module")
def synth():
    from post_weight_quantization_rowwise_b200 import synth as s
    return s


def _random_q4_0(rng, rows, k):
    """Random Q4_0 bytes: finite binary16 scales of both signs over many binades, random
    nibbles."""
    nb = k // 32
    d16 = rng.integers(0x0400, 0x5800, (rows, nb)).astype(np.uint16)
    d16 |= (rng.integers(0, 2, (rows, nb)) << 15).astype(np.uint16)
    b = np.empty((rows, nb, 18), np.uint8)
    b[:, :, 0:2] = d16.view(np.uint8).reshape(rows, nb, 2)
    b[:, :, 2:] = rng.integers(0, 256, (rows, nb, 16), dtype=np.uint8)
    return b.reshape(rows, nb * 18)


def _activations(synth, tok, k, seed):
    a = synth.activations(tok, k, seed=seed).numpy()
    blocks, _ = oracle.quantize_q8_k128(a)
    return blocks


def _check(y, yo, s, k):
    y = y.astype(np.float64)
    bound = 2.0 ** -24 * np.abs(yo) + 2.0 ** -149 + (k + k / 32 + 16) * 2.0 ** -53 * s
    bad = np.abs(y - yo) > bound
    assert not bad.any(), (int(bad.sum()), float(np.max(np.abs(y - yo) - bound)))
    exact = float(np.mean(y == yo.astype(np.float32).astype(np.float64)))
    assert exact >= 0.99, exact
    return exact


def _gpu(iqq, w, a, n_out, k, n_tok):
    wd = torch.from_numpy(np.ascontiguousarray(w)).cuda()
    ad = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = iqq.gemv_q4_0_q8_k128(wd, ad, n_out, k, n_tok, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    return y.cpu().numpy()


@pytest.mark.parametrize("n_out,k,n_tok", [
    (64, 4096, 1), (37, 11008, 3), (5, 128, 1), (9, 384, 8), (130, 4224, 5),
    (1, 256, 9), (17, 14336, 2), (3, 65536, 1), (11, 65408, 2), (200, 1024, 16),
    (7, 4096, 4), (301, 512, 7), (1000, 53248, 1), (333, 40064, 1)])
def test_gemv_random_blocks(iqq, synth, n_out, k, n_tok):
    """Chunk tails (odd row counts, rows of 8 mod 16 bytes), one and several token tiles,
    every token-tile width, K up to the maximum."""
    rng = np.random.default_rng(n_out * 7 + k + n_tok)
    w = _random_q4_0(rng, n_out, k)
    a = _activations(synth, n_tok, k, seed=k + n_tok)
    y = _gpu(iqq, w, a, n_out, k, n_tok)
    yo, s = oracle.dot_q4_0_q8_k128(w, a, n_out, k, n_tok)
    _check(y, yo, s, k)


@pytest.mark.parametrize("n_out,k", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_gemv_layer_shapes_full_size(iqq, synth, n_out, k):
    """The Llama-2-7B-shaped matrices at full size, one token (decode), every output."""
    rng = np.random.default_rng(n_out + k)
    w = _random_q4_0(rng, n_out, k)
    a = _activations(synth, 1, k, seed=5)
    y = _gpu(iqq, w, a, n_out, k, 1)
    yo, s = oracle.dot_q4_0_q8_k128(w, a, n_out, k, 1)
    _check(y, yo, s, k)


def test_gemv_on_quantized_weights(iqq, synth):
    """End to end on the oracle's own Q4_0 and Q8_K_128 blocks of synthetic weights and
    spiky activations (values beyond the binary16 range)."""
    x = synth.weight_matrix(96, 4096, seed=11).numpy()
    qw = synth.imatrix(4096, seed=12).numpy()
    w, _ = oracle.quantize_q4_0_w(x, qw)
    act = synth.activations(6, 4096, seed=13, spike_frac=1e-3).numpy()
    a, _ = oracle.quantize_q8_k128(act)
    y = _gpu(iqq, w, a, 96, 4096, 6)
    yo, s = oracle.dot_q4_0_q8_k128(w, a, 96, 4096, 6)
    _check(y, yo, s, 4096)


def test_gemv_reproducible_and_empty(iqq, synth):
    rng = np.random.default_rng(3)
    w = torch.from_numpy(_random_q4_0(rng, 50, 2048)).cuda()
    a = torch.from_numpy(_activations(synth, 3, 2048, seed=4)).cuda()
    y1 = iqq.gemv_q4_0_q8_k128(w, a, 50, 2048, 3)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y2 = iqq.gemv_q4_0_q8_k128(w, a, 50, 2048, 3, stream=s)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y0 = torch.full((3, 50), 7.0, device="cuda")
    iqq.iqq_gemv_q4_0_q8_k128(w, a, y0, 0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y0).item() == 0


def test_gemv_batch_matches_single_calls(iqq, synth):
    """A list of problems of different shapes, token counts and widths (incl. empty and
    k == 0 ones, and more than one launch's worth): every output equals the single call's
    bit for bit and lies within the bound of the oracle's value."""
    rng = np.random.default_rng(40)
    shapes = [(64, 4096, 1), (37, 11008, 3), (5, 128, 1), (130, 4224, 5), (1, 256, 9), (0, 512, 2),
              (7, 0, 2), (300, 1024, 1)] + [(3 + i % 5, 128 * (1 + i % 4), 1 + i % 3) for i in range(66)]
    items, singles, refs = [], [], []
    for i, (n_out, k, n_tok) in enumerate(shapes):
        w = torch.from_numpy(_random_q4_0(rng, max(n_out, 1), max(k, 128))).cuda()
        a = torch.from_numpy(_activations(synth, n_tok, max(k, 128), seed=i)).cuda()
        y = torch.full((n_tok, n_out), float("nan"), device="cuda")
        items.append((w, a, y, k))
        singles.append(iqq.gemv_q4_0_q8_k128(w, a, n_out, k, n_tok) if n_out and n_tok else None)
        refs.append((w, a, n_out, k, n_tok))
    probs = iqq.gemv_problems(items)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    iqq.iqq_gemv_q4_0_q8_k128_batch(probs, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    for (w, a, y, k), single, (_, _, n_out, _, n_tok) in zip(items, singles, refs):
        if single is None:
            continue
        assert torch.equal(y, single)
        if k == 0:
            assert torch.count_nonzero(y).item() == 0
            continue
        yo, s = oracle.dot_q4_0_q8_k128(w.cpu().numpy(), a.cpu().numpy(), n_out, k, n_tok)
        _check(y.cpu().numpy(), yo, s, k)


def test_gemv_batch_ctas_spanning_problems(iqq, synth):
    """64 small problems (1-5 rows, k up to 768, 1-9 tokens): the launch has a dozen CTAs,
    each taking rows of several problems in turn, and the second token tile skips the
    problems with at most 8 tokens inside a CTA.  Every output equals its single call bit
    for bit and lies within the bound of the oracle's value."""
    rng = np.random.default_rng(41)
    items, singles, refs = [], [], []
    for i in range(64):
        n_out, k, n_tok = 1 + (i * 7) % 5, 128 * (1 + (i * 3) % 6), 1 + (i * 5) % 9
        w = torch.from_numpy(_random_q4_0(rng, n_out, k)).cuda()
        a = torch.from_numpy(_activations(synth, n_tok, k, seed=100 + i)).cuda()
        y = torch.full((n_tok, n_out), float("nan"), device="cuda")
        items.append((w, a, y, k))
        singles.append(iqq.gemv_q4_0_q8_k128(w, a, n_out, k, n_tok))
        refs.append((n_out, k, n_tok))
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    iqq.iqq_gemv_q4_0_q8_k128_batch(iqq.gemv_problems(items), flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    for (w, a, y, k), single, (n_out, _, n_tok) in zip(items, singles, refs):
        assert torch.equal(y, single)
        yo, s = oracle.dot_q4_0_q8_k128(w.cpu().numpy(), a.cpu().numpy(), n_out, k, n_tok)
        _check(y.cpu().numpy(), yo, s, k)


def test_gemv_batch_rows_wider_than_a_share(iqq, synth):
    """One 65536-wide row among 40 one-row problems of width 128: the CTAs split the bytes
    evenly, so one CTA takes the wide row alone and another has no row to start; every
    output equals its single call bit for bit and lies within the bound of the oracle's
    value."""
    rng = np.random.default_rng(42)
    items, singles, refs = [], [], []
    for i, (n_out, k, n_tok) in enumerate([(1, 65536, 2)] + [(1, 128, 1 + i % 3) for i in range(40)]):
        w = torch.from_numpy(_random_q4_0(rng, n_out, k)).cuda()
        a = torch.from_numpy(_activations(synth, n_tok, k, seed=200 + i)).cuda()
        y = torch.full((n_tok, n_out), float("nan"), device="cuda")
        items.append((w, a, y, k))
        singles.append(iqq.gemv_q4_0_q8_k128(w, a, n_out, k, n_tok))
        refs.append((n_out, k, n_tok))
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    iqq.iqq_gemv_q4_0_q8_k128_batch(iqq.gemv_problems(items), flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    for (w, a, y, k), single, (n_out, _, n_tok) in zip(items, singles, refs):
        assert torch.equal(y, single)
        yo, s = oracle.dot_q4_0_q8_k128(w.cpu().numpy(), a.cpu().numpy(), n_out, k, n_tok)
        _check(y.cpu().numpy(), yo, s, k)
