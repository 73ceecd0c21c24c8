"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Criteria:
  Q4_0 (imatrix weighted): d16 and codes bit-exact in >= 99.99% of blocks; any other
    block's weighted error within 1e-5 (relative) of the oracle's.  The one expected
    source of difference is the binary64 row sum behind sigma2, whose summation order
    differs (a tree on the GPU, left to right in the oracle).
  Q8_K_128: d, codes and sums bit-exact.
  Dequantization: bit-exact.
  Weighted RMSE: sums within 1e-9 relative (binary64 atomics have no fixed order), max
    |e| exact.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import compare_q4_0

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


def _gpu_q4_0(iqq, x, qw, rows_per_qw=0, mode=0):
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    qd = None if qw is None else torch.from_numpy(np.ascontiguousarray(qw)).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = iqq.quantize_q4_0_w(xd, qd, rows_per_qw, mode, flags)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(flags.item())


# ------------------------------------------------------------------ Q4_0 weighted

@pytest.mark.parametrize("mode", [0, 1])
def test_q4_0_single_matrix_1024x4096(iqq, synth, mode):
    t = synth.single_matrix_1024x4096()
    x = t.weights().numpy()
    qw = t.qw().numpy()
    g, gf = _gpu_q4_0(iqq, x, qw, mode=mode)
    o, of = oracle.quantize_q4_0_w(x, qw, weight_mode=mode)
    assert gf == of == 0
    compare_q4_0(x, qw, g, o, weight_mode=mode)


@pytest.mark.parametrize("mode", [2, 3, 4, 5])
def test_q4_0_magnitude_weight_forms(iqq, synth, mode):
    """The importance forms x^2, |x|, sigma^2 + x^2, sigma + |x| (times qw, and alone)."""
    x = synth.weight_matrix(96, 4096, seed=40 + mode).numpy()
    qw = synth.imatrix(4096, seed=50 + mode).numpy()
    for q in (qw, None):
        g, gf = _gpu_q4_0(iqq, x, q, mode=mode)
        o, of = oracle.quantize_q4_0_w(x, q, weight_mode=mode)
        assert gf == of == 0
        compare_q4_0(x, q, g, o, weight_mode=mode)


@pytest.mark.parametrize("rows,n", [(37, 4192), (3, 32), (5, 11008), (9, 2048), (2, 7168), (1, 12320)])
def test_q4_0_ragged_shapes(iqq, synth, rows, n):
    """Several 128-block chunks per row with a ragged last chunk, single-block rows."""
    x = synth.weight_matrix(rows, n, seed=rows * 1000 + n).numpy()
    qw = synth.imatrix(n, seed=n).numpy()
    g, _ = _gpu_q4_0(iqq, x, qw)
    o, _ = oracle.quantize_q4_0_w(x, qw)
    compare_q4_0(x, qw, g, o, min_exact=1.0 if rows * n < 100000 else 0.9999)


def test_q4_0_no_imatrix_and_stacked_imatrix(iqq, synth):
    x = synth.weight_matrix(48, 1024, seed=77).numpy()
    g, _ = _gpu_q4_0(iqq, x, None)
    o, _ = oracle.quantize_q4_0_w(x, None)
    compare_q4_0(x, None, g, o)
    qw = np.stack([synth.imatrix(1024, seed=s, boost_frac=0.05).numpy() for s in range(4)])
    g, _ = _gpu_q4_0(iqq, x, qw, rows_per_qw=12)
    o, _ = oracle.quantize_q4_0_w(x, qw, rows_per_qw=12)
    compare_q4_0(x, qw, g, o, rows_per_qw=12)


def test_q4_0_degenerate_blocks_and_flags(iqq, synth):
    rng = np.random.default_rng(5)
    x = synth.weight_matrix(8, 256, seed=5).numpy()
    qw = synth.imatrix(256, seed=6).numpy()
    x[0, :32] = 0.0                         # all-zero block
    x[1, 32:64] = np.float32(0.02)          # constant block
    qw[64:96] = 0.0                         # no weight anywhere in block 2 -> fallback
    x[2, 96:128] = np.float32(2.0 ** -6) * rng.integers(-8, 8, 32).astype(np.float32)
    x[2, 96] = np.float32(-8 * 2.0 ** -6)   # exactly representable block
    x[3, 128:160] = x[3, 128:160] * np.float32(1e8)   # scale beyond binary16
    g, gf = _gpu_q4_0(iqq, x, qw)
    o, of = oracle.quantize_q4_0_w(x, qw)
    assert gf == of == 4                    # IQQ_FLAG_SCALE_OVERFLOW
    assert np.array_equal(g, o)
    xn = x.copy()
    xn[5, 7] = np.nan
    qn = qw.copy()
    qn[200] = -1.0
    g2, gf2 = _gpu_q4_0(iqq, xn, qn)
    o2, of2 = oracle.quantize_q4_0_w(xn, qn)
    assert gf2 == of2 == 1 | 2 | 4
    # a NaN row and a block holding a negative importance are flagged and their bytes
    # unspecified; everything else is untouched
    keep = [r for r in range(8) if r != 5]
    g2b = g2.reshape(8, 8, 18)[keep]
    o2b = o2.reshape(8, 8, 18)[keep]
    cols = [c for c in range(8) if c != 200 // 32]
    assert np.array_equal(g2b[:, cols], o2b[:, cols])


def test_q4_0_exact_golden_blocks(iqq):
    from conftest import read_golden
    for rec in read_golden("q4_0_exact_blocks.txt"):
        d0 = float(rec["d0"])
        n = np.array([int(v) for v in rec["n"].split()], np.float32)
        x = (np.float32(d0) * n).reshape(1, 32)
        for mode in (0, 1):
            g, _ = _gpu_q4_0(iqq, x, np.ones(32, np.float32), mode=mode)
            o, _ = oracle.quantize_q4_0_w(x, np.ones(32, np.float32), weight_mode=mode)
            assert np.array_equal(g, o)


@pytest.mark.parametrize("shape", [(4096, 4096), (11008, 4096), (4096, 11008), (2048, 7168),
                                   (7168, 2048), (16384, 53248)])
def test_q4_0_full_size_sampled_rows(iqq, synth, shape):
    """Full-size tensors quantized in one launch as the benchmark does; a seeded sample
    of rows (plus the first and last) checked against the oracle."""
    r, n = shape
    bf16 = shape in ((4096, 4096), (11008, 4096), (4096, 11008))
    xg = synth.weight_matrix(r, n, seed=3000 + r + n, bf16=bf16, device="cuda")
    qg = synth.imatrix(n, seed=11 + n, boost_frac=0.05 if n in (7168, 2048) else 0.0, device="cuda")
    out = iqq.quantize_q4_0_w(xg, qg)
    torch.cuda.synchronize()
    rng = np.random.default_rng(r + n)
    rows = sorted(set([0, r - 1] + rng.choice(r, size=24, replace=False).tolist()))
    x = xg[rows].cpu().numpy()
    qw = qg.cpu().numpy()
    g = out[rows].cpu().numpy()
    del xg, out
    o, _ = oracle.quantize_q4_0_w(x, qw)
    compare_q4_0(x, qw, g, o)


# ------------------------------------------------------------------ Q8_K_128

def _gpu_q8(iqq, x):
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = iqq.quantize_q8_k128(xd, flags)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(flags.item())


def test_q8_k128_activations_4096x7168_bit_exact(iqq, synth):
    x = synth.activation_batch_4096x7168().numpy()
    g, gf = _gpu_q8(iqq, x)
    o, of = oracle.quantize_q8_k128(x)
    assert gf == of == 0
    assert np.array_equal(g, o)


def test_q8_k128_edge_blocks(iqq):
    x = np.random.default_rng(3).standard_normal((6, 384)).astype(np.float32)
    x[0, :128] = 0.0                                     # zero block
    x[1, 128:256] = 1e-38                                # tiny amax: 127/amax overflows
    x[1, 130] = 0.0
    x[2, :128] = np.float32(65504.0) * 3                 # beyond fp16
    x[3, 5] = 1.0e30
    x[4, :] = np.arange(384, dtype=np.float32) - 192     # ramps with exact products
    g, gf = _gpu_q8(iqq, x)
    o, of = oracle.quantize_q8_k128(x)
    assert gf == of == 0
    assert np.array_equal(g, o)
    xn = x.copy()
    xn[5, 300] = np.inf
    g, gf = _gpu_q8(iqq, xn)
    o, of = oracle.quantize_q8_k128(xn)
    assert gf == of == 1
    assert np.array_equal(g.reshape(6, 3, 140)[:5], o.reshape(6, 3, 140)[:5])


@pytest.mark.parametrize("rows,n", [(1, 128), (3, 1280), (17, 7168), (1000, 256)])
def test_q8_k128_shapes(iqq, rows, n):
    x = (np.random.default_rng(rows + n).standard_normal((rows, n)) * 3).astype(np.float32)
    g, _ = _gpu_q8(iqq, x)
    o, _ = oracle.quantize_q8_k128(x)
    assert np.array_equal(g, o)


# ------------------------------------------------------------------ Q5_0 / Q6_0 / Q8_0 weighted

@pytest.mark.parametrize("bits", [5, 6, 8])
@pytest.mark.parametrize("rows,n", [(256, 4096), (7, 4192), (3, 11008)])
def test_qx_0_weighted_and_dequant(iqq, synth, bits, rows, n):
    x = synth.weight_matrix(rows, n, seed=bits * 100 + rows).numpy()
    qw = synth.imatrix(n, seed=bits + n).numpy()
    xd, qd = torch.from_numpy(x).cuda(), torch.from_numpy(qw).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = iqq.quantize_qx_0_w(bits, xd, qd, flags=flags)
    y = iqq.dequant_qx_0(bits, g, rows, n)
    torch.cuda.synchronize()
    o, of = oracle.quantize_qx_0_w(bits, x, qw)
    bb = oracle.qx_block_bytes(bits)
    gb = g.cpu().numpy().reshape(-1, bb)
    ob = o.reshape(-1, bb)
    same = np.all(gb == ob, axis=1)
    assert int(flags.item()) == of == 0
    assert same.mean() >= 0.9999
    # dequantization of the GPU's blocks is bit-exact against the oracle's decoder
    assert np.array_equal(y.cpu().numpy(), oracle.dequant_qx_0(bits, g.cpu().numpy(), rows, n))
    # the weighted RMSE of the GPU's blocks against the oracle's reduction of the same blocks
    acc = iqq.weighted_rmse_qx(bits, xd, g, qd)
    torch.cuda.synchronize()
    ref = oracle.weighted_rmse_qx(bits, x, g.cpu().numpy(), qw)
    a = acc.cpu().numpy()
    assert np.allclose(a[:3], ref[:3], rtol=1e-9, atol=0) and a[3] == ref[3]
    # the one-pass dequantization + round trip: same y bits, same sums
    y2 = torch.empty_like(xd)
    acc2 = torch.zeros(4, dtype=torch.float64, device="cuda")
    iqq.iqq_dequant_rmse_qx(bits, xd, g, qd, y2, acc2)
    torch.cuda.synchronize()
    assert torch.equal(y2, y)
    a2 = acc2.cpu().numpy()
    assert np.allclose(a2[:3], ref[:3], rtol=1e-9, atol=0) and a2[3] == ref[3]
    # any differing block: weighted error within 1e-5 of the oracle's
    if not same.all():
        yo = oracle.dequant_qx_0(bits, o, rows, n).reshape(-1, 32).astype(np.float64)
        yg = y.cpu().numpy().reshape(-1, 32).astype(np.float64)
        xb = x.reshape(-1, 32).astype(np.float64)
        for i in np.nonzero(~same)[0]:
            r = i // (n // 32)
            w = oracle.block_weights(x[r, 32 * (i % (n // 32)):][:32], qw[32 * (i % (n // 32)):][:32],
                                     oracle.row_sigma2(x[r]), 0).astype(np.float64)
            eg, eo = np.sum(w * (xb[i] - yg[i]) ** 2), np.sum(w * (xb[i] - yo[i]) ** 2)
            assert abs(eg - eo) <= 1e-5 * eo


def _compare_qx(bits, x, qw, g, o, rows, n, min_exact=0.9999, mode=0, fudge=1.0):
    bb = oracle.qx_block_bytes(bits)
    gb = g.reshape(-1, bb)
    ob = o.reshape(-1, bb)
    same = np.all(gb == ob, axis=1)
    assert same.mean() >= min_exact, same.mean()
    if not same.all():
        yo = oracle.dequant_qx_0(bits, o, rows, n).reshape(-1, 32).astype(np.float64)
        yg = oracle.dequant_qx_0(bits, g, rows, n).reshape(-1, 32).astype(np.float64)
        xb = x.reshape(-1, 32).astype(np.float64)
        for i in np.nonzero(~same)[0]:
            r, c = divmod(int(i), n // 32)
            s2 = float(np.float32(fudge) * np.float32(oracle.row_sigma2(x[r])))
            w = oracle.block_weights(x[r, 32 * c:32 * c + 32], qw[32 * c:32 * c + 32], s2, mode).astype(np.float64)
            eg, eo = np.sum(w * (xb[i] - yg[i]) ** 2), np.sum(w * (xb[i] - yo[i]) ** 2)
            assert abs(eg - eo) <= 1e-5 * eo


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rows,n", [(3, 53248), (5, 16416), (2, 12320)])
def test_qx_0_workspace_wide_rows(iqq, synth, bits, rows, n):
    """Rows spanning 4 or more CTAs: sigma2 from the per-row pass into the workspace."""
    assert iqq.qx_0_w_workspace_bytes(rows, n) > 0
    x = synth.weight_matrix(rows, n, seed=rows + n + bits).numpy()
    qw = synth.imatrix(n, seed=n + 1).numpy()
    xd, qd = torch.from_numpy(x).cuda(), torch.from_numpy(qw).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    g_ws = iqq.quantize_qx_0_w_ws(bits, xd, qd, flags=flags)
    g_fused = iqq.quantize_qx_0_w(bits, xd, qd)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    o, _ = oracle.quantize_qx_0_w(bits, x, qw)
    _compare_qx(bits, x, qw, g_ws.cpu().numpy(), o, rows, n)
    assert np.mean(np.all(g_ws.cpu().numpy().reshape(-1, oracle.qx_block_bytes(bits)) ==
                          g_fused.cpu().numpy().reshape(-1, oracle.qx_block_bytes(bits)), axis=1)) >= 0.9999


@pytest.mark.parametrize("bits,rows,n,rpq", [(4, 64, 4096, 0), (4, 9, 11008, 3), (5, 5, 53248, 0),
                                              (8, 3, 12320, 1), (6, 37, 4192, 0)])
def test_quantize_with_fused_round_trip_error(iqq, synth, bits, rows, n, rpq):
    """One pass: the quantizer's dequantized output equals the dequantization kernel's bit for
    bit, its accumulation of the round trip equals the oracle's weighted-RMSE reduction of
    the same blocks (sums within 1e-9, max |e| exact), and its blocks equal the plain entry
    point's."""
    x = synth.weight_matrix(rows, n, seed=60 + rows).numpy()
    nq = 1 if rpq == 0 else (rows + rpq - 1) // rpq
    qw = np.stack([synth.imatrix(n, seed=70 + i).numpy() for i in range(nq)])
    xd, qd = torch.from_numpy(x).cuda(), torch.from_numpy(qw if rpq else qw[0]).cuda()
    acc = torch.zeros(4, dtype=torch.float64, device="cuda")
    out = torch.empty(rows * (n // 32) * iqq.QX_0_BLOCK_BYTES[bits], dtype=torch.uint8, device="cuda")
    nws = iqq.qx_0_w_workspace_bytes(rows, n)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda") if nws else None
    y = torch.empty_like(xd)
    iqq.iqq_quantize_qx_0_w_ex(bits, xd, qd, out, ws, acc, rpq, y=y)
    plain = iqq.quantize_qx_0_w(bits, xd, qd, rpq)
    y_ref = iqq.dequant_qx_0(bits, out, rows, n)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    g = out.cpu().numpy()
    same = np.mean(np.all(g.reshape(-1, oracle.qx_block_bytes(bits)) ==
                          plain.cpu().numpy().reshape(-1, oracle.qx_block_bytes(bits)), axis=1))
    assert same >= 0.9999
    ref = oracle.weighted_rmse_qx(bits, x, g, qw if rpq else qw[0], rpq)
    a = acc.cpu().numpy()
    assert np.allclose(a[:3], ref[:3], rtol=1e-9, atol=0) and a[3] == ref[3]


@pytest.mark.parametrize("bits,mode,fudge", [(4, 0, 0.5), (4, 0, 4.0), (4, 0, 0.0), (4, 4, 2.0),
                                              (5, 5, 0.25), (8, 0, 3.0)])
def test_quantize_fudge_factor(iqq, synth, bits, mode, fudge):
    """The importance's correction factor on sigma2 against the oracle's reading of it."""
    rows, n = 48, 4096
    x = synth.weight_matrix(rows, n, seed=90 + bits + mode).numpy()
    qw = synth.imatrix(n, seed=91).numpy()
    xd, qd = torch.from_numpy(x).cuda(), torch.from_numpy(qw).cuda()
    out = torch.empty(rows * (n // 32) * iqq.QX_0_BLOCK_BYTES[bits], dtype=torch.uint8, device="cuda")
    iqq.iqq_quantize_qx_0_w_ex(bits, xd, qd, out, weight_mode=mode, fudge=fudge)
    torch.cuda.synchronize()
    o, _ = oracle.quantize_qx_0_w(bits, x, qw, 0, mode, fudge=fudge)
    _compare_qx(bits, x, qw, out.cpu().numpy(), o, rows, n, mode=mode, fudge=fudge)


def test_qx_0_workspace_flags_nonfinite(iqq, synth):
    x = synth.weight_matrix(2, 53248, seed=1)
    x[1, 40000] = float("inf")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = iqq.quantize_qx_0_w_ws(4, x.cuda(), None, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & 1
    # the finite row is unaffected
    o, _ = oracle.quantize_qx_0_w(4, x[:1].numpy(), None)
    assert np.mean(np.all(g.cpu().numpy()[:1].reshape(-1, 18) == o.reshape(-1, 18), axis=1)) >= 0.9999


def test_qx_0_bits4_is_q4_0(iqq, synth):
    x = synth.weight_matrix(64, 4096, seed=9, device="cuda")
    q = synth.imatrix(4096, seed=10, device="cuda")
    assert torch.equal(iqq.quantize_qx_0_w(4, x, q), iqq.quantize_q4_0_w(x, q))
    with pytest.raises(iqq.IQQError, match="ARG"):
        iqq._check("q", iqq._lib.iqq_quantize_qx_0_w(7, x.data_ptr(), None, x.data_ptr(), 64, 4096, 0, 0,
                                                     None, None))


# ------------------------------------------------------------------ Q8_1 (overflow contrast)

def test_q8_1_bit_exact_and_overflow_count(iqq, synth):
    """On the activation batch with spikes beyond fp16, Q8_1's fp16 sums overflow in
    some blocks (counted identically on both sides) while Q8_K_128 stays finite."""
    x = synth.activation_batch_4096x7168().numpy()
    xd = torch.from_numpy(x).cuda()
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = iqq.quantize_q8_1(xd, cnt, flags)
    torch.cuda.synchronize()
    o, n_over = oracle.quantize_q8_1(x)
    assert np.array_equal(g.cpu().numpy(), o)
    assert int(cnt.item()) == n_over > 0 and int(flags.item()) == 0
    k = iqq.quantize_q8_k128(xd)
    d, _, _ = oracle.decode_q8_k128(k.cpu().numpy(), 4096, 7168)
    assert np.isfinite(d).all()


@pytest.mark.parametrize("rows,n", [(1, 32), (3, 96), (5, 160), (7, 4096)])
def test_q8_1_ragged_shapes(iqq, rows, n):
    x = (np.random.default_rng(rows * n).standard_normal((rows, n)) * 5e3).astype(np.float32)
    g = iqq.quantize_q8_1(torch.from_numpy(x).cuda()).cpu().numpy()
    o, _ = oracle.quantize_q8_1(x)
    assert np.array_equal(g, o)


# ------------------------------------------------------------------ dequant, weighted RMSE

def test_dequant_bit_exact(iqq, synth):
    t = synth.single_matrix_1024x4096()
    x = t.weights().numpy()
    qw = t.qw().numpy()
    o, _ = oracle.quantize_q4_0_w(x, qw)
    yg = iqq.dequant_q4_0(torch.from_numpy(o).cuda(), 1024, 4096)
    yo = oracle.dequant_q4_0(o, 1024, 4096)
    assert np.array_equal(yg.cpu().numpy().view(np.uint32), yo.view(np.uint32))
    # arbitrary block bytes: every finite binary16 scale, random nibbles
    rng = np.random.default_rng(9)
    raw = rng.integers(0, 256, size=(4096, 18), dtype=np.uint8)
    d16 = rng.integers(0, 0x7C00, size=4096).astype(np.uint16) | (rng.integers(0, 2, 4096) << 15).astype(np.uint16)
    raw[:, 0:2] = d16.view(np.uint8).reshape(-1, 2)
    yg = iqq.dequant_q4_0(torch.from_numpy(raw.reshape(64, -1)).cuda(), 64, 2048)
    yo = oracle.dequant_q4_0(raw.reshape(64, -1), 64, 2048)
    assert np.array_equal(yg.cpu().numpy().view(np.uint32), yo.view(np.uint32))


@pytest.mark.parametrize("shape", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_dequant_rmse_one_pass_full_size(iqq, synth, shape):
    """The bench's one-pass dequantization + round trip at the layer set's full sizes, in its
    launch configuration: every dequantized value bit-exact against the oracle's decoder, and
    the sums of the whole tensor within 1e-9 of the oracle's reduction."""
    r, n = shape
    xg = synth.weight_matrix(r, n, seed=700 + r + n, bf16=True, device="cuda")
    qg = synth.imatrix(n, seed=n + 7, device="cuda")
    blocks = iqq.quantize_q4_0_w(xg, qg)
    y = torch.empty_like(xg)
    acc = torch.zeros(4, dtype=torch.float64, device="cuda")
    iqq.iqq_dequant_rmse_qx(4, xg, blocks, qg, y, acc)
    torch.cuda.synchronize()
    x, qw, b = xg.cpu().numpy(), qg.cpu().numpy(), blocks.cpu().numpy()
    assert np.array_equal(y.cpu().numpy(), oracle.dequant_q4_0(b, r, n))
    ref = oracle.weighted_rmse(x, b, qw)
    a = acc.cpu().numpy()
    assert np.allclose(a[:3], ref[:3], rtol=1e-9, atol=0) and a[3] == ref[3]


@pytest.mark.parametrize("rows_per_qw", [0, 256])
def test_weighted_rmse(iqq, synth, rows_per_qw):
    t = synth.single_matrix_1024x4096()
    x = t.weights().numpy()
    qw = t.qw().numpy() if rows_per_qw == 0 else \
        np.stack([synth.imatrix(4096, seed=s).numpy() for s in range(4)])
    o, _ = oracle.quantize_q4_0_w(x, qw, rows_per_qw=rows_per_qw)
    acc = iqq.weighted_rmse(torch.from_numpy(x).cuda(), torch.from_numpy(o).cuda(),
                            torch.from_numpy(qw).cuda(), rows_per_qw).cpu().numpy()
    ref = oracle.weighted_rmse(x, o, qw, rows_per_qw)
    assert np.allclose(acc[:3], ref[:3], rtol=1e-9, atol=0)
    assert acc[3] == ref[3]
    # no imatrix: weights 1
    acc = iqq.weighted_rmse(torch.from_numpy(x).cuda(), torch.from_numpy(o).cuda()).cpu().numpy()
    ref = oracle.weighted_rmse(x, o, None)
    assert np.allclose(acc[:3], ref[:3], rtol=1e-9, atol=0) and acc[1] == x.size


def _random_q4_0_blocks(rng, nrows, n):
    """Seeded Q4_0 block bytes: random nibbles, finite binary16 scales of either sign."""
    raw = rng.integers(0, 256, size=(nrows * (n // 32), 18), dtype=np.uint8)
    d16 = rng.integers(0x1000, 0x3C00, size=raw.shape[0]).astype(np.uint16)
    d16 |= (rng.integers(0, 2, raw.shape[0]) << 15).astype(np.uint16)
    raw[:, 0:2] = d16.view(np.uint8).reshape(-1, 2)
    return raw.reshape(nrows, -1) if nrows else raw.reshape(0, 0)


def test_dequant_rmse_batch(iqq, synth):
    """The batched dequantization + round trip over 54 tensors (two launches of 48 and 6):
    mixed widths with ragged column tiles, shared and per-row-group imatrices, no imatrix, no
    y, an empty tensor.  Every y is bit-exact against the oracle's decoder and the per-tensor
    call, the accumulator holds the oracle's sums over all the tensors within 1e-9 and their
    exact max|e|."""
    rng = np.random.default_rng(31)
    specs = [(5, 4096, 0, True, True), (37, 4192, 0, True, True), (64, 11008, 16, True, True),
             (3, 32, 0, False, True), (0, 4096, 0, True, True), (9, 128, 1, True, False)]
    specs += [(2 + i % 5, 64 * (1 + i % 3), 0, i % 2 == 0, True) for i in range(48)]
    items, ref = [], np.zeros(4, np.float64)
    for i, (r, n, rpq, has_qw, has_y) in enumerate(specs):
        x = synth.weight_matrix(max(r, 1), n, seed=900 + i)[:r].contiguous()
        qrows = (r + rpq - 1) // rpq if rpq else 1
        qw = torch.stack([synth.imatrix(n, seed=i * 11 + k) for k in range(max(qrows, 1))]) if has_qw else None
        if qw is not None and rpq == 0:
            qw = qw[0].contiguous()
        b = _random_q4_0_blocks(rng, r, n)
        oracle.weighted_rmse(x.numpy(), b, None if qw is None else qw.numpy(), rpq, acc=ref)
        items.append((x, b, qw, rpq, has_y))
    dev = [(x.cuda(), torch.from_numpy(b).cuda(), None if qw is None else qw.cuda(),
            torch.full_like(x, float("nan"), device="cuda") if has_y else None, rpq)
           for x, b, qw, rpq, has_y in items]
    acc = torch.zeros(4, dtype=torch.float64, device="cuda")
    iqq.iqq_dequant_rmse_q4_0_batch(iqq.dequant_rmse_problems(dev), acc)
    torch.cuda.synchronize()
    a = acc.cpu().numpy()
    assert np.allclose(a[:3], ref[:3], rtol=1e-9, atol=0) and a[3] == ref[3]
    acc1 = torch.zeros(4, dtype=torch.float64, device="cuda")
    for (x, b, qw, y, rpq), (r, n, _, _, _) in zip(dev, specs):
        if y is not None:
            assert np.array_equal(y.cpu().numpy(), oracle.dequant_q4_0(b.cpu().numpy(), r, n))
            y1 = torch.empty_like(y)
            iqq.iqq_dequant_rmse_qx(4, x, b, qw, y1, acc1, rows_per_qw=rpq)
            assert torch.equal(y1, y)
        else:
            iqq.iqq_weighted_rmse(x, b, qw, acc1, rows_per_qw=rpq)
    a1 = acc1.cpu().numpy()
    assert np.allclose(a[:3], a1[:3], rtol=1e-12, atol=0) and a[3] == a1[3]


# ------------------------------------------------------------------ the C ABI's host checks

def test_abi_rejects_bad_arguments(iqq):
    x = torch.zeros(4, 64, device="cuda")
    out = torch.zeros(4 * 2 * 18, dtype=torch.uint8, device="cuda")
    with pytest.raises(iqq.IQQError, match="ALIGN"):
        iqq._check("q", iqq._lib.iqq_quantize_q4_0_w(x.data_ptr() + 4, None, out.data_ptr(), 3, 64,
                                                     0, 0, None, None))
    with pytest.raises(iqq.IQQError, match="SHAPE"):
        iqq.quantize_q8_k128(torch.zeros(2, 96, device="cuda"))
    with pytest.raises(iqq.IQQError, match="ARG"):
        iqq.quantize_q4_0_w(x, None, weight_mode=6)
    # empty input is a no-op
    iqq.quantize_q4_0_w(torch.zeros(0, 64, device="cuda"))


def test_runs_on_a_side_stream(iqq, synth):
    x = synth.weight_matrix(64, 4096, seed=1, device="cuda")
    ref = iqq.quantize_q4_0_w(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out = iqq.quantize_q4_0_w(x, stream=s)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("bits", [4, 5, 6, 8])
@pytest.mark.parametrize("rows,n,rpq", [(64, 4096, 0), (9, 11008, 3), (3, 53248, 0), (7, 4192, 1)])
def test_bf16_input_equals_the_widened_tensor(iqq, synth, bits, rows, n, rpq):
    """bf16 weights give, bit for bit, the blocks and flags of their exact binary32 widening
    (fused path, and with the workspace for wide rows), and the one-pass round trip against
    the bf16 tensor gives the binary32 one's y, sums and max|e|; the blocks meet the oracle
    bar."""
    xb = synth.weight_matrix(rows, n, seed=rows * 7 + n + bits, bf16=True).to(torch.bfloat16).cuda()
    x32 = xb.float()
    nq = (rows + rpq - 1) // rpq if rpq else 1
    qw = torch.stack([synth.imatrix(n, seed=n + i) for i in range(nq)]) if rpq else synth.imatrix(n, seed=n)
    qd = qw.cuda()
    f32, fbf = (torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(2))
    g32 = iqq.quantize_qx_0_w(bits, x32, qd, rows_per_qw=rpq, flags=f32)
    gbf = torch.empty_like(g32)
    iqq.iqq_quantize_qx_0_w_bf16(bits, xb, qd, gbf, rows_per_qw=rpq, flags=fbf)
    torch.cuda.synchronize()
    assert torch.equal(gbf, g32) and int(fbf.item()) == int(f32.item()) == 0
    nws = iqq.qx_0_w_workspace_bytes(rows, n)
    if nws > 0:
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        g32w = iqq.quantize_qx_0_w_ws(bits, x32, qd, rows_per_qw=rpq)
        gbfw = torch.empty_like(g32)
        iqq.iqq_quantize_qx_0_w_bf16(bits, xb, qd, gbfw, rows_per_qw=rpq, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(gbfw, g32w)
    if rpq == 0:
        x = x32.cpu().numpy()
        o, _ = oracle.quantize_qx_0_w(bits, x, qw.numpy())
        _compare_qx(bits, x, qw.numpy(), gbf.cpu().numpy(), o, rows, n)
    y32, ybf = torch.empty_like(x32), torch.empty_like(x32)
    a32, abf = (torch.zeros(4, dtype=torch.float64, device="cuda") for _ in range(2))
    iqq.iqq_dequant_rmse_qx(bits, x32, g32, qd, y32, a32, rows_per_qw=rpq)
    iqq.iqq_dequant_rmse_qx_bf16(bits, xb, g32, qd, ybf, abf, rows_per_qw=rpq)
    torch.cuda.synchronize()
    assert torch.equal(ybf, y32)
    a32, abf = a32.cpu().tolist(), abf.cpu().tolist()
    for i in range(3):  # binary64 atomics: the order of the per-CTA partial sums may vary
        assert abs(abf[i] - a32[i]) <= 1e-12 * abs(a32[i])
    assert abf[3] == a32[3]


def test_bf16_input_flags_nonfinite(iqq):
    """An infinity in bf16 x raises IQQ_FLAG_NONFINITE_INPUT on the fused path and in the
    per-row pass of wide rows."""
    for n in (4096, 53248):
        x = torch.zeros(4, n, dtype=torch.bfloat16, device="cuda")
        x[2, 100] = float("inf")
        out = torch.empty((4, (n // 32) * 18), dtype=torch.uint8, device="cuda")
        flags = torch.zeros(1, dtype=torch.int32, device="cuda")
        nws = iqq.qx_0_w_workspace_bytes(4, n)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda") if nws else None
        iqq.iqq_quantize_qx_0_w_bf16(4, x, None, out, workspace=ws, flags=flags)
        torch.cuda.synchronize()
        assert int(flags.item()) & iqq.FLAG_NONFINITE_INPUT
