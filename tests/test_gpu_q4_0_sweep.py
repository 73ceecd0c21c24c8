"""The Q4_0 quantizer's transition-based sweep (iqq_quantize_q4_0_w) against the direct
sweep (iqq_quantize_q4_0_w_direct, every candidate's exact sums), byte for byte, and the
DeepSeek-shaped expert tensors against the CPU oracle.

The two GPU paths compute the same definition, so they must agree on every block, flags
included, whatever the input: shapes whose rows are not a multiple of 32 blocks, rows of
one block, bf16-valued weights (many exact rounding ties), boosted imatrix columns, every
importance form, stacked imatrix rows, and blocks outside the range where the sweep's
error bounds hold (tiny, huge, zero, non-finite values, zero weights)."""
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


def _both(iqq, x, qw, rows_per_qw=0, mode=0):
    nrows, n = x.shape
    a = torch.empty(iqq.q4_0_nbytes(nrows, n), dtype=torch.uint8, device=x.device)
    b = torch.empty_like(a)
    fa = torch.zeros(1, dtype=torch.int32, device=x.device)
    fb = torch.zeros(1, dtype=torch.int32, device=x.device)
    iqq.iqq_quantize_q4_0_w(x, qw, a, rows_per_qw, mode, fa)
    iqq.iqq_quantize_q4_0_w_direct(x, qw, b, rows_per_qw, mode, fb)
    torch.cuda.synchronize()
    return a, b, int(fa.item()), int(fb.item())


def _assert_same(a, b, fa, fb, what):
    if not torch.equal(a, b):
        d = (a.view(-1, 18) != b.view(-1, 18)).any(1).nonzero().flatten()
        raise AssertionError(f"{what}: {d.numel()} blocks differ, first {d[:8].tolist()}")
    assert fa == fb, (what, fa, fb)


@pytest.mark.parametrize("rows,n,bf16", [(4096, 4096, True), (1024, 11008, True), (4096, 4096, False),
                                         (333, 1056, False), (257, 32, False), (129, 64, False),
                                         (65, 96, False), (3, 53248, False)])
def test_layer_shapes_equal_direct_sweep(iqq, synth, rows, n, bf16):
    x = synth.weight_matrix(rows, n, seed=rows + n, bf16=bf16, device="cuda")
    qw = synth.imatrix(n, seed=n + 7, device="cuda")
    _assert_same(*_both(iqq, x, qw), f"{rows}x{n}")


@pytest.mark.parametrize("rows,n", [(2048, 7168), (7168, 2048)])
def test_expert_shapes_equal_direct_sweep(iqq, synth, rows, n):
    """DeepSeek-shaped experts (gate/up 2048x7168, down 7168x2048) with 5% of the imatrix
    columns boosted x100."""
    x = synth.weight_matrix(rows, n, seed=4_000_000 + rows, sigma=0.015, device="cuda")
    qw = synth.imatrix(n, seed=4_500_000 + rows, boost_frac=0.05, device="cuda")
    _assert_same(*_both(iqq, x, qw), f"expert {rows}x{n}")


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4, 5])
def test_importance_forms_equal_direct_sweep(iqq, synth, mode):
    x = synth.weight_matrix(512, 4096, seed=900 + mode, device="cuda")
    qw = synth.imatrix(4096, seed=910 + mode, device="cuda")
    for q in (qw, None):
        _assert_same(*_both(iqq, x, q, mode=mode), f"mode {mode} qw {q is not None}")


def test_stacked_imatrix_equals_direct_sweep(iqq, synth):
    x = synth.weight_matrix(300, 2048, seed=31, device="cuda")
    qw = synth.imatrix(2048 * 30, seed=32, boost_frac=0.05, device="cuda").view(30, 2048)
    _assert_same(*_both(iqq, x, qw, rows_per_qw=10), "rows_per_qw 10")


def test_blocks_outside_the_bounds_equal_direct_sweep(iqq, synth):
    """Blocks the filtered sweep hands to the direct sweep, and blocks at its edges."""
    rows, n = 64, 1024
    x = synth.weight_matrix(rows, n, seed=41, device="cuda")
    qw = synth.imatrix(n, seed=42, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(43)
    x[0, :32] = 0.0                                           # all zero
    x[1, :32] *= 1e-30                                        # tiny values
    x[2, :32] *= 1e30                                         # huge values (scale overflows binary16)
    x[3, :32] = 2.0 ** -130                                   # subnormal
    x[4, :32] = torch.randint(-8, 8, (32,), generator=g, device="cuda").float() * 0.01  # few magnitudes
    x[5, :] = torch.randint(-3, 4, (n,), generator=g, device="cuda").float() * 2.0 ** -7  # exact ties
    x[6, 5] = 1e-38                                            # one subnormal-range element
    x[7, :32] = x[7, :1].abs() * torch.tensor([1.0, -1.0] * 16, device="cuda")  # +-xmax repeated
    x[8, :32] = torch.tensor([0.625, -1.0, 0.5, 0.75] * 8, device="cuda")  # ratios on candidates
    q = qw.clone()
    q[64:96] = 0.0                                            # a block with no weight
    q[96:100] = 1e-30                                         # tiny weights inside a block
    _assert_same(*_both(iqq, x, q), "edge blocks")
    xn = x.clone()
    xn[10, 3] = float("nan")
    xn[11, 40] = float("inf")
    qn = q.clone()
    qn[200] = -1.0
    a, b, fa, fb = _both(iqq, xn, qn)
    assert fa == fb == 1 | 2 | 4
    keep = [r for r in range(rows) if r not in (10, 11)]
    cols = [c for c in range(n // 32) if c != 200 // 32]
    av, bv = a.view(rows, n // 32, 18)[keep][:, cols], b.view(rows, n // 32, 18)[keep][:, cols]
    assert torch.equal(av, bv)


def test_bf16_entry_uses_the_same_sweep(iqq, synth):
    xb = synth.weight_matrix(1024, 11008, seed=51, bf16=True, device="cuda").to(torch.bfloat16)
    x = xb.float()
    qw = synth.imatrix(11008, seed=52, device="cuda")
    a, b, _, _ = _both(iqq, x, qw)
    c = torch.empty_like(a)
    iqq.iqq_quantize_qx_0_w_bf16(4, xb, qw, c)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(a, c)


@pytest.mark.parametrize("which", ["gate", "down"])
def test_expert_tensor_against_oracle(iqq, synth, which):
    """A full-size expert tensor of the DeepSeek-shaped set (first expert, 5% of the imatrix
    columns boosted x100) against the oracle on a sample of rows, the first and the last
    included: >= 99.99% of the blocks bit-exact, any other within 1e-5 weighted error."""
    t = [e for e in synth.moe_experts(1) if e.name.endswith(which)][0]
    x = t.weights()
    qw = t.qw()
    blocks = iqq.quantize_q4_0_w(x.cuda(), qw.cuda()).cpu().numpy()
    rng = np.random.default_rng(7)
    rows = sorted({0, t.rows - 1, *rng.choice(t.rows, 94, replace=False).tolist()})
    xs = x.numpy()[rows]
    o, _ = oracle.quantize_q4_0_w(xs, qw.numpy())
    stats = compare_q4_0(xs, qw.numpy(), blocks.reshape(t.rows, -1)[rows], o, rows=None)
    assert stats["blocks"] == len(rows) * (t.cols // 32)


@pytest.mark.parametrize("rows,n,rpq,with_y", [(4096, 4096, 0, True), (2048, 7168, 0, True), (333, 1056, 0, True),
                                               (129, 64, 10, False), (3, 53248, 1, True)])
def test_epilogue_variant(iqq, synth, rows, n, rpq, with_y):
    """The quantizer with its epilogue (iqq_quantize_qx_0_w_ex with y and acc): the blocks are
    those of the plain entry point byte for byte, y is the dequantization kernel's bit for bit,
    and the round-trip sums are the weighted-RMSE kernel's up to the order of the binary64
    additions (max |e| exact)."""
    x = synth.weight_matrix(rows, n, seed=rows + n, bf16=True, device="cuda")
    nq = 1 if rpq == 0 else (rows + rpq - 1) // rpq
    qw = torch.stack([synth.imatrix(n, seed=n + i, boost_frac=0.05, device="cuda") for i in range(nq)])
    qw = qw if rpq else qw[0]
    out = torch.empty(iqq.q4_0_nbytes(rows, n), dtype=torch.uint8, device="cuda")
    acc = torch.zeros(4, dtype=torch.float64, device="cuda")
    y = torch.empty_like(x) if with_y else None
    iqq.iqq_quantize_qx_0_w_ex(4, x, qw, out, None, acc, rpq, y=y)
    plain = torch.empty_like(out)
    iqq.iqq_quantize_q4_0_w(x, qw, plain, rpq)
    ref = torch.zeros(4, dtype=torch.float64, device="cuda")
    iqq.iqq_weighted_rmse(x, plain, qw, ref, rpq)
    torch.cuda.synchronize()
    assert torch.equal(out, plain)
    if with_y:
        assert torch.equal(y, iqq.dequant_q4_0(out, rows, n))
    a, r = acc.cpu().numpy(), ref.cpu().numpy()
    assert np.allclose(a[:3], r[:3], rtol=1e-10, atol=0) and a[3] == r[3]


def test_batched_launches_equal_single_tensor_calls(iqq, synth):
    """iqq_quantize_q4_0_w_batch: 70 tensors of mixed shapes (more than one launch's 64; ragged
    last tiles, one-block rows, stacked and shared imatrix rows, an empty tensor, a row with a
    NaN) give the blocks of single-tensor calls byte for byte, and the flags of the tensors."""
    rng = np.random.default_rng(5)
    shapes = [(4096, 4096), (333, 1056), (129, 64), (65, 96), (3, 53248), (1, 32), (257, 32), (0, 4096)]
    items, singles = [], []
    shared = synth.imatrix(1056, seed=77, device="cuda")
    for i in range(70):
        rows, n = shapes[i % len(shapes)] if i < 16 else (int(rng.integers(1, 300)), 32 * int(rng.integers(1, 40)))
        x = synth.weight_matrix(rows, n, seed=500 + i, bf16=(i % 2 == 0), device="cuda") if rows else \
            torch.empty(0, n, device="cuda")
        rpq = 0 if i % 3 else 4
        if n == 1056 and rpq == 0:
            qw = shared
        elif rpq:
            nq = max(1, (rows + rpq - 1) // rpq)
            qw = torch.stack([synth.imatrix(n, seed=600 + i * 10 + j, device="cuda") for j in range(nq)])
        else:
            qw = synth.imatrix(n, seed=600 + i, boost_frac=0.05, device="cuda")
        out = torch.empty(max(1, iqq.q4_0_nbytes(rows, n)), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(out)
        if rows:
            iqq.iqq_quantize_q4_0_w(x, qw, ref, rpq)
        items.append((x, qw, out, rpq))
        singles.append(ref)
    bad = items[0][0].clone()
    bad[7, 100] = float("nan")
    items.append((bad, items[0][1], torch.empty_like(items[0][2]), 0))
    fb = torch.zeros(1, dtype=torch.int32, device="cuda")
    iqq.iqq_quantize_q4_0_w_batch(iqq.q4_0_problems(items[:-1]), flags=fb)
    fn = torch.zeros(1, dtype=torch.int32, device="cuda")
    iqq.iqq_quantize_q4_0_w_batch(iqq.q4_0_problems(items[-1:]), flags=fn)
    torch.cuda.synchronize()
    for i, ((x, _, out, _), ref) in enumerate(zip(items[:-1], singles)):
        if x.shape[0]:
            assert torch.equal(out, ref), i
    assert int(fb.item()) == 0
    assert int(fn.item()) & iqq.FLAG_NONFINITE_INPUT
