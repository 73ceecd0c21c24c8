"""iqq_quantize_qx_0_w_static: the per-row sigma2 pass into the library's own device array
(nothing allocated) against the workspace entry point, call after call, bytes equal."""
import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

STATIC_ROWS = 16384  # IQQ_STATIC_WS_ROWS


@pytest.fixture(scope="module")
def iqq():
    import post_weight_quantization_rowwise_b200 as m
    return m


@pytest.fixture(scope="module")
def synth():
    from post_weight_quantization_rowwise_b200 import synth as s
    return s


def _static(iqq, bits, x, qw, rows_per_qw=0, flags=None):
    nrows, n = x.shape
    out = torch.empty(nrows * (n // 32) * iqq.QX_0_BLOCK_BYTES[bits], dtype=torch.uint8, device=x.device)
    return iqq.iqq_quantize_qx_0_w_static(bits, x, qw, out, rows_per_qw, 0, flags)


def test_two_calls_match_the_workspace_entry(iqq, synth):
    """Two calls on different tensors (the array is reused): each equals the workspace path."""
    for rows, n, seed, bits in ((3, 53248, 11, 4), (5, 16416, 12, 8)):
        x = synth.weight_matrix(rows, n, seed=seed, device="cuda")
        qw = synth.imatrix(n, seed=seed + 1, device="cuda")
        a = _static(iqq, bits, x, qw)
        b = iqq.quantize_qx_0_w_ws(bits, x, qw)
        torch.cuda.synchronize()
        assert torch.equal(a, b.view(-1))


def test_row_batches_and_imatrix_segments(iqq, synth):
    """More rows than the static array: batches of rows, with a shared imatrix row, with one
    imatrix row per 3 rows (batches of 16383 rows, whole groups) and with one per 4 rows (4
    divides the array's rows: the second batch takes its imatrix rows from row 4096 on)."""
    rows, n = STATIC_ROWS + 3, 12320
    x = synth.weight_matrix(rows, n, seed=21, device="cuda")
    q1 = synth.imatrix(n, seed=22, device="cuda")
    q3 = torch.stack([synth.imatrix(n, seed=100 + i, device="cuda") for i in range((rows + 2) // 3)])
    q4 = synth.imatrix(n * ((rows + 3) // 4), seed=200_000, device="cuda").view(-1, n)
    for bits in (4, 8):
        for qw, rpq in ((q1, 0), (q3, 3), (q4, 4)):
            a = _static(iqq, bits, x, qw, rpq)
            b = iqq.quantize_qx_0_w_ws(bits, x, qw, rows_per_qw=rpq)
            torch.cuda.synchronize()
            assert torch.equal(a, b.view(-1)), (bits, rpq)


def test_narrow_rows_and_flags(iqq, synth):
    """Rows within three CTAs take the fused path; a non-finite x is reported."""
    x = synth.weight_matrix(64, 4096, seed=31, device="cuda")
    a = _static(iqq, 5, x, None)
    b = iqq.quantize_qx_0_w(5, x, None)
    x2 = synth.weight_matrix(2, 53248, seed=32, device="cuda")
    x2[1, 7] = float("nan")
    f = torch.zeros(1, dtype=torch.int32, device="cuda")
    _static(iqq, 4, x2, None, flags=f)
    torch.cuda.synchronize()
    assert torch.equal(a, b.view(-1))
    assert int(f.item()) & 1
