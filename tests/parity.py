"""Helpers for comparing the CUDA path with the CPU oracle (test infrastructure)."""
import numpy as np

import oracle


def q4_0_block_errors(x, qw, blocks, rows_per_qw=0, weight_mode=0, rows=None):
    """Weighted error sum w (x - y)^2 (binary64) of every block, with the quantizer's
    own weights (sigma2 + the weight formula evaluated by the oracle)."""
    nrows, n = x.shape
    nb = n // 32
    rows = range(nrows) if rows is None else rows
    d16, codes = oracle.decode_q4_0(blocks, len(blocks), n)
    out = np.zeros((len(rows), nb))
    for i, r in enumerate(rows):
        s2 = oracle.row_sigma2(x[r])
        q = None
        if qw is not None:
            q = qw if qw.ndim == 1 else qw[(r // rows_per_qw) if rows_per_qw else 0]
        y = d16[i].view(np.float16).astype(np.float64)[:, None] * codes[i].reshape(nb, 32)
        for b in range(nb):
            xb = x[r, 32 * b:32 * b + 32]
            w = oracle.block_weights(xb, None if q is None else q[32 * b:32 * b + 32], s2, weight_mode)
            out[i, b] = np.sum(w.astype(np.float64) * (xb.astype(np.float64) - y[b]) ** 2)
    return out


def compare_q4_0(x, qw, gpu_blocks, ref_blocks, rows_per_qw=0, weight_mode=0, rows=None,
                 min_exact=0.9999, err_rtol=1e-5):
    """Asserts the parity criterion: >= min_exact of the blocks bit-exact, and every other
    block's weighted error within err_rtol (relative) of the oracle's.  Returns stats."""
    nrows_cmp = gpu_blocks.shape[0]
    g = gpu_blocks.reshape(nrows_cmp, -1, 18)
    o = ref_blocks.reshape(nrows_cmp, -1, 18)
    diff = np.any(g != o, axis=2)
    nblk = diff.size
    ndiff = int(diff.sum())
    stats = {"blocks": nblk, "differing": ndiff, "exact_fraction": 1.0 - ndiff / max(nblk, 1)}
    if ndiff:
        ri, bi = np.nonzero(diff)
        urows = sorted(set(ri.tolist()))
        row_ids = [rows[r] if rows is not None else r for r in urows]
        eg = q4_0_block_errors(x, qw, gpu_blocks[urows], rows_per_qw, weight_mode, row_ids)
        eo = q4_0_block_errors(x, qw, ref_blocks[urows], rows_per_qw, weight_mode, row_ids)
        pos = {r: i for i, r in enumerate(urows)}
        worst = 0.0
        for r, b in zip(ri, bi):
            a, e = eg[pos[r], b], eo[pos[r], b]
            rel = abs(a - e) / max(e, 1e-300)
            worst = max(worst, rel)
        stats["worst_rel_err_diff"] = worst
        assert worst <= err_rtol, stats
    assert stats["exact_fraction"] >= min_exact, stats
    return stats
