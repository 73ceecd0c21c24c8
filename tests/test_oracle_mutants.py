"""The oracle's pins must be able to fail: each planted mistake below (a wrong sign,
a dropped term, a transposed layout, a wrong tie rule, ...) is compiled into a
scratch copy of the oracle on the CPU, and the pin suite run against that copy
must report at least one failure.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "nibble_order": ("blk[2 + i] = (uint8_t)((L[i] + 8) | ((L[i + 16] + 8) << 4));",
                     "blk[2 + i] = (uint8_t)((L[2*i] + 8) | ((L[2*i + 1] + 8) << 4));"),
    "sigma2_dropped": ("default: m = sqrtf(sigma2 + t); break;", "default: m = sqrtf(t); break;"),
    "greedy_direction": ("float s = g > 0.0f ? 1.0f : -1.0f;", "float s = g > 0.0f ? -1.0f : 1.0f;"),
    "iscale_sign": ("float iscale = -c / xmax;", "float iscale = c / xmax;"),
    "xmax_unsigned": ("if (a > amax) { amax = a; xmax = xb[j]; }",
                      "if (a > amax) { amax = a; xmax = a; }"),
    "ties_to_last_k": ("if (score > best) {", "if (score >= best) {"),
    "symmetric_clamp": ("const float lo = (float)(-nmax), hi = (float)(nmax - 1);\n    for (int j = 0; j < n; ++j) {\n        float v",
                        "const float lo = (float)(1 - nmax), hi = (float)(nmax - 1);\n    for (int j = 0; j < n; ++j) {\n        float v"),
    "greedy_trial_term": ("float nl2 = fmaf(w[j], 2.0f * s * lbest[j] + 1.0f, suml2);",
                          "float nl2 = fmaf(w[j], 2.0f * s * lbest[j], suml2);"),
    "q8_scale_128": ("float d = amax / 127.0f;\n        float id = amax > 0.0f ? 127.0f / amax : 0.0f;\n        int8_t q",
                     "float d = amax / 128.0f;\n        float id = amax > 0.0f ? 127.0f / amax : 0.0f;\n        int8_t q"),
    "q8_1_sum_unscaled": ("float sf = d * (float)sum;", "float sf = (float)sum;"),
    "q5_0_high_bit_order": ("if (bits == 5) qh |= (uint64_t)((n >> 4) & 1u) << j;",
                            "if (bits == 5) qh |= (uint64_t)((n >> 4) & 1u) << (31 - j);"),
    "q6_0_high_bits_dropped": ("else qh |= (uint64_t)((n >> 4) & 3u) << (2 * j);",
                               "else qh |= (uint64_t)((n >> 4) & 1u) << (2 * j);"),
    "qx_candidate_step": ("float c = (float)(nmax * (80 + k)) / 80.0f;",
                          "float c = (float)(nmax * (80 + 2 * k)) / 80.0f;"),
    "q8_truncation": ("float r = fminf(fmaxf(rintf(v), -127.0f), 127.0f);",
                      "float r = fminf(fmaxf(truncf(v), -127.0f), 127.0f);"),
    "rmse_unweighted": ("acc[0] += q * (ed * ed);", "acc[0] += (ed * ed);"),
    "dot_offset_7": ("* (double)(nib - 8);", "* (double)(nib - 7);"),
    "dot_nibble_order": ("const int nib = i < 16 ? (wb[2 + i] & 0xf) : (wb[2 + i - 16] >> 4);",
                         "const int nib = i < 16 ? (wb[2 + i] >> 4) : (wb[2 + i - 16] & 0xf);"),
    "dot_activation_scale_dropped": ("const double av = (double)d8 * (double)(int8_t)ab[4 + j % ORACLE_QK8];",
                                     "const double av = (double)(int8_t)ab[4 + j % ORACLE_QK8];"),
    "fudge_dropped": ("float sigma2 = fudge * oracle_row_sigma2(xr, n_per_row);",
                      "float sigma2 = oracle_row_sigma2(xr, n_per_row);"),
    "rmse_qw_row_index": ("const float *qr = qw ? qw + (rows_per_qw > 0 ? r / rows_per_qw : 0) * n_per_row : NULL;\n        for (int64_t b = 0; b < nb; ++b) {\n            const uint8_t *blk",
                           "const float *qr = qw ? qw + (rows_per_qw > 0 ? r / (rows_per_qw + 1) : 0) * n_per_row : NULL;\n        for (int64_t b = 0; b < nb; ++b) {\n            const uint8_t *blk"),
    "qx_qw_row_index": ("int8_t L[32];\n    for (int64_t r = 0; r < nrows; ++r) {\n        const float *xr = x + r * n_per_row;\n        const float *qr = qw ? qw + (rows_per_qw > 0 ? r / rows_per_qw : 0)",
                         "int8_t L[32];\n    for (int64_t r = 0; r < nrows; ++r) {\n        const float *xr = x + r * n_per_row;\n        const float *qr = qw ? qw + (rows_per_qw > 0 ? r / (rows_per_qw + 1) : 0)"),
    "mode5_sigma2_for_sigma": ("case 5: m = sigma + fabsf(x); break;", "case 5: m = sigma2 + fabsf(x); break;"),
    "mode4_sqrt": ("case 4: m = sigma2 + t; break;", "case 4: m = sqrtf(sigma2 + t); break;"),
    "greedy_four_passes": ("for (int pass = 0; pass < 5; ++pass) {", "for (int pass = 0; pass < 4; ++pass) {"),
    "greedy_six_passes": ("for (int pass = 0; pass < 5; ++pass) {", "for (int pass = 0; pass < 6; ++pass) {"),
    "sweep_drops_last_candidate": ("for (int k = -9; k <= 9; ++k) {", "for (int k = -9; k <= 8; ++k) {"),
    "fallback_scale_sign": ("return 1.0f / iscale0;", "return -1.0f / iscale0;"),
    "sigma2_sample_mean": ("return (float)(s / (double)n);", "return (float)(s / (double)(n - 1));"),
    "mode3_signed": ("case 3: m = fabsf(x); break;", "case 3: m = x; break;"),
    "q8_bsum_stride": ("for (int j = 0; j < 32; ++j) s += q[32 * i + j];",
                       "for (int j = 0; j < 32; ++j) s += q[4 * j + i];"),
    "q8_0_offset_codes": ("for (int j = 0; j < 32; ++j) blk[2 + j] = (uint8_t)L[j];",
                          "for (int j = 0; j < 32; ++j) blk[2 + j] = (uint8_t)(L[j] + 128);"),
    "fp16_ties_down": ("if (rem > half || (rem == half && (q & 1u))) q += 1u;",
                       "if (rem > half) q += 1u;"),
}

PIN_FILES = ["test_oracle_q4_0.py", "test_oracle_q8.py", "test_oracle_dequant_rmse.py",
             "test_oracle_qx.py", "test_oracle_dot.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_detect_planted_mistake(tmp_path, name):
    src = open(os.path.join(ROOT, "oracle", "iqq_oracle.c"), encoding="utf-8").read()
    a, b = MUTANTS[name]
    assert src.count(a) == 1, "mutation anchor must appear once"
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "*.tmp*", "__pycache__"))
    (tmp_path / "tests").mkdir()
    files = ["conftest.py", *PIN_FILES]
    if name.startswith("fp16"):
        files = ["conftest.py", "test_oracle_fp16.py"]
    for f in files:
        shutil.copy(os.path.join(ROOT, "tests", f), tmp_path / "tests" / f)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), tmp_path / "tests" / "golden")
    (tmp_path / "oracle" / "iqq_oracle.c").write_text(src.replace(a, b), encoding="utf-8")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "-k", "not exhaustive and not random_sample", "tests"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, r.stdout[-2000:]
    assert " failed" in r.stdout
