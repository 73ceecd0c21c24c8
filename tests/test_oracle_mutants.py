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
    "sigma2_dropped": ("float u = sigma2 + t;", "float u = t;"),
    "greedy_direction": ("float s = g > 0.0f ? 1.0f : -1.0f;", "float s = g > 0.0f ? -1.0f : 1.0f;"),
    "iscale_sign": ("float iscale = -c / xmax;", "float iscale = c / xmax;"),
    "xmax_unsigned": ("if (a > amax) { amax = a; xmax = xb[j]; }",
                      "if (a > amax) { amax = a; xmax = a; }"),
    "ties_to_last_k": ("if (score > best) {", "if (score >= best) {"),
    "symmetric_clamp": ("l[j] = fminf(fmaxf(r, -8.0f), 7.0f);", "l[j] = fminf(fmaxf(r, -7.0f), 7.0f);"),
    "greedy_trial_term": ("float nl2 = fmaf(w[j], 2.0f * s * lbest[j] + 1.0f, suml2);",
                          "float nl2 = fmaf(w[j], 2.0f * s * lbest[j], suml2);"),
    "q8_scale_128": ("float d = amax / 127.0f;", "float d = amax / 128.0f;"),
    "q8_truncation": ("float r = fminf(fmaxf(rintf(v), -127.0f), 127.0f);",
                      "float r = fminf(fmaxf(truncf(v), -127.0f), 127.0f);"),
    "rmse_unweighted": ("acc[0] += q * (ed * ed);", "acc[0] += (ed * ed);"),
    "fp16_ties_down": ("if (rem > half || (rem == half && (q & 1u))) q += 1u;",
                       "if (rem > half) q += 1u;"),
}

PIN_FILES = ["test_oracle_q4_0.py", "test_oracle_q8.py", "test_oracle_dequant_rmse.py"]


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
