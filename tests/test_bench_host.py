"""Host-side logic of bench.py (no GPU): the peak denominators, the clock summary, the
warm-up guard and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_peaks_read_the_measured_file_or_fall_back():
    import bench
    p = bench.peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        assert p["source"] == "measured"
        assert p["hbm_gbs"] == float(m["hbm_gbs"]) and p["sm_max_mhz"] == float(m["sm_max_mhz"])
    else:
        assert p == {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}


def test_clock_summary_keeps_the_window_and_the_reasons():
    import bench
    c = bench.ClockSampler(0)
    row = "0, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, {sw}, {cap}"
    c.lines = [(0.5, row.format(mhz=500, sw="Not Active", cap="Not Active")),      # before the window
               (1.0, row.format(mhz=1965, sw="Not Active", cap="Active")),
               (1.1, row.format(mhz=1800, sw="Not Active", cap="Not Active")),
               (1.2, row.format(mhz=1900, sw="Active", cap="Not Active")),
               (1.3, "garbage"),
               (9.0, row.format(mhz=100, sw="Not Active", cap="Not Active"))]     # after it
    out = c.summarize(0.9, 1.25)
    assert out["samples"] == 3 and out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, "bench.py", "--warmup", "2"], cwd=ROOT, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 2 and "warmup" in r.stderr


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "vs_baseline", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun only rank 0 runs and prints the reference arm; the others exit 0
    without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                       timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_y_slices_of_a_launch_are_disjoint():
    """The bench's dequantized outputs: within each launch of the batched entry the tensors'
    slices are disjoint, 16-byte aligned and inside the buffer."""
    import bench
    from post_weight_quantization_rowwise_b200 import synth
    numels = [t.numel for t in synth.llama2_7b_layer_set(32)] + [5, 3, 4096]
    offs, size = bench.y_slices(numels)
    for g in range(0, len(numels), bench.RMSE_BATCH):
        spans = sorted((offs[i], offs[i] + numels[i]) for i in range(g, min(g + bench.RMSE_BATCH, len(numels))))
        assert all(a % 4 == 0 and b <= size for a, b in spans)
        assert all(spans[k][1] <= spans[k + 1][0] for k in range(len(spans) - 1))
    assert size == max(sum(-(-n // 4) * 4 for n in numels[g:g + bench.RMSE_BATCH])
                       for g in range(0, len(numels), bench.RMSE_BATCH))
