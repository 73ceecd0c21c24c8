"""Benchmark: imatrix-weighted Q4_0 + Q8_K_128 quantization on B200.

One step = one pass of the whole path over the Llama-2-7B-shaped layer set
(32 layers x {q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008}, fp32
weights from bf16 N(0, 0.02) with 0.1% t(3) outliers, per-tensor log-normal
imatrix), for every tensor: weighted Q4_0 quantization, dequantization and the
weighted-RMSE reduction; plus Q8_K_128 quantization of a 4096 x 7168 activation
batch.  Inputs are synthetic and resident in HBM (25.9 GB of weights, far larger
than the 126 MB L2, so no L2 flush is needed between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU under torchrun;
every rank quantizes its own copy of the layer set (weak scaling, no collective
on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Gelem/s quantized (imatrix Q4_0, Q8_K_128) on 1 B200; % of HBM/FP32 roofline"
UNIT = "Gelem/s"
WORKLOAD = "llama2-7b layer set x32 (q4_0 imatrix + dequant + wrmse) + q8_k128 4096x7168"

# Algorithmic work per value:
#   Q4_0 weighted: 145 + 8*p binary32 lane operations per value, p = mean greedy passes:
#   1 for sigma2, 5 for the weight and w*x, 19 x 7 for the candidate sweep, about 2 for the
#   per-block constants, 4 for the final sums and packing, 8 per greedy pass;
#   Q8_K_128: 4 + 140/128 bytes per value; dequant + round trip: 4 + 18/32 + 4 (y written).
Q4_0_OPS_BASE = 145.0
Q4_0_OPS_PER_PASS = 8.0
Q8_BYTES_PER_VALUE = 4.0 + 140.0 / 128.0
DEQ_RMSE_BYTES_PER_VALUE = 4.0 + 18.0 / 32.0 + 4.0  # read x and the blocks, write y
B200_SMS = 148
FP32_LANES_PER_SM = 128
# DRAM bytes (read + write) per value of q4_0_w_kernel<float, false> from one ncu capture of
# the current kernel (the batched launch of the layer set's first layer, 7 tensors: see the
# q4_0_w_kernel profile summary); None whenever the kernel changes until it is captured again.
Q4_0_DRAM_BYTES_PER_VALUE = 4.5362
# tensors per launch of the batched dequantization + round-trip entry
RMSE_BATCH = 48


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def mark(self):
        """Start of the region whose samples count (the sampler is already running)."""
        self.t0 = time.perf_counter()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t1 = time.perf_counter()
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return self.summarize(getattr(self, "t0", 0.0), t1)

    def summarize(self, t0: float, t1: float):
        """Median SM clock, the maximum, and the throttle reasons active in [t0, t1 + 0.1]."""
        mhz, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ts, ln in self.lines:
            if ts < t0 or ts > t1 + 0.1:
                continue
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_chunk(args):
    """Worker: the oracle's whole path on one chunk of the fixed sample (a spawned process).
    The inputs are drawn first and not timed (the GPU arm's inputs are resident too)."""
    import oracle
    from post_weight_quantization_rowwise_b200 import synth
    kind, rows, cols, seed, bf16 = args
    if kind == "q8":
        a = synth.activations(rows, cols, seed=seed).numpy()
        t0 = time.perf_counter()
        oracle.quantize_q8_k128(a)
        return a.size, time.perf_counter() - t0, 0, 0
    x = synth.weight_matrix(rows, cols, seed=seed, bf16=bf16).numpy()
    qw = synth.imatrix(cols, seed=seed + 1).numpy()
    t0 = time.perf_counter()
    blocks, _, passes = oracle.quantize_q4_0_w(x, qw, want_passes=True)
    oracle.dequant_q4_0(blocks, rows, cols)
    oracle.weighted_rmse(x, blocks, qw)
    return x.size, time.perf_counter() - t0, int(passes.sum()), int(passes.size)


# The oracle's sample of the workload: 2^25 Q4_0 values (quantize + dequant + weighted RMSE)
# spread over the seven tensor shapes of the layer set in the set's proportions, plus Q8_K_128
# activation rows in the step's proportion (4096 x 7168 per 32 layers), cut into chunks of
# about 1 M values so that every core stays busy.  The same fixed sample serves the
# cpu_baseline leg and every step of the reference arm.
ORACLE_SAMPLE_Q4_VALUES = 1 << 25
ORACLE_CHUNK_VALUES = 1 << 20


def oracle_jobs():
    from post_weight_quantization_rowwise_b200 import synth
    layer = synth.LLAMA2_7B_TENSORS
    layer_elems = sum(r * c for _, r, c in layer)
    jobs = []
    for i, (name, r, c) in enumerate(layer):
        rows = max(1, round(ORACLE_SAMPLE_Q4_VALUES * (r * c) / layer_elems / c))
        per = max(1, ORACLE_CHUNK_VALUES // c)
        for k, r0 in enumerate(range(0, rows, per)):
            jobs.append(("q4", min(per, rows - r0), c, 9000 + 100 * i + k, True))
    q8_rows = max(1, round(ORACLE_SAMPLE_Q4_VALUES * 4096 * 7168 / (32 * layer_elems) / 7168))
    jobs.append(("q8", q8_rows, 7168, 2, False))
    return jobs


def oracle_sample(cores: int | None = None, pool=None):
    """Times the unchanged single-threaded oracle on the fixed sample, one process per host
    core.  Each chunk's oracle time is measured in its process; the step time is the sum of
    those times over the cores (the processes are independent).
    Returns (Gelem/s, cores, sample description, mean greedy passes, step seconds)."""
    import multiprocessing as mp
    cores = cores or os.cpu_count() or 1
    jobs = oracle_jobs()
    if pool is None:
        with mp.get_context("spawn").Pool(cores) as own:
            res = own.map(_oracle_chunk, jobs, chunksize=1)
    else:
        res = pool.map(_oracle_chunk, jobs, chunksize=1)
    elems = sum(r[0] for r in res)
    busy = sum(r[1] for r in res)
    pass_sum = sum(r[2] for r in res)
    pass_n = sum(r[3] for r in res)
    step_s = busy / cores
    sample = (f"fixed sample of {elems / 1e6:.1f} M values: {ORACLE_SAMPLE_Q4_VALUES / 1e6:.1f} M Q4_0 "
              f"(quantize + dequant + weighted RMSE) over the layer set's 7 shapes in its proportions, "
              f"plus {jobs[-1][1]} Q8_K_128 rows of 7168; {len(jobs)} chunks on {cores} processes, "
              f"{busy:.1f} s of oracle time per pass")
    return elems / step_s / 1e9, cores, sample, pass_sum / max(pass_n, 1), step_s


# ----------------------------------------------------------------------------- the GPU step

def y_slices(numels, batch: int = RMSE_BATCH):
    """Offsets (floats) of the tensors' dequantized outputs in one buffer, and its size: the
    tensors of one launch of the batched entry (`batch` a launch) write disjoint 16-byte
    aligned slices; the next launch reuses them (launches run in stream order)."""
    offs, size, off = [], 0, 0
    for i, n in enumerate(numels):
        if i % batch == 0:
            off = 0
        offs.append(off)
        off += -(-n // 4) * 4
        size = max(size, off)
    return offs, size


class Workload:
    def __init__(self, dev, rank: int, layers: int = 32):
        import torch
        from post_weight_quantization_rowwise_b200 import synth
        self.tensors = synth.llama2_7b_layer_set(layers)
        self.x, self.qw, self.blocks = [], [], []
        from post_weight_quantization_rowwise_b200 import replicas
        seed_off = replicas.rank_seed_offset(rank)
        for t in self.tensors:
            g = synth.Tensor2D(t.name, t.rows, t.cols, t.seed + seed_off, t.sigma, t.bf16,
                               t.boost_frac)
            self.x.append(g.weights(device=dev))
            self.qw.append(g.qw(device=dev))
            self.blocks.append(torch.empty(t.rows * (t.cols // 32) * 18, dtype=torch.uint8,
                                           device=dev))
        self.y_off, ysize = y_slices([t.numel for t in self.tensors])
        self.y = torch.empty(ysize, dtype=torch.float32, device=dev)
        self.acc = torch.zeros(4, dtype=torch.float64, device=dev)
        self.act = synth.activations(4096, 7168, seed=2 + seed_off, device=dev)
        self.q8 = torch.empty(4096 * 56 * 140, dtype=torch.uint8, device=dev)
        self.q4_elems = sum(t.numel for t in self.tensors)
        self.q8_elems = self.act.numel()
        self.q4_problems = None
        self.rmse_problems = None


def run_step(iqq, w: Workload, stream, ev=None):
    """Enqueues one step.  ev: optional list of 4 events bracketing the 3 phases: the
    weighted Q4_0 quantization of every tensor (the batched entry: 64 tensors a launch); the
    dequantization of every tensor with its round-trip weighted error accumulated in the same
    pass (the batched entry: 48 tensors a launch); Q8_K_128 of the activations."""
    import torch
    if w.q4_problems is None:  # the batched entries' descriptions, built and checked once
        w.q4_problems = iqq.q4_0_problems(list(zip(w.x, w.qw, w.blocks)))
        w.rmse_problems = iqq.dequant_rmse_problems(
            [(x, b, qw, w.y[o:o + t.numel].view(t.rows, t.cols))
             for t, x, qw, b, o in zip(w.tensors, w.x, w.qw, w.blocks, w.y_off)])
    if ev is not None:
        ev[0].record(stream)
    iqq.iqq_quantize_q4_0_w_batch(w.q4_problems, stream=stream)
    if ev is not None:
        ev[1].record(stream)
    w.acc.zero_()
    iqq.iqq_dequant_rmse_q4_0_batch(w.rmse_problems, w.acc, stream=stream)
    if ev is not None:
        ev[2].record(stream)
    iqq.iqq_quantize_q8_k128(w.act, w.q8, stream=stream)
    if ev is not None:
        ev[3].record(stream)
    return q4_launches(w) + rmse_launches(w) + 1


def q4_launches(w: Workload) -> int:
    """The quantization phase's launches: 64 tensors per launch of the batched entry."""
    return (len(w.tensors) + 63) // 64


def rmse_launches(w: Workload) -> int:
    """The dequantization phase's launches: RMSE_BATCH tensors per launch of the batched entry."""
    return (len(w.tensors) + RMSE_BATCH - 1) // RMSE_BATCH


def run_gemv_phase(iqq, w: Workload, dev, reps: int = 5):
    """One token through every quantized matrix of the layer set: y = W . a with the Q4_0
    blocks of the step and a Q8_K_128 activation of each matrix's width (4096 or 11008).
    The 224 launches are captured in one CUDA graph (the host-side cost of a launch exceeds
    a 9 MB matrix's device time); replays are timed with CUDA events.  The 3.6 GB of blocks
    exceed L2, so every replay streams them from HBM.  Returns (ms per pass, bytes)."""
    import torch
    from post_weight_quantization_rowwise_b200 import synth
    acts = {}
    for k in sorted({t.cols for t in w.tensors}):
        a = synth.activations(1, k, seed=7 + k, device=dev)
        acts[k] = iqq.quantize_q8_k128(a)
    y = torch.empty(max(t.rows for t in w.tensors), dtype=torch.float32, device=dev)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())

    def enqueue():
        for t, b in zip(w.tensors, w.blocks):
            iqq.iqq_gemv_q4_0_q8_k128(b, acts[t.cols], y[:t.rows].view(1, t.rows), t.cols, stream=s)

    with torch.cuda.stream(s):
        enqueue()  # outside the capture: fills the library's per-device launch caches
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        enqueue()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    with torch.cuda.stream(s):
        for _ in range(reps):
            g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = sum(t.rows * (t.cols // 32) * 18 + (t.cols // 128) * 140 + 4 * t.rows for t in w.tensors)
    del g
    # the same pass through the batched entry point (64 matrices per launch, 4 launches)
    ys = [torch.empty(1, t.rows, dtype=torch.float32, device=dev) for t in w.tensors]
    probs = iqq.gemv_problems([(b, acts[t.cols], y1, t.cols) for t, b, y1 in zip(w.tensors, w.blocks, ys)])
    bms = _timed(lambda: iqq.iqq_gemv_q4_0_q8_k128_batch(probs), reps=reps)
    # one large matrix (the widest scaling-sweep tensor, 490 MB of blocks): the kernel's
    # streaming rate once launch and ramp no longer matter
    big = synth.scaling_sweep()[3]
    xb = big.weights(device=dev)
    bb = iqq.quantize_q4_0_w(xb, big.qw(device=dev))
    del xb
    large = {}
    for tok in (1, 8):
        ab = iqq.quantize_q8_k128(synth.activations(tok, big.cols, seed=9, device=dev))
        yb = torch.empty(tok, big.rows, dtype=torch.float32, device=dev)
        lms = _timed(lambda: iqq.iqq_gemv_q4_0_q8_k128(bb, ab, yb, big.cols), reps=5)
        lbytes = big.rows * (big.cols // 32) * 18 + tok * (big.cols // 128) * 140 + 4 * tok * big.rows
        large[f"tokens_{tok}"] = {"ms": round(lms, 4), "bytes": int(lbytes), "gb_s": round(lbytes / lms / 1e6, 1)}
    del bb
    return ms, nbytes, {"matrix": f"{big.rows}x{big.cols}", **large}, bms


def _timed(fn, reps: int = 3):
    """Device ms per call of fn (one untimed call first), CUDA events on the current stream."""
    import torch
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def run_extras(iqq, dev, p_mean: float, peak_ops: float, hbm_gbs: float):
    """The other formats, importance forms and the Q8_1 contrast, each measured once:
      formats      Q4_0/Q5_0/Q6_0/Q8_0 weighted quantization, dequantization and weighted RMSE
                   of the 8192^2 tensor of the scaling sweep (256 MB, beyond L2);
      weight_modes the six importance forms on the same tensor (Q4_0);
      sweep_ab     weight = qw against qw*sqrt(sigma2 + x^2) on every scaling-sweep tensor;
      q8_1         Q8_1 against Q8_K_128 on the 4096x7168 activations with spikes."""
    import torch
    from post_weight_quantization_rowwise_b200 import synth
    out = {}
    sweep = synth.scaling_sweep()
    t = sweep[1]
    x, qw = t.weights(device=dev), t.qw(device=dev)
    n = x.numel()
    ops = Q4_0_OPS_BASE + Q4_0_OPS_PER_PASS * p_mean
    fm = {}
    for bits in (4, 5, 6, 8):
        blocks = torch.empty(t.rows * (t.cols // 32) * iqq.QX_0_BLOCK_BYTES[bits], dtype=torch.uint8, device=dev)
        y = torch.empty_like(x)
        qms = _timed(lambda: iqq.iqq_quantize_qx_0_w(bits, x, qw, blocks))
        dms = _timed(lambda: iqq.iqq_dequant_qx_0(bits, blocks, y))
        acc = iqq.weighted_rmse_qx(bits, x, blocks, qw)
        rms = _timed(lambda: iqq.iqq_weighted_rmse_qx(bits, x, blocks, qw, acc.zero_()))
        a = acc.cpu().tolist()
        dbytes = n * (4 + iqq.QX_0_BLOCK_BYTES[bits] / 32)
        fm[f"q{bits}_0"] = {"quantize_gelem_s": round(n / qms / 1e6, 3),
                            "quantize_frac": round(n * ops / (qms / 1e3) / 1e12 / peak_ops, 4),
                            "dequant_gb_s": round(dbytes / dms / 1e6, 1),
                            "dequant_hbm_frac": round(dbytes / dms / 1e6 / hbm_gbs, 4),
                            "rmse_gb_s": round(dbytes / rms / 1e6, 1),
                            "wrmse": math.sqrt(a[0] / a[1])}
        del blocks, y
    out["formats"] = {"tensor": t.name, "values": n, **fm}
    blocks = torch.empty(t.rows * (t.cols // 32) * 18, dtype=torch.uint8, device=dev)
    wm = {}
    for mode in range(6):
        qms = _timed(lambda: iqq.iqq_quantize_q4_0_w(x, qw, blocks, 0, mode))
        acc = iqq.weighted_rmse(x, blocks, qw)
        a = acc.cpu().tolist()
        wm[str(mode)] = {"gelem_s": round(n / qms / 1e6, 3), "wrmse": math.sqrt(a[0] / a[1])}
    out["weight_modes"] = {"tensor": t.name, "modes": "0 qw*sqrt(s2+x2), 1 qw, 2 qw*x2, 3 qw*|x|, "
                           "4 qw*(s2+x2), 5 qw*(sqrt(s2)+|x|)", **wm}
    fz = {}
    for f in (0.0, 0.25, 0.5, 1.0, 2.0, 4.0):
        iqq.iqq_quantize_qx_0_w_ex(4, x, qw, blocks, weight_mode=0, fudge=f)
        a = iqq.weighted_rmse(x, blocks, qw).cpu().tolist()
        fz[str(f)] = {"wrmse": math.sqrt(a[0] / a[1])}
    out["fudge"] = {"tensor": t.name, "mode": "qw*sqrt(fudge*s2 + x2)", **fz}
    del x, qw, blocks
    ab = {}
    for tt in sweep:
        x, qw = tt.weights(device=dev), tt.qw(device=dev)
        blocks = torch.empty(tt.rows * (tt.cols // 32) * 18, dtype=torch.uint8, device=dev)
        nws = iqq.qx_0_w_workspace_bytes(tt.rows, tt.cols)
        ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None
        row = {"workspace_bytes": nws}
        for mode, name in ((1, "qw"), (0, "qw_sqrt_s2_x2")):
            qms = _timed(lambda: iqq.iqq_quantize_qx_0_w_ws(4, x, qw, blocks, ws, 0, mode), reps=2)
            a = iqq.weighted_rmse(x, blocks, qw).cpu().tolist()
            row[name] = {"gelem_s": round(x.numel() / qms / 1e6, 3), "wrmse": math.sqrt(a[0] / a[1])}
        # the direct sweep (every candidate's exact sums) on the same tensor, for comparison
        qms = _timed(lambda: iqq.iqq_quantize_q4_0_w_direct(x, qw, blocks, 0, 0), reps=2)
        row["qw_sqrt_s2_x2_direct_sweep"] = {"gelem_s": round(x.numel() / qms / 1e6, 3)}
        ab[tt.name] = row
        del x, qw, blocks, ws
    out["sweep_ab"] = ab
    act = synth.activation_batch_4096x7168(device=dev)
    q81 = torch.empty(act.numel() // 32 * 36, dtype=torch.uint8, device=dev)
    q8k = torch.empty(act.numel() // 128 * 140, dtype=torch.uint8, device=dev)
    over = torch.zeros(1, dtype=torch.int64, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    iqq.iqq_quantize_q8_1(act, q81, over)
    iqq.iqq_quantize_q8_k128(act, q8k, flags)
    torch.cuda.synchronize()
    n_over = int(over.item())
    m1 = _timed(lambda: iqq.iqq_quantize_q8_1(act, q81))
    mk = _timed(lambda: iqq.iqq_quantize_q8_k128(act, q8k))
    na = act.numel()
    out["q8_1"] = {"values": na, "blocks": na // 32, "overflowed_blocks": n_over,
                   "q8_k128_nonfinite_flag": int(flags.item()),
                   "q8_1_gb_s": round(na * (4 + 36 / 32) / m1 / 1e6, 1),
                   "q8_k128_gb_s": round(na * (4 + 140 / 128) / mk / 1e6, 1)}
    return out


def run_moe(iqq, dev, peak_ops: float, p_mean: float, experts: int = 256):
    """DeepSeek-shaped MoE expert tensors (gate/up 2048x7168, down 7168x2048, N(0, 0.015) with
    outliers, a per-expert imatrix with 5% of the columns boosted x100), streamed expert by
    expert: each expert's three tensors are drawn on the device (not timed), then quantized
    (Q4_0, imatrix weighted) in one launch of the batched entry, timed with CUDA events, and
    again in three single launches (the per-shape rates); their round trip is accumulated.
    Returns Gelem/s and the ALU-model fraction of the batched launches, the single launches'
    rate, per-shape rates and the weighted RMSE over all experts."""
    import torch
    from post_weight_quantization_rowwise_b200 import synth
    ts = synth.moe_experts(experts)
    acc = torch.zeros(4, dtype=torch.float64, device=dev)
    ms = {"gate": 0.0, "up": 0.0, "down": 0.0}
    vals = {"gate": 0, "up": 0, "down": 0}
    batched_ms = 0.0
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2: the tensors start in HBM
    for e in range(experts):
        trio = ts[3 * e:3 * e + 3]
        xs = [t.weights(device=dev) for t in trio]
        qs = [t.qw(device=dev) for t in trio]
        bl = [torch.empty(t.rows * (t.cols // 32) * 18, dtype=torch.uint8, device=dev) for t in trio]
        # the expert's three tensors in one launch of the batched entry
        probs = iqq.q4_0_problems(list(zip(xs, qs, bl)))
        flush.zero_()
        ev[0].record()
        iqq.iqq_quantize_q4_0_w_batch(probs)
        ev[1].record()
        torch.cuda.synchronize()
        batched_ms += ev[0].elapsed_time(ev[1])
        # and one launch per tensor, for the rates of the three shapes
        flush.zero_()
        ev[0].record()
        for i, (t, x, q, b) in enumerate(zip(trio, xs, qs, bl)):
            iqq.iqq_quantize_q4_0_w(x, q, b)
            ev[i + 1].record()
        for t, x, q, b in zip(trio, xs, qs, bl):
            iqq.iqq_weighted_rmse(x, b, q, acc)
        torch.cuda.synchronize()
        for i, t in enumerate(trio):
            kind = t.name.rsplit(".", 1)[1]
            ms[kind] += ev[i].elapsed_time(ev[i + 1])
            vals[kind] += t.numel
    a = acc.cpu().tolist()
    n = sum(vals.values())
    total_ms = sum(ms.values())
    ops = Q4_0_OPS_BASE + Q4_0_OPS_PER_PASS * p_mean
    return {"experts": experts, "values": n, "quantize_ms": round(batched_ms, 3),
            "gelem_s": round(n / batched_ms / 1e6, 3),
            "frac": round(n * ops / (batched_ms / 1e3) / 1e12 / peak_ops, 4),
            "entry": "iqq_quantize_q4_0_w_batch, one launch per expert (its gate, up and down)",
            "single_launches": {"quantize_ms": round(total_ms, 3), "gelem_s": round(n / total_ms / 1e6, 3)},
            "per_shape_gelem_s": {k: round(vals[k] / ms[k] / 1e6, 3) for k in ms},
            "wrmse": math.sqrt(a[0] / a[1]), "maxerr": a[3],
            "timing": "CUDA events around each expert's batched launch and around its three single "
                      "launches; tensors drawn, then L2 flushed (256 MB write), before each"}


def run_e2e(iqq, w: Workload, dev, steps: int, layers: int, barrier=None):
    """The same step through the public API from pinned host buffers, every byte of input
    crossing PCIe each step: per tensor H2D of x (binary32: the layer set's outliers are not
    bf16 values) and qw, its two kernels, D2H of the blocks; H2D of the activations,
    Q8_K_128, D2H of its blocks and of the accumulator.
    The copies run on their own streams (host to device, device to host) with two device
    staging slots, so tensor i + 1 uploads and tensor i - 1 downloads while tensor i
    computes; events order every reuse of a slot or buffer.  ``barrier`` (several ranks)
    runs after the warm-up pass so that every rank's timed copies share the host at once.
    Returns (line, seconds per step, values per step)."""
    import torch
    n = 7 * layers

    def pinned_copy(t, dtype=None):
        h = torch.empty(t.shape, dtype=dtype or t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    host_x = [pinned_copy(w.x[i]) for i in range(n)]
    host_qw = [pinned_copy(w.qw[i]) for i in range(n)]
    host_b = [torch.empty(w.blocks[i].numel(), dtype=torch.uint8, pin_memory=True) for i in range(n)]
    host_act = pinned_copy(w.act)
    host_q8 = torch.empty(w.q8.numel(), dtype=torch.uint8, pin_memory=True)
    host_acc = torch.empty(4, dtype=torch.float64, pin_memory=True)
    big = max(t.numel for t in w.tensors[:n])
    xd = [torch.empty(big, dtype=torch.float32, device=dev) for _ in range(2)]
    qd = [torch.empty(max(t.cols for t in w.tensors[:n]), dtype=torch.float32, device=dev) for _ in range(2)]
    cs = torch.cuda.current_stream()
    up, dn = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    act_up, q8_done, acc_read = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
    downloaded = [torch.cuda.Event() for _ in range(n)]
    h2d = sum(h.numel() * 4 for h in host_x) + sum(h.numel() * 4 for h in host_qw) + host_act.numel() * 4
    d2h = sum(h.numel() for h in host_b) + host_q8.numel() + 32

    def one():
        cs.wait_event(acc_read)  # the previous step's accumulator has been read
        w.acc.zero_()
        for i in range(n):
            t, k = w.tensors[i], i % 2
            xv, qv = xd[k][:t.numel].view(t.rows, t.cols), qd[k][:t.cols]
            with torch.cuda.stream(up):
                up.wait_event(computed[k])  # slot k is free once tensor i - 2 is done
                xv.copy_(host_x[i], non_blocking=True)
                qv.copy_(host_qw[i], non_blocking=True)
                uploaded[k].record(up)
            cs.wait_event(uploaded[k])
            cs.wait_event(downloaded[i])  # the previous step's copy of these blocks is done
            iqq.iqq_quantize_q4_0_w(xv, qv, w.blocks[i], stream=cs)
            iqq.iqq_dequant_rmse_qx(4, xv, w.blocks[i], qv, w.y[:t.numel].view(t.rows, t.cols), w.acc,
                                    stream=cs)
            computed[k].record(cs)
            with torch.cuda.stream(dn):
                dn.wait_event(computed[k])
                host_b[i].copy_(w.blocks[i], non_blocking=True)
                downloaded[i].record(dn)
        with torch.cuda.stream(up):
            up.wait_event(q8_done)  # the previous step's Q8_K_128 has read w.act
            w.act.copy_(host_act, non_blocking=True)
            act_up.record(up)
        cs.wait_event(act_up)
        iqq.iqq_quantize_q8_k128(w.act, w.q8, stream=cs)
        q8_done.record(cs)
        with torch.cuda.stream(dn):
            dn.wait_event(q8_done)
            host_q8.copy_(w.q8, non_blocking=True)
            host_acc.copy_(w.acc, non_blocking=True)
            acc_read.record(dn)

    one()
    torch.cuda.synchronize()
    if barrier is not None:
        barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    end_up, end_dn = torch.cuda.Event(), torch.cuda.Event()
    e0.record(cs)
    up.wait_event(e0)
    dn.wait_event(e0)
    for _ in range(steps):
        one()
    end_up.record(up)
    end_dn.record(dn)
    cs.wait_event(end_up)
    cs.wait_event(end_dn)
    e1.record(cs)
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3 / steps
    elems = sum(t.numel for t in w.tensors[:n]) + w.act.numel()
    return ({"value": elems / sec / 1e9, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
             "d2h_bytes_per_step": int(d2h), "layers": layers,
             "h2d_gb_s": round(h2d / sec / 1e9, 1), "x_dtype": "f32",
            "overlap": "copies on two streams beside the kernels"},
            sec, elems)


def main_ours(args):
    import torch
    import torch.distributed as dist

    import post_weight_quantization_rowwise_b200 as iqq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    # the oracle pool is spawned before this process touches the GPU
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    w = Workload(dev, rank, args.layers)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        run_step(iqq, w, stream)
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(1.0)  # nvidia-smi's first sample arrives after start-up
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark()
    launches = 0
    for s in range(args.steps):
        launches += run_step(iqq, w, stream, ev[s])
    torch.cuda.synchronize()
    clk = clocks.stop()
    phase = [0.0] * 3
    for s in range(args.steps):
        for p in range(3):
            phase[p] += ev[s][p].elapsed_time(ev[s][p + 1])
    total_ms = ev[0][0].elapsed_time(ev[-1][3])
    from post_weight_quantization_rowwise_b200 import replicas
    times = replicas.max_over_ranks([total_ms] + phase, device=dev)  # the slowest rank
    if world > 1:
        dist.barrier()
    total_ms, phase = times[0], times[1:]
    # the round trip of every tensor quantized by every rank (the job's statistics)
    rt = replicas.job_rmse(w.acc, w.q4_elems, device=dev)

    gemv = None
    if not args.no_gemv:
        gemv = run_gemv_phase(iqq, w, dev)
    extras = None
    if rank == 0 and not args.no_extras:
        pk0 = peaks()
        peak0 = B200_SMS * FP32_LANES_PER_SM * pk0["sm_max_mhz"] * 1e6 / 1e12
        extras = run_extras(iqq, dev, cpu[3] if cpu else 1.1, peak0, pk0["hbm_gbs"])
        extras["moe"] = run_moe(iqq, dev, peak0, cpu[3] if cpu else 1.1, args.moe_experts)

    e2e = None
    if not args.no_e2e:
        # every rank streams its own share of the layers (the pinned host memory of the
        # whole job stays that of one rank at --e2e-layers); the slowest rank's time counts
        e2e_layers = max(1, args.e2e_layers // world)
        e2e, e2e_sec, e2e_elems = run_e2e(iqq, w, dev, max(1, min(args.steps, 3)), e2e_layers,
                                          barrier=dist.barrier if world > 1 else None)
        if world > 1:
            e2e_sec = replicas.max_over_ranks([e2e_sec], device=dev)[0]
            elems, h2d, d2h = replicas.sum_over_ranks(
                [e2e_elems, e2e["h2d_bytes_per_step"], e2e["d2h_bytes_per_step"]], device=dev)
            e2e.update(value=elems / e2e_sec / 1e9, h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h),
                       h2d_gb_s=round(h2d / e2e_sec / 1e9, 1), layers_per_rank=e2e_layers, ranks=world)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    K = args.steps
    ms_step = total_ms / K
    elems = (w.q4_elems + w.q8_elems) * world
    value = elems / (ms_step / 1e3) / 1e9
    pk = peaks()
    p_mean = cpu[3] if cpu else 1.1
    q4_ms = phase[0] / K
    n_q4 = q4_launches(w)
    ops_per_value = Q4_0_OPS_BASE + Q4_0_OPS_PER_PASS * p_mean
    achieved = w.q4_elems * ops_per_value / (q4_ms / 1e3) / 1e12          # Tops/s
    peak_ops = B200_SMS * FP32_LANES_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e12
    drm_gbs = w.q4_elems * DEQ_RMSE_BYTES_PER_VALUE / (phase[1] / K / 1e3) / 1e9
    q8_gbs = w.q8_elems * Q8_BYTES_PER_VALUE / (phase[2] / K / 1e3) / 1e9
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; no model weights or calibration data)",
        "config": {"workload": WORKLOAD, "layers": args.layers, "tensors": len(w.tensors),
                   "q4_0_values": w.q4_elems, "q8_k128_values": w.q8_elems,
                   "l2": "inputs 25.9 GB >> 126 MB L2, no flush", "parallelism": f"dp{world} (a layer set per rank, no data-path collective)"},
        "roofline": {"bound": "alu", "kernel": "q4_0_w_kernel<float, false>",
                     "achieved": round(achieved, 3),
                     "peak": round(peak_ops, 3), "unit": "Tops/s",
                     "frac": round(achieved / peak_ops, 4),
                     "traffic": (None if Q4_0_DRAM_BYTES_PER_VALUE is None else
                                 round(Q4_0_DRAM_BYTES_PER_VALUE * w.q4_elems / n_q4)),
                     "traffic_unit": "bytes per launch (ncu dram read+write, scaled by values)",
                     "ops_per_value": round(ops_per_value, 2), "greedy_passes_mean": round(p_mean, 4),
                     "avg_launch_ms": round(q4_ms / n_q4, 5),
                     "peak_basis": f"{B200_SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x "
                                   f"{pk['sm_max_mhz']:.0f} MHz ({pk['source']} max clock)"},
        "kernels": {
            "q4_0_w": {"ms": round(q4_ms, 4), "gelem_s": round(w.q4_elems / (q4_ms / 1e3) / 1e9, 3)},
            "dequant_rmse_q4_0": {"ms": round(phase[1] / K, 4), "gb_s": round(drm_gbs, 1),
                                  "hbm_frac": round(drm_gbs / pk["hbm_gbs"], 4),
                                  "kernel": "weighted_rmse_batch_kernel (48 tensors a launch) writing y",
                                  "bytes_per_value": DEQ_RMSE_BYTES_PER_VALUE,
                                  "wrmse": rt["wrmse"], "rmse": rt["rmse"], "maxerr": rt["maxerr"],
                                  "round_trip_values": rt["values"],
                                  "round_trip_scope": "all ranks' tensors (accumulators reduced over ranks)"},
            "q8_k128": {"ms": round(phase[2] / K, 4), "gb_s": round(q8_gbs, 1),
                        "hbm_frac": round(q8_gbs / pk["hbm_gbs"], 4),
                        "gelem_s": round(w.q8_elems / (phase[2] / K / 1e3) / 1e9, 3)},
        },
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
    }
    if extras is not None:
        out["extras"] = extras
    if gemv is not None:
        gms, gbytes, glarge, gbms = gemv
        ggbs = gbytes / (gms / 1e3) / 1e9
        for v in glarge.values():
            if isinstance(v, dict):
                v["hbm_frac"] = round(v["gb_s"] / pk["hbm_gbs"], 4)
        out["kernels"]["gemv_q4_0_q8_k128"] = {
            "ms": round(gms, 4), "gb_s": round(ggbs, 1), "hbm_frac": round(ggbs / pk["hbm_gbs"], 4),
            "tokens": 1, "launches": len(w.tensors), "timing": "one CUDA graph of the launches, "
            "outside the step", "bytes": int(gbytes), "large_matrix": glarge,
            "batched": {"ms": round(gbms, 4), "gb_s": round(gbytes / gbms / 1e6, 1),
                        "hbm_frac": round(gbytes / gbms / 1e6 / pk["hbm_gbs"], 4),
                        "launches": (len(w.tensors) + 63) // 64,
                        "entry": "iqq_gemv_q4_0_q8_k128_batch, one call for the layer set"}}
    if cpu:
        out["cpu_baseline"] = {"value": round(cpu[0], 5), "unit": UNIT, "cores": cpu[1],
                               "kind": "oracle", "sample": cpu[2]}
    print(json.dumps(out), flush=True)


def main_reference(args):
    """The oracle (plain single-threaded C, one process per host core) as the reference arm:
    every step is one pass over the fixed sample of the workload (ORACLE_SAMPLE_Q4_VALUES),
    timed as in the cpu_baseline leg."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import multiprocessing as mp
    vals, secs, cores, sample = [], [], None, None
    ncores = os.cpu_count() or 1
    with mp.get_context("spawn").Pool(ncores) as pool:
        for i in range(args.warmup + args.steps):
            v, cores, sample, _, step_s = oracle_sample(ncores, pool)
            if i >= args.warmup:
                vals.append(v)
                secs.append(step_s)
    step = statistics.median(secs)
    value = statistics.median(vals)
    out = {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step * 1e3, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic (seeded; no model weights or calibration data)",
           "config": {"workload": WORKLOAD, "layers": args.layers,
                      "step": "one pass of the oracle over the fixed sample below", "sample": sample},
           "impl": "reference",
           "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def profile_case(name: str):
    """Fixed cases for ncu captures (one GPU, a few launches): gemv_11008x4096 (25 MB of
    blocks), gemv_16384x53248 (490 MB, the large matrix of the GEMV phase) and
    moe_experts_4 (the first 4 MoE experts' gate, up and down tensors quantized once each,
    12 launches in expert order, 704 MB of x)."""
    import torch
    import post_weight_quantization_rowwise_b200 as iqq
    if name == "moe_experts_4":
        from post_weight_quantization_rowwise_b200 import synth
        ts = synth.moe_experts(4)
        xs = [t.weights(device="cuda") for t in ts]
        qs = [t.qw(device="cuda") for t in ts]
        bl = [torch.empty(t.rows * (t.cols // 32) * 18, dtype=torch.uint8, device="cuda") for t in ts]
        for t, x, q, b in zip(ts, xs, qs, bl):
            iqq.iqq_quantize_q4_0_w(x, q, b)
        torch.cuda.synchronize()
        print("ok", " ".join(f"{t.name}:{t.rows}x{t.cols}" for t in ts))
        return
    shapes = {"gemv_11008x4096": (11008, 4096), "gemv_16384x53248": (16384, 53248)}
    if name not in shapes:
        raise SystemExit(f"unknown profile case {name}")
    torch.manual_seed(0)
    n_out, k = shapes[name]
    w = torch.randint(0, 256, (n_out * (k // 32) * 18,), dtype=torch.uint8, device="cuda")
    w.view(-1, 18)[:, 1] &= 0x3B  # finite binary16 scales
    a1 = iqq.quantize_q8_k128(torch.randn(1, k, device="cuda"))
    a8 = iqq.quantize_q8_k128(torch.randn(8, k, device="cuda"))
    y1 = torch.empty(1, n_out, device="cuda")
    y8 = torch.empty(8, n_out, device="cuda")
    for _ in range(4):
        iqq.iqq_gemv_q4_0_q8_k128(w, a1, y1, k)
    iqq.iqq_gemv_q4_0_q8_k128(w, a8, y8, k)
    torch.cuda.synchronize()
    print("ok", float(y1.abs().sum()), float(y8.abs().sum()))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--e2e-layers", type=int, default=32)
    ap.add_argument("--moe-experts", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-gemv", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--profile-case", default=None, help="run one small ncu case and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        main_reference(args)
    else:
        main_ours(args)


if __name__ == "__main__":
    main()
