"""The C-ABI library loads without a GPU, exports every function iqq.h declares, and
rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "iqq.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(iqq_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    import post_weight_quantization_rowwise_b200 as m
    return m._lib


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("iqq_quantize_q4_0_w", "iqq_quantize_q8_k128", "iqq_dequant_q4_0",
              "iqq_weighted_rmse", "iqq_quantize_q8_1", "iqq_status_string",
              "iqq_quantize_qx_0_w", "iqq_dequant_qx_0", "iqq_gemv_q4_0_q8_k128",
              "iqq_weighted_rmse_qx", "iqq_quantize_qx_0_w_ws", "iqq_quantize_qx_0_w_workspace_bytes",
              "iqq_quantize_qx_0_w_static", "iqq_gemv_q4_0_q8_k128_batch",
              "iqq_quantize_qx_0_w_ex", "iqq_dequant_rmse_qx", "iqq_quantize_qx_0_w_bf16",
              "iqq_dequant_rmse_qx_bf16", "iqq_quantize_q4_0_w_direct", "iqq_quantize_q4_0_w_batch",
              "iqq_dequant_rmse_q4_0_batch"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n


def test_exported_symbols_are_c_linkage():
    import post_weight_quantization_rowwise_b200 as m
    raw = ctypes.CDLL(m.LIB_PATH)
    for n in _declared_functions():
        ctypes.cast(getattr(raw, n), ctypes.c_void_p)  # resolvable unmangled


def test_host_validation_without_gpu(lib):
    V = ctypes.c_void_p
    # shape: n_per_row not a multiple of 32 / 128, negative sizes
    assert lib.iqq_quantize_q4_0_w(None, None, None, 4, 33, 0, 0, None, None) == 2
    assert lib.iqq_quantize_q4_0_w(None, None, None, -1, 32, 0, 0, None, None) == 2
    assert lib.iqq_quantize_q8_k128(None, None, 2, 96, None, None) == 2
    assert lib.iqq_dequant_q4_0(None, None, 2, 48, None) == 2
    assert lib.iqq_weighted_rmse(None, None, None, 2, 32, -1, None, None) == 2
    # overflowing byte counts
    assert lib.iqq_quantize_q4_0_w(V(16), None, V(16), 1 << 40, 1 << 30, 0, 0, None, None) == 2
    # empty input is a no-op even with NULL pointers
    assert lib.iqq_quantize_q4_0_w(None, None, None, 0, 64, 0, 0, None, None) == 0
    assert lib.iqq_quantize_q8_k128(None, None, 5, 0, None, None) == 0
    # NULL pointers
    assert lib.iqq_quantize_q4_0_w(None, None, None, 4, 32, 0, 0, None, None) == 1
    assert lib.iqq_weighted_rmse(V(16), V(16), None, 2, 32, 0, None, None) == 1
    # alignment
    assert lib.iqq_quantize_q4_0_w(V(8), None, V(16), 4, 32, 0, 0, None, None) == 3
    assert lib.iqq_quantize_q4_0_w(V(16), V(20), V(16), 4, 32, 0, 0, None, None) == 3
    assert lib.iqq_quantize_q4_0_w(V(16), None, V(17), 4, 32, 0, 0, None, None) == 3
    assert lib.iqq_quantize_q8_k128(V(16), V(18), 1, 128, None, None) == 3
    assert lib.iqq_quantize_q8_1(V(16), V(16), 1, 48, None, None, None) == 2
    assert lib.iqq_quantize_q8_1(None, V(16), 1, 32, None, None, None) == 1
    assert lib.iqq_quantize_q8_1(V(16), V(16), 1, 32, V(12), None, None) == 3
    assert lib.iqq_dequant_q4_0(V(16), V(8), 1, 32, None) == 3
    assert lib.iqq_weighted_rmse(V(16), V(16), None, 1, 32, 0, V(4), None) == 3
    # enumerated argument
    assert lib.iqq_quantize_q4_0_w(V(16), None, V(16), 4, 32, 0, 6, None, None) == 5
    assert lib.iqq_quantize_q4_0_w(V(16), None, V(16), 4, 32, 0, -1, None, None) == 5
    # the generic block formats: bits checked first, then as for Q4_0
    for bits in (3, 7, 0, 16):
        assert lib.iqq_quantize_qx_0_w(bits, V(16), None, V(16), 4, 32, 0, 0, None, None) == 5
        assert lib.iqq_dequant_qx_0(bits, V(16), V(16), 1, 32, None) == 5
    for bits in (4, 5, 6, 8):
        assert lib.iqq_quantize_qx_0_w(bits, None, None, None, 4, 33, 0, 0, None, None) == 2
        assert lib.iqq_quantize_qx_0_w(bits, None, None, None, 0, 64, 0, 0, None, None) == 0
        assert lib.iqq_quantize_qx_0_w(bits, V(16), None, V(17), 4, 32, 0, 0, None, None) == 3
        assert lib.iqq_quantize_qx_0_w(bits, V(16), None, V(16), 4, 32, 0, 6, None, None) == 5
        assert lib.iqq_dequant_qx_0(bits, V(16), V(16), 2, 48, None) == 2
        assert lib.iqq_dequant_qx_0(bits, None, V(16), 1, 32, None) == 1
        assert lib.iqq_dequant_qx_0(bits, V(16), V(8), 1, 32, None) == 3
    for bits in (3, 7):
        assert lib.iqq_weighted_rmse_qx(bits, V(16), V(16), None, 1, 32, 0, V(16), None) == 5
    for bits in (4, 5, 6, 8):
        assert lib.iqq_weighted_rmse_qx(bits, V(16), V(16), None, 2, 48, 0, V(16), None) == 2
        assert lib.iqq_weighted_rmse_qx(bits, V(16), V(16), None, 1, 32, 0, V(4), None) == 3
        assert lib.iqq_weighted_rmse_qx(bits, None, None, None, 0, 32, 0, None, None) == 0
    # workspace variant: size rule, and the workspace checks
    WB = lib.iqq_quantize_qx_0_w_workspace_bytes
    WB.restype = ctypes.c_size_t
    WB.argtypes = [ctypes.c_int64, ctypes.c_int64]
    assert WB(10, 4096) == 0 and WB(10, 12288) == 0       # 3 CTAs per row: fused
    assert WB(10, 12320) == 256 and WB(100, 53248) == 512  # 4 and 13 CTAs per row
    assert WB(0, 53248) == 0
    Q = lib.iqq_quantize_qx_0_w_ws
    assert Q(4, V(16), None, V(16), 2, 53248, 0, 0, None, 0, None, None) == 1
    assert Q(4, V(16), None, V(16), 2, 53248, 0, 0, V(16), 8, None, None) == 2
    assert Q(4, V(16), None, V(16), 2, 53248, 0, 0, V(8), 256, None, None) == 3
    assert Q(7, V(16), None, V(16), 2, 53248, 0, 0, V(16), 256, None, None) == 5
    assert Q(4, V(16), None, V(16), 2, 4096, 0, 9, None, 0, None, None) == 5  # no workspace needed
    assert Q(4, None, None, None, 0, 4096, 0, 0, None, 0, None, None) == 0
    S = lib.iqq_quantize_qx_0_w_static
    assert S(3, V(16), None, V(16), 2, 53248, 0, 0, None, None) == 5
    assert S(4, V(16), None, V(16), 2, 53248 + 16, 0, 0, None, None) == 2
    assert S(4, None, None, V(16), 2, 53248, 0, 0, None, None) == 1
    assert S(4, V(16), None, V(16), 2, 53248, 0, 7, None, None) == 5
    assert S(4, V(8), None, V(16), 2, 53248, 0, 0, None, None) == 3
    assert S(4, None, None, None, 0, 53248, 0, 0, None, None) == 0
    # the batched product: checks of every problem before anything is enqueued
    import post_weight_quantization_rowwise_b200 as m
    B = lib.iqq_gemv_q4_0_q8_k128_batch
    ok = m.GemvProblem(16, 16, 16, 4, 128, 1)
    bad = m.GemvProblem(16, 16, 16, 4, 96, 1)
    arr = (m.GemvProblem * 3)(ok, bad, ok)
    assert B(ctypes.cast(arr, V), 3, None, None) == 2
    assert B(None, 2, None, None) == 1
    assert B(ctypes.cast(arr, V), -1, None, None) == 2
    assert B(None, 0, None, None) == 0
    empty = (m.GemvProblem * 2)(m.GemvProblem(0, 0, 0, 0, 128, 1), m.GemvProblem(16, 16, 16, 4, 128, 0))
    assert B(ctypes.cast(empty, V), 2, None, None) == 0
    unaligned = (m.GemvProblem * 1)(m.GemvProblem(8, 16, 16, 4, 128, 1))
    assert B(ctypes.cast(unaligned, V), 1, None, None) == 3
    # the batched Q4_0 quantizer: checks of every tensor before anything is enqueued
    QB4 = lib.iqq_quantize_q4_0_w_batch
    QB4.argtypes = [V, ctypes.c_int64, ctypes.c_int, ctypes.c_float, V, V]
    good = m.Q4_0Problem(16, None, 16, 2, 4096, 0)
    arr = (m.Q4_0Problem * 3)(good, m.Q4_0Problem(16, None, 16, 2, 4097, 0), good)
    assert QB4(ctypes.cast(arr, V), 3, 0, 1.0, None, None) == 2
    assert QB4(None, 2, 0, 1.0, None, None) == 1
    assert QB4(ctypes.cast(arr, V), -1, 0, 1.0, None, None) == 2
    assert QB4(None, 0, 0, 1.0, None, None) == 0
    one = (m.Q4_0Problem * 1)(good)
    assert QB4(ctypes.cast(one, V), 1, 6, 1.0, None, None) == 5             # weight mode
    assert QB4(ctypes.cast(one, V), 1, 0, float("nan"), None, None) == 5    # fudge
    assert QB4(ctypes.cast(one, V), 1, 0, 1.0, V(2), None) == 3             # flags alignment
    for prob, code in ((m.Q4_0Problem(8, None, 16, 2, 4096, 0), 3),         # x alignment
                       (m.Q4_0Problem(16, 8, 16, 2, 4096, 0), 3),           # qw alignment
                       (m.Q4_0Problem(16, None, 1, 2, 4096, 0), 3),         # out alignment
                       (m.Q4_0Problem(None, None, 16, 2, 4096, 0), 1),
                       (m.Q4_0Problem(16, None, None, 2, 4096, 0), 1),
                       (m.Q4_0Problem(16, None, 16, 2, 4096, -1), 2),
                       (m.Q4_0Problem(16, None, 16, 2, 1 << 27, 0), 2),     # 2^22 blocks a row
                       (m.Q4_0Problem(None, None, None, 0, 4096, 0), 0)):   # empty: nothing to do
        two = (m.Q4_0Problem * 2)(prob, prob)
        assert QB4(ctypes.cast(two, V), 2, 0, 1.0, None, None) == code, (prob.x, prob.qw, prob.out, code)
    # the batched dequantization + round trip: the same, with the accumulator shared
    RB = lib.iqq_dequant_rmse_q4_0_batch
    RB.argtypes = [V, ctypes.c_int64, V, V]
    P = m.DequantRmseProblem
    bad = P(16, 16, None, 16, 2, 4097, 0)
    arr = (P * 2)(bad, P(16, 16, None, 16, 2, 4096, 0))
    assert RB(ctypes.cast(arr, V), 2, V(16), None) == 2
    assert RB(None, 2, V(16), None) == 1
    assert RB(ctypes.cast(arr, V), -1, V(16), None) == 2
    assert RB(None, 0, None, None) == 0
    one = (P * 1)(P(16, 16, None, 16, 2, 4096, 0))
    assert RB(ctypes.cast(one, V), 1, V(12), None) == 3                      # acc alignment
    assert RB(ctypes.cast(one, V), 1, None, None) == 1                       # acc NULL
    for prob, code in ((P(8, 16, None, 16, 2, 4096, 0), 3),                  # x alignment
                       (P(16, 1, None, 16, 2, 4096, 0), 3),                  # blocks alignment
                       (P(16, 16, 8, 16, 2, 4096, 0), 3),                    # qw alignment
                       (P(16, 16, None, 8, 2, 4096, 0), 3),                  # y alignment
                       (P(None, 16, None, 16, 2, 4096, 0), 1),
                       (P(16, None, None, 16, 2, 4096, 0), 1),
                       (P(16, 16, None, 16, 2, 4096, -1), 2),
                       (P(16, 16, None, 16, -2, 4096, 0), 2),
                       (P(16, 16, None, 16, 2, 4100, 0), 2),
                       (P(None, None, None, None, 0, 4096, 0), 0)):          # empty: nothing to do
        two = (P * 2)(prob, prob)
        assert RB(ctypes.cast(two, V), 2, V(16), None) == code, (prob.x, prob.blocks, prob.qw, prob.y, code)
    X = lib.iqq_quantize_qx_0_w_ex
    assert X(4, V(16), None, V(16), 2, 4096, 0, 0, 1.0, None, 0, None, V(12), None, None) == 3   # d_acc alignment
    assert X(4, V(16), None, V(16), 2, 4096, 0, 0, 1.0, None, 0, V(8), None, None, None) == 3    # y alignment
    assert X(4, V(16), None, V(16), 2, 53248, 0, 0, 1.0, V(16), 8, None, None, None, None) == 2  # workspace too small
    assert X(9, V(16), None, V(16), 2, 4096, 0, 0, 1.0, None, 0, None, None, None, None) == 5
    assert X(4, V(16), None, V(16), 2, 4096, 0, 0, -1.0, None, 0, None, None, None, None) == 5   # fudge < 0
    assert X(4, V(16), None, V(16), 2, 4096, 0, 0, float("nan"), None, 0, None, None, None, None) == 5
    assert X(4, None, None, None, 0, 4096, 0, 0, 1.0, None, 0, None, None, None, None) == 0
    DR = lib.iqq_dequant_rmse_qx
    assert DR(4, V(16), V(16), None, 1, 32, 0, None, V(16), None) == 1
    assert DR(4, V(16), V(16), None, 1, 32, 0, V(8), V(16), None) == 3
    assert DR(7, V(16), V(16), None, 1, 32, 0, V(16), V(16), None) == 5
    assert DR(4, V(16), V(16), None, 1, 48, 0, V(16), V(16), None) == 2
    # bf16 weights: the same checks (x 16-byte aligned), the optional workspace
    QB = lib.iqq_quantize_qx_0_w_bf16
    assert QB(7, V(16), None, V(16), 2, 4096, 0, 0, None, 0, None, None) == 5
    assert QB(4, V(16), None, V(16), 2, 4097, 0, 0, None, 0, None, None) == 2
    assert QB(4, None, None, V(16), 2, 4096, 0, 0, None, 0, None, None) == 1
    assert QB(4, V(8), None, V(16), 2, 4096, 0, 0, None, 0, None, None) == 3
    assert QB(4, V(16), None, V(16), 2, 4096, 0, 6, None, 0, None, None) == 5
    assert QB(4, V(16), None, V(16), 2, 53248, 0, 0, V(16), 8, None, None) == 2   # workspace too small
    assert QB(4, V(16), None, V(16), 2, 53248, 0, 0, V(8), 256, None, None) == 3
    assert QB(4, None, None, None, 0, 4096, 0, 0, None, 0, None, None) == 0
    DB = lib.iqq_dequant_rmse_qx_bf16
    assert DB(4, V(16), V(16), None, 1, 32, 0, None, V(16), None) == 1
    assert DB(4, V(8), V(16), None, 1, 32, 0, V(16), V(16), None) == 3
    assert DB(7, V(16), V(16), None, 1, 32, 0, V(16), V(16), None) == 5
    assert DB(4, V(16), V(16), None, 1, 48, 0, V(16), V(16), None) == 2
    # Q4_0 x Q8_K_128 matrix-vector product
    G = lib.iqq_gemv_q4_0_q8_k128
    assert G(V(16), V(16), V(16), 4, 96, 1, None, None) == 2          # k not a multiple of 128
    assert G(V(16), V(16), V(16), 4, 65536 + 128, 1, None, None) == 2  # k above the maximum
    assert G(V(16), V(16), V(16), -1, 128, 1, None, None) == 2
    assert G(None, None, None, 0, 128, 1, None, None) == 0             # empty
    assert G(None, None, None, 4, 128, 0, None, None) == 0
    assert G(V(16), V(16), None, 4, 128, 1, None, None) == 1
    assert G(None, V(16), V(16), 4, 128, 1, None, None) == 1
    assert G(V(8), V(16), V(16), 4, 128, 1, None, None) == 3           # weights 16-byte aligned
    assert G(V(16), V(18), V(16), 4, 128, 1, None, None) == 3
    assert G(V(16), V(16), V(18), 4, 128, 1, None, None) == 3


def test_status_strings(lib):
    for s in range(6):
        assert lib.iqq_status_string(s)
    assert lib.iqq_last_cuda_error() == 0


def test_python_binding_requires_cuda_tensors():
    import torch
    import post_weight_quantization_rowwise_b200 as m
    with pytest.raises(ValueError):
        m.quantize_q4_0_w(torch.zeros(2, 64))


def test_binding_rejects_an_imatrix_the_kernels_would_overrun():
    """The binding checks qw's size against the rows it covers before any CUDA call: one
    imatrix row per rows_per_qw rows (ceil), or one shared row."""
    import torch
    import post_weight_quantization_rowwise_b200 as m
    assert m.qw_rows_needed(6, 3) == 2 and m.qw_rows_needed(7, 3) == 3
    assert m.qw_rows_needed(5, 0) == 1 and m.qw_rows_needed(0, 4) == 0
    with pytest.raises(ValueError):
        m.qw_rows_needed(4, -1)
    n = 64
    m._check_qw(None, 6, n, 3)                                  # qw = 1: nothing to read
    m._check_qw(torch.zeros(2 * n), 6, n, 3)                    # exactly enough
    with pytest.raises(ValueError):
        m._check_qw(torch.zeros(n), 6, n, 3)                    # one row for two groups
    with pytest.raises(ValueError):
        m._check_qw(torch.zeros(2 * n), 7, n, 3)                # the third group's row is missing
    with pytest.raises(ValueError):
        m._check_qw(torch.zeros(n - 1), 1, n, 0)                # a short shared row
    with pytest.raises(ValueError):
        m._check_qw(torch.zeros(n), 1, n, 0, device=torch.device("meta"))  # another device


def test_importing_the_package_maps_no_library():
    """Only a call loads libiqq.so: the input generators can be imported without it."""
    import subprocess
    import sys
    code = ("import post_weight_quantization_rowwise_b200 as m\n"
            "from post_weight_quantization_rowwise_b200 import synth\n"
            "assert not m.loaded()\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libiqq.so' not in maps, 'mapped at import'\n"
            "m.version()\n"
            "assert m.loaded() and 'libiqq.so' in open('/proc/self/maps').read()\n")
    subprocess.run([sys.executable, "-c", code], check=True, cwd=ROOT)
