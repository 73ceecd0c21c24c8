"""CPU oracle for the imatrix-weighted Q4_0 / Q8_K_128 path (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference leg may import this package.  The product path (the CUDA
library and its binding) never imports it.

Thin ctypes wrappers over ``liboracle.so`` (built from ``iqq_oracle.c`` by
``oracle/build.py``); every computation happens in the C file, whose header
cites the page and section each function follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_f32p = ctypes.POINTER(ctypes.c_float)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i8p = ctypes.POINTER(ctypes.c_int8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64

Q4_0_BYTES = 18
Q8_K128_BYTES = 140


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_fp16_from_float.restype = ctypes.c_uint16
        L.oracle_fp16_from_float.argtypes = [ctypes.c_float]
        L.oracle_fp16_to_float.restype = ctypes.c_float
        L.oracle_fp16_to_float.argtypes = [ctypes.c_uint16]
        L.oracle_row_sigma2.restype = ctypes.c_float
        L.oracle_row_sigma2.argtypes = [_f32p, _i64]
        L.oracle_block_weights.restype = None
        L.oracle_block_weights.argtypes = [_f32p, _f32p, ctypes.c_int, ctypes.c_float,
                                           ctypes.c_int, _f32p]
        L.oracle_q4_0_block_search.restype = ctypes.c_float
        L.oracle_q4_0_block_search.argtypes = [ctypes.c_int, _f32p, _f32p, _i8p, _i8p, _i32p]
        L.oracle_quantize_q4_0_w.restype = ctypes.c_int
        L.oracle_quantize_q4_0_w.argtypes = [_f32p, _f32p, _u8p, _i64, _i64, _i64, ctypes.c_int,
                                             _u32p, _i32p]
        L.oracle_dequant_q4_0.restype = ctypes.c_int
        L.oracle_dequant_q4_0.argtypes = [_u8p, _f32p, _i64, _i64]
        L.oracle_weighted_rmse.restype = ctypes.c_int
        L.oracle_weighted_rmse.argtypes = [_f32p, _u8p, _f32p, _i64, _i64, _i64, _f64p]
        L.oracle_fp16_from_float_array.restype = None
        L.oracle_fp16_from_float_array.argtypes = [_f32p, ctypes.POINTER(ctypes.c_uint16), _i64]
        L.oracle_fp16_to_float_array.restype = None
        L.oracle_fp16_to_float_array.argtypes = [ctypes.POINTER(ctypes.c_uint16), _f32p, _i64]
        L.oracle_qx_block_search.restype = ctypes.c_float
        L.oracle_qx_block_search.argtypes = [ctypes.c_int, ctypes.c_int, _f32p, _f32p, _i8p, _i8p, _i32p]
        L.oracle_quantize_qx_0_w.restype = ctypes.c_int
        L.oracle_quantize_qx_0_w.argtypes = [ctypes.c_int, _f32p, _f32p, _u8p, _i64, _i64, _i64,
                                             ctypes.c_int, _u32p]
        L.oracle_quantize_qx_0_w_f.restype = ctypes.c_int
        L.oracle_quantize_qx_0_w_f.argtypes = [ctypes.c_int, _f32p, _f32p, _u8p, _i64, _i64, _i64,
                                               ctypes.c_int, ctypes.c_float, _u32p]
        L.oracle_dequant_qx_0.restype = ctypes.c_int
        L.oracle_dequant_qx_0.argtypes = [ctypes.c_int, _u8p, _f32p, _i64, _i64]
        L.oracle_qx_block_bytes.restype = ctypes.c_int
        L.oracle_qx_block_bytes.argtypes = [ctypes.c_int]
        L.oracle_quantize_q8_1.restype = ctypes.c_int64
        L.oracle_quantize_q8_1.argtypes = [_f32p, _u8p, _i64, _i64]
        L.oracle_quantize_q8_k128.restype = ctypes.c_int
        L.oracle_quantize_q8_k128.argtypes = [_f32p, _u8p, _i64, _i64, _u32p]
        L.oracle_q4_0_block_bytes.argtypes = []
        L.oracle_q8_k128_block_bytes.argtypes = []
        L.oracle_weighted_rmse_qx.restype = ctypes.c_int
        L.oracle_weighted_rmse_qx.argtypes = [ctypes.c_int, _f32p, _u8p, _f32p, _i64, _i64, _i64, _f64p]
        L.oracle_dot_q4_0_q8_k128.restype = ctypes.c_int
        L.oracle_dot_q4_0_q8_k128.argtypes = [_u8p, _u8p, _f64p, _f64p, _i64, _i64, _i64]
        _LIB = L
    return _LIB


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def fp16_from_float(v: float) -> int:
    return int(lib().oracle_fp16_from_float(ctypes.c_float(v)))


def fp16_to_float(h: int) -> float:
    return float(lib().oracle_fp16_to_float(ctypes.c_uint16(h)))


def fp16_from_float_array(f):
    f = _f32(f)
    h = np.empty(f.shape, np.uint16)
    lib().oracle_fp16_from_float_array(_ptr(f, _f32p), _ptr(h, ctypes.POINTER(ctypes.c_uint16)),
                                       f.size)
    return h


def fp16_to_float_array(h):
    h = np.ascontiguousarray(h, dtype=np.uint16)
    f = np.empty(h.shape, np.float32)
    lib().oracle_fp16_to_float_array(_ptr(h, ctypes.POINTER(ctypes.c_uint16)), _ptr(f, _f32p),
                                     h.size)
    return f


def row_sigma2(x) -> float:
    x = _f32(x)
    return float(lib().oracle_row_sigma2(_ptr(x, _f32p), x.size))


def block_weights(xb, qwb, sigma2: float, weight_mode: int = 0):
    xb = _f32(xb)
    qwb = None if qwb is None else _f32(qwb)
    w = np.empty_like(xb)
    lib().oracle_block_weights(_ptr(xb, _f32p), _ptr(qwb, _f32p), xb.size,
                               ctypes.c_float(sigma2), weight_mode, _ptr(w, _f32p))
    return w


def block_search(xb, w):
    """Scale search of one block of length n <= 64.

    Returns (d, codes, sweep_codes, info) with info = [k_sweep, passes, fallback, 0].
    """
    xb = _f32(xb)
    w = _f32(w)
    n = xb.size
    L = np.zeros(n, np.int8)
    Ls = np.zeros(n, np.int8)
    info = np.zeros(4, np.int32)
    d = lib().oracle_q4_0_block_search(n, _ptr(xb, _f32p), _ptr(w, _f32p), _ptr(L, _i8p),
                                       _ptr(Ls, _i8p), _ptr(info, _i32p))
    return np.float32(d), L, Ls, info


NMAX = {4: 8, 5: 16, 6: 32, 8: 128}


def qx_block_bytes(bits: int) -> int:
    return int(lib().oracle_qx_block_bytes(bits))


def qx_block_search(xb, w, nmax: int):
    """Scale search of one block with codes in [-nmax, nmax-1]; as block_search."""
    xb = _f32(xb)
    w = _f32(w)
    n = xb.size
    L = np.zeros(n, np.int8)
    Ls = np.zeros(n, np.int8)
    info = np.zeros(4, np.int32)
    d = lib().oracle_qx_block_search(n, nmax, _ptr(xb, _f32p), _ptr(w, _f32p), _ptr(L, _i8p),
                                     _ptr(Ls, _i8p), _ptr(info, _i32p))
    return np.float32(d), L, Ls, info


def quantize_qx_0_w(bits: int, x, qw=None, rows_per_qw: int = 0, weight_mode: int = 0, fudge: float = 1.0):
    """Weighted quantization to the 32-value format with `bits` (4, 5, 6, 8); (blocks, flags).
    fudge scales the sigma2 term of the importance (weight modes 0, 4, 5)."""
    x = _f32(x)
    nrows, n = x.shape
    qw = None if qw is None else _f32(qw)
    bb = qx_block_bytes(bits)
    if bb < 0:
        raise ValueError("bits must be 4, 5, 6 or 8")
    out = np.zeros((nrows, (n // 32) * bb), np.uint8)
    flags = np.zeros(1, np.uint32)
    rc = lib().oracle_quantize_qx_0_w_f(bits, _ptr(x, _f32p), _ptr(qw, _f32p), _ptr(out, _u8p), nrows, n,
                                        rows_per_qw, weight_mode, ctypes.c_float(fudge), _ptr(flags, _u32p))
    if rc != 0:
        raise ValueError("oracle_quantize_qx_0_w: bad arguments")
    return out, int(flags[0])


def dequant_qx_0(bits: int, blocks, nrows: int, n_per_row: int):
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    y = np.empty((nrows, n_per_row), np.float32)
    rc = lib().oracle_dequant_qx_0(bits, _ptr(blocks, _u8p), _ptr(y, _f32p), nrows, n_per_row)
    if rc != 0:
        raise ValueError("oracle_dequant_qx_0: bad arguments")
    return y


def quantize_q4_0_w(x, qw=None, rows_per_qw: int = 0, weight_mode: int = 0,
                    want_passes: bool = False):
    """Quantize a [nrows, n_per_row] float32 matrix; returns (blocks uint8 [nrows, nb*18], flags[, passes])."""
    x = _f32(x)
    nrows, n = x.shape
    qw = None if qw is None else _f32(qw)
    out = np.zeros((nrows, (n // 32) * Q4_0_BYTES), np.uint8)
    flags = np.zeros(1, np.uint32)
    passes = np.zeros((nrows, n // 32), np.int32) if want_passes else None
    rc = lib().oracle_quantize_q4_0_w(_ptr(x, _f32p), _ptr(qw, _f32p), _ptr(out, _u8p), nrows, n,
                                      rows_per_qw, weight_mode, _ptr(flags, _u32p),
                                      _ptr(passes, _i32p))
    if rc != 0:
        raise ValueError("oracle_quantize_q4_0_w: bad shape")
    if want_passes:
        return out, int(flags[0]), passes
    return out, int(flags[0])


def dequant_q4_0(blocks, nrows: int, n_per_row: int):
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    y = np.empty((nrows, n_per_row), np.float32)
    rc = lib().oracle_dequant_q4_0(_ptr(blocks, _u8p), _ptr(y, _f32p), nrows, n_per_row)
    if rc != 0:
        raise ValueError("oracle_dequant_q4_0: bad shape")
    return y


def weighted_rmse(x, blocks, qw=None, rows_per_qw: int = 0, acc=None):
    """Returns the accumulator [sum qw e^2, sum qw, sum e^2, max|e|] (binary64)."""
    x = _f32(x)
    nrows, n = x.shape
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    qw = None if qw is None else _f32(qw)
    acc = np.zeros(4, np.float64) if acc is None else acc
    rc = lib().oracle_weighted_rmse(_ptr(x, _f32p), _ptr(blocks, _u8p), _ptr(qw, _f32p), nrows, n,
                                    rows_per_qw, _ptr(acc, _f64p))
    if rc != 0:
        raise ValueError("oracle_weighted_rmse: bad shape")
    return acc


def weighted_rmse_qx(bits: int, x, blocks, qw=None, rows_per_qw: int = 0, acc=None):
    """weighted_rmse for Q4_0/Q5_0/Q6_0/Q8_0 blocks (bits 4/5/6/8)."""
    x = _f32(x)
    nrows, n = x.shape
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    qw = None if qw is None else _f32(qw)
    acc = np.zeros(4, np.float64) if acc is None else acc
    rc = lib().oracle_weighted_rmse_qx(bits, _ptr(x, _f32p), _ptr(blocks, _u8p), _ptr(qw, _f32p), nrows,
                                       n, rows_per_qw, _ptr(acc, _f64p))
    if rc != 0:
        raise ValueError("oracle_weighted_rmse_qx: bad bits or shape")
    return acc


def quantize_q8_k128(x):
    """Quantize a [nrows, n_per_row] float32 matrix; returns (blocks uint8 [nrows, nb*140], flags)."""
    x = _f32(x)
    nrows, n = x.shape
    out = np.zeros((nrows, (n // 128) * Q8_K128_BYTES), np.uint8)
    flags = np.zeros(1, np.uint32)
    rc = lib().oracle_quantize_q8_k128(_ptr(x, _f32p), _ptr(out, _u8p), nrows, n,
                                       _ptr(flags, _u32p))
    if rc != 0:
        raise ValueError("oracle_quantize_q8_k128: bad shape")
    return out, int(flags[0])


Q8_1_BYTES = 36


def quantize_q8_1(x):
    """Q8_1 blocks of a [nrows, n_per_row] float32 matrix; returns (blocks uint8, overflow count)."""
    x = _f32(x)
    nrows, n = x.shape
    out = np.zeros((nrows, (n // 32) * Q8_1_BYTES), np.uint8)
    cnt = lib().oracle_quantize_q8_1(_ptr(x, _f32p), _ptr(out, _u8p), nrows, n)
    if cnt < 0:
        raise ValueError("oracle_quantize_q8_1: bad shape")
    return out, int(cnt)


def decode_q8_1(blocks, nrows: int, n_per_row: int):
    """Split Q8_1 bytes into (d uint16 [nrows, nb], s uint16 [nrows, nb], qs int8 [nrows, n])."""
    nb = n_per_row // 32
    b = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(nrows, nb, Q8_1_BYTES)
    d = b[:, :, 0:2].copy().view(np.uint16).reshape(nrows, nb)
    s = b[:, :, 2:4].copy().view(np.uint16).reshape(nrows, nb)
    qs = b[:, :, 4:36].copy().view(np.int8).reshape(nrows, n_per_row)
    return d, s, qs


def decode_q8_k128(blocks, nrows: int, n_per_row: int):
    """Split Q8_K_128 bytes into (d float32 [nrows, nb], qs int8 [nrows, n], bsums int16 [nrows, nb, 4])."""
    nb = n_per_row // 128
    b = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(nrows, nb, Q8_K128_BYTES)
    d = b[:, :, 0:4].copy().view(np.float32).reshape(nrows, nb)
    qs = b[:, :, 4:132].copy().view(np.int8).reshape(nrows, n_per_row)
    bs = b[:, :, 132:140].copy().view(np.int16).reshape(nrows, nb, 4)
    return d, qs, bs


def dot_q4_0_q8_k128(w_blocks, a_blocks, n_out: int, k: int, n_tok: int):
    """y[t, r] = dequant(W)[r] . dequant(A)[t] in binary64 (exact products, summed left
    to right), and the sum of |products| beside it.  Returns (y, absum), both float64
    [n_tok, n_out]."""
    w = np.ascontiguousarray(w_blocks, dtype=np.uint8)
    a = np.ascontiguousarray(a_blocks, dtype=np.uint8)
    if w.size < n_out * (k // 32) * Q4_0_BYTES or a.size < n_tok * (k // 128) * Q8_K128_BYTES:
        raise ValueError("dot_q4_0_q8_k128: buffers too small")
    y = np.empty((n_tok, n_out), np.float64)
    s = np.empty((n_tok, n_out), np.float64)
    if lib().oracle_dot_q4_0_q8_k128(_ptr(w, _u8p), _ptr(a, _u8p), _ptr(y, _f64p), _ptr(s, _f64p),
                                     n_out, k, n_tok) != 0:
        raise ValueError("dot_q4_0_q8_k128: k must be a multiple of 128")
    return y, s


def decode_q4_0(blocks, nrows: int, n_per_row: int):
    """Split Q4_0 bytes into (d16 uint16 [nrows, nb], codes int8 [nrows, n] in [-8, 7])."""
    nb = n_per_row // 32
    b = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(nrows, nb, Q4_0_BYTES)
    d16 = b[:, :, 0:2].copy().view(np.uint16).reshape(nrows, nb)
    qs = b[:, :, 2:18].astype(np.int16)
    codes = np.concatenate([(qs & 0xF) - 8, (qs >> 4) - 8], axis=2).astype(np.int8)
    return d16, codes.reshape(nrows, n_per_row)


__all__ = [n for n in dir() if not n.startswith("_")]
del os
