"""imatrix-weighted Q4_0 and Q8_K_128 quantization on B200 (sm_100a).

Thin Python binding over the C ABI in ``include/iqq.h`` (``libiqq.so`` in this
package).  The functions have the ABI's names; they only check and marshal
arguments (torch CUDA tensors -> device pointers, sizes and the current CUDA
stream).  Every step of the computation runs in the library's CUDA kernels:
there is no CPU or PyTorch fallback.

The library is loaded on the first call into it (importing the package alone,
for example for its ``synth`` input generators, maps no native code); that
first call raises ImportError if ``libiqq.so`` is missing or fails to load.

Block formats (little endian):
  Q4_0      18 bytes per 32 values: binary16 d | qs[16], qs[i] = (l[i]+8) | (l[i+16]+8) << 4
  Q8_K_128  140 bytes per 128 values: float d | int8 qs[128] | int16 bsums[4]
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libiqq.so")

Q4_0_BLOCK_VALUES = 32
Q4_0_BLOCK_BYTES = 18
Q8_K128_BLOCK_VALUES = 128
Q8_K128_BLOCK_BYTES = 140

FLAG_NONFINITE_INPUT = 1
FLAG_NEG_QW = 2
FLAG_SCALE_OVERFLOW = 4

STATUS = {0: "IQQ_OK", 1: "IQQ_ERR_NULL", 2: "IQQ_ERR_SHAPE", 3: "IQQ_ERR_ALIGN",
          4: "IQQ_ERR_CUDA", 5: "IQQ_ERR_ARG"}

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python post_weight_quantization_rowwise_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    sigs = {
        "iqq_quantize_q4_0_w": [_vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp, _vp],
        "iqq_quantize_q4_0_w_direct": [_vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp, _vp],
        "iqq_quantize_q4_0_w_batch": [_vp, _i64, ctypes.c_int, ctypes.c_float, _vp, _vp],
        "iqq_quantize_q8_k128": [_vp, _vp, _i64, _i64, _vp, _vp],
        "iqq_dequant_q4_0": [_vp, _vp, _i64, _i64, _vp],
        "iqq_quantize_q8_1": [_vp, _vp, _i64, _i64, _vp, _vp, _vp],
        "iqq_quantize_qx_0_w": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp, _vp],
        "iqq_dequant_qx_0": [ctypes.c_int, _vp, _vp, _i64, _i64, _vp],
        "iqq_gemv_q4_0_q8_k128": [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
        "iqq_gemv_q4_0_q8_k128_batch": [_vp, _i64, _vp, _vp],
        "iqq_weighted_rmse_qx": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
        "iqq_dequant_rmse_qx": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp],
        "iqq_quantize_qx_0_w_ws": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp,
                                   ctypes.c_size_t, _vp, _vp],
        "iqq_quantize_qx_0_w_static": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp, _vp],
        "iqq_quantize_qx_0_w_ex": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, ctypes.c_float,
                                   _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp],
        "iqq_weighted_rmse": [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
        "iqq_quantize_qx_0_w_bf16": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp,
                                     ctypes.c_size_t, _vp, _vp],
        "iqq_dequant_rmse_qx_bf16": [ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp],
        "iqq_dequant_rmse_q4_0_batch": [_vp, _i64, _vp, _vp],
    }
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.iqq_status_string.argtypes = [ctypes.c_int]
    lib.iqq_status_string.restype = ctypes.c_char_p
    lib.iqq_last_cuda_error.argtypes = []
    lib.iqq_last_cuda_error.restype = ctypes.c_int
    lib.iqq_version.argtypes = []
    lib.iqq_version.restype = ctypes.c_char_p
    lib.iqq_quantize_qx_0_w_workspace_bytes.restype = ctypes.c_size_t
    lib.iqq_quantize_qx_0_w_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
    return lib


class _LazyLib:
    """libiqq.so, loaded on first use (ImportError when missing: no fallback exists)."""

    _handle = None

    def __getattr__(self, name):
        if _LazyLib._handle is None:
            _LazyLib._handle = _load()
        return getattr(_LazyLib._handle, name)


_lib = _LazyLib()


def loaded() -> bool:
    """True once libiqq.so has been loaded into this process."""
    return _LazyLib._handle is not None


class IQQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib.iqq_status_string(status).decode()
        extra = ""
        if status == 4:
            extra = f" (cudaError {_lib.iqq_last_cuda_error()})"
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}{extra}")
        self.status = status


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise IQQError(fn, status)


def version() -> str:
    return _lib.iqq_version().decode()


def status_string(status: int) -> str:
    return _lib.iqq_status_string(status).decode()


# ----------------------------------------------------------------------------
# tensor marshalling (torch is used for memory and streams only)
# ----------------------------------------------------------------------------

def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(name, t, dtype=None):
    import torch
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def qw_rows_needed(nrows: int, rows_per_qw: int) -> int:
    """imatrix rows an operation over nrows rows reads: one per rows_per_qw rows
    (ceil), or one shared row when rows_per_qw is 0."""
    if rows_per_qw < 0:
        raise ValueError("rows_per_qw must be >= 0")
    if nrows <= 0:
        return 0
    return -(-nrows // rows_per_qw) if rows_per_qw > 0 else 1


def _check_qw(qw, nrows: int, n_per_row: int, rows_per_qw: int, device=None) -> None:
    """Rejects an imatrix the kernels would read past: qw must hold
    qw_rows_needed(nrows, rows_per_qw) * n_per_row values (None: qw = 1) and live on
    the device of the data it weights."""
    need = qw_rows_needed(nrows, rows_per_qw) * n_per_row
    if qw is None:
        return
    if qw.numel() < need:
        raise ValueError(f"qw holds {qw.numel()} values; {nrows} rows of {n_per_row} with "
                         f"rows_per_qw={rows_per_qw} read {need}")
    if device is not None and qw.device != device:
        raise ValueError(f"qw is on {qw.device}, the data on {device}")


def _same_device(x, **others) -> None:
    for name, t in others.items():
        if t is not None and t.device != x.device:
            raise ValueError(f"{name} is on {t.device}, x on {x.device}")


def _shape2(x):
    if x.dim() != 2:
        raise ValueError("x must be 2-D [nrows, n_per_row]")
    return int(x.shape[0]), int(x.shape[1])


def q4_0_nbytes(nrows: int, n_per_row: int) -> int:
    return nrows * (n_per_row // Q4_0_BLOCK_VALUES) * Q4_0_BLOCK_BYTES


def q8_k128_nbytes(nrows: int, n_per_row: int) -> int:
    return nrows * (n_per_row // Q8_K128_BLOCK_VALUES) * Q8_K128_BLOCK_BYTES


# ----------------------------------------------------------------------------
# the four entry points
# ----------------------------------------------------------------------------

def iqq_quantize_q4_0_w(x, qw, out, rows_per_qw: int = 0, weight_mode: int = 0, flags=None,
                        stream=None):
    """Q4_0 blocks of x [nrows, n_per_row] float32 into out (uint8, q4_0_nbytes)."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, out=out, flags=flags)
    if out.numel() < q4_0_nbytes(nrows, n):
        raise ValueError("out is too small")
    _check("iqq_quantize_q4_0_w",
           _lib.iqq_quantize_q4_0_w(_ptr(x), _ptr(qw), _ptr(out), nrows, n, rows_per_qw,
                                    weight_mode, _ptr(flags), _stream(stream)))
    return out


def iqq_quantize_q4_0_w_direct(x, qw, out, rows_per_qw: int = 0, weight_mode: int = 0, flags=None,
                               stream=None):
    """iqq_quantize_q4_0_w by the direct sweep (every candidate's exact sums): the same bytes
    and flags, kept to cross-check the default path."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, out=out, flags=flags)
    if out.numel() < q4_0_nbytes(nrows, n):
        raise ValueError("out is too small")
    _check("iqq_quantize_q4_0_w_direct",
           _lib.iqq_quantize_q4_0_w_direct(_ptr(x), _ptr(qw), _ptr(out), nrows, n, rows_per_qw,
                                           weight_mode, _ptr(flags), _stream(stream)))
    return out


class Q4_0Problem(ctypes.Structure):
    """iqq_q4_0_problem."""
    _fields_ = [("x", ctypes.c_void_p), ("qw", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("nrows", ctypes.c_int64), ("n_per_row", ctypes.c_int64), ("rows_per_qw", ctypes.c_int64)]


def q4_0_problems(items):
    """A ctypes array of iqq_q4_0_problem from (x, qw, out) or (x, qw, out, rows_per_qw) tuples
    of CUDA tensors on one device (qw may be None), checked here; the tensors must outlive
    every call that uses the array."""
    import torch
    arr = (Q4_0Problem * len(items))()
    dev = None
    for i, it in enumerate(items):
        x, qw, out = it[0], it[1], it[2]
        rpq = it[3] if len(it) > 3 else 0
        _need_cuda("x", x, torch.float32)
        _need_cuda("qw", qw, torch.float32)
        _need_cuda("out", out, torch.uint8)
        nrows, n = _shape2(x)
        _check_qw(qw, nrows, n, rpq, x.device)
        _same_device(x, out=out)
        if dev is not None and x.device != dev:
            raise ValueError(f"problem {i}: every tensor must be on the same device")
        dev = x.device
        if out.numel() < q4_0_nbytes(nrows, n):
            raise ValueError(f"problem {i}: out is too small")
        arr[i] = Q4_0Problem(x.data_ptr(), qw.data_ptr() if qw is not None else None, out.data_ptr(), nrows, n,
                             rpq)
    return arr


def iqq_quantize_q4_0_w_batch(problems, weight_mode: int = 0, flags=None, stream=None, fudge: float = 1.0):
    """iqq_quantize_q4_0_w for every tensor of a q4_0_problems() array, in launches of up to 64
    tensors."""
    import torch
    _need_cuda("flags", flags, torch.int32)
    _check("iqq_quantize_q4_0_w_batch",
           _lib.iqq_quantize_q4_0_w_batch(ctypes.cast(problems, ctypes.c_void_p), len(problems), weight_mode,
                                          fudge, _ptr(flags), _stream(stream)))


QX_0_BLOCK_BYTES = {4: 18, 5: 22, 6: 26, 8: 34}


def iqq_quantize_qx_0_w(bits, x, qw, out, rows_per_qw: int = 0, weight_mode: int = 0, flags=None,
                        stream=None):
    """Weighted Q4_0/Q5_0/Q6_0/Q8_0 (bits 4/5/6/8) blocks of x into out (uint8)."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, out=out, flags=flags)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if out.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits]:
        raise ValueError("out is too small")
    _check("iqq_quantize_qx_0_w",
           _lib.iqq_quantize_qx_0_w(bits, _ptr(x), _ptr(qw), _ptr(out), nrows, n, rows_per_qw,
                                    weight_mode, _ptr(flags), _stream(stream)))
    return out


def iqq_dequant_qx_0(bits, blocks, y, stream=None):
    import torch
    _need_cuda("blocks", blocks, torch.uint8)
    _need_cuda("y", y, torch.float32)
    nrows, n = _shape2(y)
    _same_device(y, blocks=blocks)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if blocks.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits]:
        raise ValueError("blocks is too small")
    _check("iqq_dequant_qx_0", _lib.iqq_dequant_qx_0(bits, _ptr(blocks), _ptr(y), nrows, n, _stream(stream)))
    return y


def qx_0_w_workspace_bytes(nrows: int, n_per_row: int) -> int:
    """Device workspace iqq_quantize_qx_0_w_ws needs (0: none)."""
    return int(_lib.iqq_quantize_qx_0_w_workspace_bytes(nrows, n_per_row))


def iqq_quantize_qx_0_w_ws(bits, x, qw, out, workspace, rows_per_qw: int = 0, weight_mode: int = 0,
                           flags=None, stream=None):
    """iqq_quantize_qx_0_w with a device workspace (uint8 tensor of at least
    qx_0_w_workspace_bytes bytes, or None when that is 0) for rows spanning many CTAs."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("workspace", workspace, torch.uint8)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, out=out, flags=flags, workspace=workspace)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if out.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits]:
        raise ValueError("out is too small")
    nbytes = 0 if workspace is None else workspace.numel()
    _check("iqq_quantize_qx_0_w_ws",
           _lib.iqq_quantize_qx_0_w_ws(bits, _ptr(x), _ptr(qw), _ptr(out), nrows, n, rows_per_qw, weight_mode,
                                       _ptr(workspace), nbytes, _ptr(flags), _stream(stream)))
    return out


def iqq_quantize_qx_0_w_bf16(bits, x, qw, out, rows_per_qw: int = 0, weight_mode: int = 0, workspace=None,
                             flags=None, stream=None):
    """iqq_quantize_qx_0_w for bf16 x [nrows, n_per_row] (widened exactly in the kernel: the
    blocks equal those of the binary32 tensor); optional workspace as for _ws."""
    import torch
    _need_cuda("x", x, torch.bfloat16)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("workspace", workspace, torch.uint8)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, out=out, flags=flags, workspace=workspace)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if out.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits]:
        raise ValueError("out is too small")
    nbytes = 0 if workspace is None else workspace.numel()
    _check("iqq_quantize_qx_0_w_bf16",
           _lib.iqq_quantize_qx_0_w_bf16(bits, _ptr(x), _ptr(qw), _ptr(out), nrows, n, rows_per_qw, weight_mode,
                                         _ptr(workspace), nbytes, _ptr(flags), _stream(stream)))
    return out


def iqq_quantize_q8_k128(x, out, flags=None, stream=None):
    """Q8_K_128 blocks of x [nrows, n_per_row] float32 into out (uint8, q8_k128_nbytes)."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _same_device(x, out=out, flags=flags)
    if out.numel() < q8_k128_nbytes(nrows, n):
        raise ValueError("out is too small")
    _check("iqq_quantize_q8_k128",
           _lib.iqq_quantize_q8_k128(_ptr(x), _ptr(out), nrows, n, _ptr(flags), _stream(stream)))
    return out


def iqq_quantize_q8_1(x, out, overflow=None, flags=None, stream=None):
    """Q8_1 blocks (36 bytes per 32 values) of x; adds the count of blocks whose fp16
    sum overflowed to `overflow` (int64 CUDA tensor of one element) when given."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("overflow", overflow, torch.int64)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _same_device(x, out=out, overflow=overflow, flags=flags)
    if out.numel() < nrows * (n // 32) * 36:
        raise ValueError("out is too small")
    _check("iqq_quantize_q8_1",
           _lib.iqq_quantize_q8_1(_ptr(x), _ptr(out), nrows, n, _ptr(overflow), _ptr(flags),
                                  _stream(stream)))
    return out


def iqq_dequant_q4_0(blocks, y, stream=None):
    """y [nrows, n_per_row] float32 from the Q4_0 blocks."""
    import torch
    _need_cuda("blocks", blocks, torch.uint8)
    _need_cuda("y", y, torch.float32)
    nrows, n = _shape2(y)
    _same_device(y, blocks=blocks)
    if blocks.numel() < q4_0_nbytes(nrows, n):
        raise ValueError("blocks is too small")
    _check("iqq_dequant_q4_0", _lib.iqq_dequant_q4_0(_ptr(blocks), _ptr(y), nrows, n, _stream(stream)))
    return y


def iqq_gemv_q4_0_q8_k128(w_blocks, a_blocks, y, k: int, flags=None, stream=None):
    """y [n_tok, n_out] float32 = dequant(W) . dequant(A) per (token, row) for Q4_0 rows W
    (n_out rows of k/32 blocks) and Q8_K_128 rows A (n_tok rows of k/128 blocks)."""
    import torch
    _need_cuda("w_blocks", w_blocks, torch.uint8)
    _need_cuda("a_blocks", a_blocks, torch.uint8)
    _need_cuda("y", y, torch.float32)
    _need_cuda("flags", flags, torch.int32)
    n_tok, n_out = _shape2(y)
    _same_device(y, w_blocks=w_blocks, a_blocks=a_blocks, flags=flags)
    if w_blocks.numel() < q4_0_nbytes(n_out, k):
        raise ValueError("w_blocks is too small")
    if a_blocks.numel() < q8_k128_nbytes(n_tok, k):
        raise ValueError("a_blocks is too small")
    _check("iqq_gemv_q4_0_q8_k128",
           _lib.iqq_gemv_q4_0_q8_k128(_ptr(w_blocks), _ptr(a_blocks), _ptr(y), n_out, k, n_tok,
                                      _ptr(flags), _stream(stream)))
    return y


class GemvProblem(ctypes.Structure):
    """iqq_gemv_problem."""
    _fields_ = [("w_blocks", ctypes.c_void_p), ("a_blocks", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("n_out", ctypes.c_int64), ("k", ctypes.c_int64), ("n_tok", ctypes.c_int64)]


def gemv_problems(items):
    """A ctypes array of iqq_gemv_problem from (w_blocks, a_blocks, y, k) tuples of CUDA
    tensors (y [n_tok, n_out]); the tensors must outlive every call that uses the array."""
    import torch
    arr = (GemvProblem * len(items))()
    for i, (w, a, y, k) in enumerate(items):
        _need_cuda("w_blocks", w, torch.uint8)
        _need_cuda("a_blocks", a, torch.uint8)
        _need_cuda("y", y, torch.float32)
        n_tok, n_out = _shape2(y)
        if w.numel() < q4_0_nbytes(n_out, k) or a.numel() < q8_k128_nbytes(n_tok, k):
            raise ValueError(f"problem {i}: blocks too small")
        arr[i] = GemvProblem(w.data_ptr(), a.data_ptr(), y.data_ptr(), n_out, k, n_tok)
    return arr


def iqq_gemv_q4_0_q8_k128_batch(problems, flags=None, stream=None):
    """Runs every problem of a gemv_problems() array."""
    import torch
    _need_cuda("flags", flags, torch.int32)
    _check("iqq_gemv_q4_0_q8_k128_batch",
           _lib.iqq_gemv_q4_0_q8_k128_batch(ctypes.cast(problems, ctypes.c_void_p), len(problems), _ptr(flags),
                                            _stream(stream)))


def iqq_weighted_rmse(x, blocks, qw, acc, rows_per_qw: int = 0, stream=None):
    """Adds {sum qw e^2, sum qw, sum e^2} to acc[0:3] and maxes acc[3] with max|e| (float64, CUDA)."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("blocks", blocks, torch.uint8)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("acc", acc, torch.float64)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, blocks=blocks, acc=acc)
    if blocks.numel() < q4_0_nbytes(nrows, n) or acc.numel() < 4:
        raise ValueError("blocks or acc is too small")
    _check("iqq_weighted_rmse",
           _lib.iqq_weighted_rmse(_ptr(x), _ptr(blocks), _ptr(qw), nrows, n, rows_per_qw, _ptr(acc),
                                  _stream(stream)))
    return acc


def iqq_dequant_rmse_qx(bits, x, blocks, qw, y, acc, rows_per_qw: int = 0, stream=None):
    """Dequantizes blocks into y and adds the round trip against x to acc, in one pass."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("blocks", blocks, torch.uint8)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("y", y, torch.float32)
    _need_cuda("acc", acc, torch.float64)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, blocks=blocks, y=y, acc=acc)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if blocks.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits] or acc.numel() < 4 or y.numel() < x.numel():
        raise ValueError("blocks, y or acc is too small")
    _check("iqq_dequant_rmse_qx",
           _lib.iqq_dequant_rmse_qx(bits, _ptr(x), _ptr(blocks), _ptr(qw), nrows, n, rows_per_qw, _ptr(y),
                                    _ptr(acc), _stream(stream)))
    return y


class DequantRmseProblem(ctypes.Structure):
    """iqq_dequant_rmse_problem."""
    _fields_ = [("x", ctypes.c_void_p), ("blocks", ctypes.c_void_p), ("qw", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("nrows", ctypes.c_int64), ("n_per_row", ctypes.c_int64),
                ("rows_per_qw", ctypes.c_int64)]


def dequant_rmse_problems(items):
    """A ctypes array of iqq_dequant_rmse_problem from (x, blocks, qw, y) or (x, blocks, qw, y,
    rows_per_qw) tuples of CUDA tensors on one device (qw and y may be None), checked here; the
    tensors must outlive every call that uses the array."""
    import torch
    arr = (DequantRmseProblem * len(items))()
    dev = None
    for i, it in enumerate(items):
        x, blocks, qw, y = it[0], it[1], it[2], it[3]
        rpq = it[4] if len(it) > 4 else 0
        _need_cuda("x", x, torch.float32)
        _need_cuda("blocks", blocks, torch.uint8)
        _need_cuda("qw", qw, torch.float32)
        _need_cuda("y", y, torch.float32)
        nrows, n = _shape2(x)
        _check_qw(qw, nrows, n, rpq, x.device)
        _same_device(x, blocks=blocks, y=y)
        if dev is not None and x.device != dev:
            raise ValueError(f"problem {i}: every tensor must be on the same device")
        dev = x.device
        if blocks.numel() < q4_0_nbytes(nrows, n) or (y is not None and y.numel() < x.numel()):
            raise ValueError(f"problem {i}: blocks or y is too small")
        arr[i] = DequantRmseProblem(x.data_ptr(), blocks.data_ptr(), qw.data_ptr() if qw is not None else None,
                                    y.data_ptr() if y is not None else None, nrows, n, rpq)
    return arr


def iqq_dequant_rmse_q4_0_batch(problems, acc, stream=None):
    """iqq_dequant_rmse_qx (bits 4) for every tensor of a dequant_rmse_problems() array, in
    launches of up to 48 tensors, all adding to acc."""
    import torch
    _need_cuda("acc", acc, torch.float64)
    if acc is None or acc.numel() < 4:
        raise ValueError("acc must hold 4 doubles")
    _check("iqq_dequant_rmse_q4_0_batch",
           _lib.iqq_dequant_rmse_q4_0_batch(ctypes.cast(problems, ctypes.c_void_p), len(problems), _ptr(acc),
                                            _stream(stream)))
    return acc


def iqq_dequant_rmse_qx_bf16(bits, x, blocks, qw, y, acc, rows_per_qw: int = 0, stream=None):
    """iqq_dequant_rmse_qx against bf16 x (widened exactly: y and acc equal those of the
    binary32 tensor)."""
    import torch
    _need_cuda("x", x, torch.bfloat16)
    _need_cuda("blocks", blocks, torch.uint8)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("y", y, torch.float32)
    _need_cuda("acc", acc, torch.float64)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, blocks=blocks, y=y, acc=acc)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if blocks.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits] or acc.numel() < 4 or y.numel() < x.numel():
        raise ValueError("blocks, y or acc is too small")
    _check("iqq_dequant_rmse_qx_bf16",
           _lib.iqq_dequant_rmse_qx_bf16(bits, _ptr(x), _ptr(blocks), _ptr(qw), nrows, n, rows_per_qw, _ptr(y),
                                         _ptr(acc), _stream(stream)))
    return y


def iqq_weighted_rmse_qx(bits, x, blocks, qw, acc, rows_per_qw: int = 0, stream=None):
    """iqq_weighted_rmse for Q4_0/Q5_0/Q6_0/Q8_0 blocks (bits 4/5/6/8)."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("blocks", blocks, torch.uint8)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("acc", acc, torch.float64)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, blocks=blocks, acc=acc)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if blocks.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits] or acc.numel() < 4:
        raise ValueError("blocks or acc is too small")
    _check("iqq_weighted_rmse_qx",
           _lib.iqq_weighted_rmse_qx(bits, _ptr(x), _ptr(blocks), _ptr(qw), nrows, n, rows_per_qw, _ptr(acc),
                                     _stream(stream)))
    return acc


# ----------------------------------------------------------------------------
# conveniences
# ----------------------------------------------------------------------------

def quantize_q4_0_w(x, qw=None, rows_per_qw: int = 0, weight_mode: int = 0, flags=None, stream=None):
    """Allocates and returns the Q4_0 blocks of x as a uint8 tensor [nrows, nb*18]."""
    import torch
    nrows, n = _shape2(x)
    out = torch.empty((nrows, (n // Q4_0_BLOCK_VALUES) * Q4_0_BLOCK_BYTES), dtype=torch.uint8,
                      device=x.device)
    return iqq_quantize_q4_0_w(x, qw, out, rows_per_qw, weight_mode, flags, stream)


def quantize_q8_k128(x, flags=None, stream=None):
    import torch
    nrows, n = _shape2(x)
    out = torch.empty((nrows, (n // Q8_K128_BLOCK_VALUES) * Q8_K128_BLOCK_BYTES), dtype=torch.uint8,
                      device=x.device)
    return iqq_quantize_q8_k128(x, out, flags, stream)


def quantize_qx_0_w(bits, x, qw=None, rows_per_qw: int = 0, weight_mode: int = 0, flags=None,
                    stream=None):
    import torch
    nrows, n = _shape2(x)
    out = torch.empty((nrows, (n // 32) * QX_0_BLOCK_BYTES[bits]), dtype=torch.uint8, device=x.device)
    return iqq_quantize_qx_0_w(bits, x, qw, out, rows_per_qw, weight_mode, flags, stream)


def iqq_quantize_qx_0_w_ex(bits, x, qw, out, workspace=None, acc=None, rows_per_qw: int = 0,
                           weight_mode: int = 0, flags=None, stream=None, y=None, fudge: float = 1.0):
    """The general quantizer: optional workspace (uint8), optional dequantized output y
    (float32 like x) and optional round-trip error accumulator acc (float64[4], zeroed by
    the caller)."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("workspace", workspace, torch.uint8)
    _need_cuda("acc", acc, torch.float64)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, out=out, flags=flags, workspace=workspace, y=y, acc=acc)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if out.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits]:
        raise ValueError("out is too small")
    if acc is not None and acc.numel() < 4:
        raise ValueError("acc needs 4 elements")
    _need_cuda("y", y, torch.float32)
    if y is not None and y.numel() < x.numel():
        raise ValueError("y is too small")
    nbytes = 0 if workspace is None else workspace.numel()
    _check("iqq_quantize_qx_0_w_ex",
           _lib.iqq_quantize_qx_0_w_ex(bits, _ptr(x), _ptr(qw), _ptr(out), nrows, n, rows_per_qw, weight_mode,
                                       fudge, _ptr(workspace), nbytes, _ptr(y), _ptr(acc), _ptr(flags),
                                       _stream(stream)))
    return out


def iqq_quantize_qx_0_w_static(bits, x, qw, out, rows_per_qw: int = 0, weight_mode: int = 0, flags=None,
                               stream=None):
    """iqq_quantize_qx_0_w_ws with the library's own static workspace (allocates nothing)."""
    import torch
    _need_cuda("x", x, torch.float32)
    _need_cuda("qw", qw, torch.float32)
    _need_cuda("out", out, torch.uint8)
    _need_cuda("flags", flags, torch.int32)
    nrows, n = _shape2(x)
    _check_qw(qw, nrows, n, rows_per_qw, x.device)
    _same_device(x, out=out, flags=flags)
    if bits not in QX_0_BLOCK_BYTES:
        raise ValueError("bits must be 4, 5, 6 or 8")
    if out.numel() < nrows * (n // 32) * QX_0_BLOCK_BYTES[bits]:
        raise ValueError("out is too small")
    _check("iqq_quantize_qx_0_w_static",
           _lib.iqq_quantize_qx_0_w_static(bits, _ptr(x), _ptr(qw), _ptr(out), nrows, n, rows_per_qw,
                                           weight_mode, _ptr(flags), _stream(stream)))
    return out


def quantize_qx_0_w_ws(bits, x, qw=None, rows_per_qw: int = 0, weight_mode: int = 0, flags=None,
                       stream=None):
    """quantize_qx_0_w through the workspace entry point (the workspace is allocated here)."""
    import torch
    nrows, n = _shape2(x)
    out = torch.empty((nrows, (n // 32) * QX_0_BLOCK_BYTES[bits]), dtype=torch.uint8, device=x.device)
    nb = qx_0_w_workspace_bytes(nrows, n)
    ws = torch.empty(nb, dtype=torch.uint8, device=x.device) if nb else None
    return iqq_quantize_qx_0_w_ws(bits, x, qw, out, ws, rows_per_qw, weight_mode, flags, stream)


def dequant_qx_0(bits, blocks, nrows: int, n_per_row: int, stream=None):
    import torch
    y = torch.empty((nrows, n_per_row), dtype=torch.float32, device=blocks.device)
    return iqq_dequant_qx_0(bits, blocks, y, stream)


def quantize_q8_1(x, overflow=None, flags=None, stream=None):
    import torch
    nrows, n = _shape2(x)
    out = torch.empty((nrows, (n // 32) * 36), dtype=torch.uint8, device=x.device)
    return iqq_quantize_q8_1(x, out, overflow, flags, stream)


def gemv_q4_0_q8_k128(w_blocks, a_blocks, n_out: int, k: int, n_tok: int, flags=None, stream=None):
    import torch
    y = torch.empty((n_tok, n_out), dtype=torch.float32, device=w_blocks.device)
    return iqq_gemv_q4_0_q8_k128(w_blocks, a_blocks, y, k, flags, stream)


def dequant_q4_0(blocks, nrows: int, n_per_row: int, stream=None):
    import torch
    y = torch.empty((nrows, n_per_row), dtype=torch.float32, device=blocks.device)
    return iqq_dequant_q4_0(blocks, y, stream)


def weighted_rmse_qx(bits, x, blocks, qw=None, rows_per_qw: int = 0, stream=None):
    """Returns the float64 accumulator [sum qw e^2, sum qw, sum e^2, max|e|] as a CUDA tensor."""
    import torch
    acc = torch.zeros(4, dtype=torch.float64, device=x.device)
    return iqq_weighted_rmse_qx(bits, x, blocks, qw, acc, rows_per_qw, stream)


def weighted_rmse(x, blocks, qw=None, rows_per_qw: int = 0, stream=None):
    """Returns the float64 accumulator [sum qw e^2, sum qw, sum e^2, max|e|] as a CUDA tensor."""
    import torch
    acc = torch.zeros(4, dtype=torch.float64, device=x.device)
    return iqq_weighted_rmse(x, blocks, qw, acc, rows_per_qw, stream)


__all__ = [n for n in dir() if n.startswith(("iqq_", "quantize", "dequant", "weighted", "Q", "FLAG",
                                             "q4", "q8", "version", "status", "IQQError", "LIB", "Dequant"))]
