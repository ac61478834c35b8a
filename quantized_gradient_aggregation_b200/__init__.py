"""quantized_gradient_aggregation_b200 -- Python binding of libqga.so.

Thin argument marshalling over the C ABI declared in ``include/qga.h``: every
function below has the name of the C entry point it calls, checks that torch
tensors have the dtype / device / size the entry point expects, passes their
data pointers and the current CUDA stream, and raises ``QGAError`` on a
non-zero status.  All computation happens in the library's CUDA kernels;
there is no CPU path.  Importing this package without a built ``libqga.so``
raises ImportError (build it with ``python
quantized_gradient_aggregation_b200/build.py``).

Methods: MXNet pull request #8342 "[WIP] 2bit gradient compression" (the 2-bit
threshold quantizer with residual, its record format and the receiver-side
merge) and the QSGD-MaxNorm b-bit scheme and its GlobalRandK sparsified
variant named in the gradient-compression README (vineeths96), as defined in
``include/qga.h``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqga.so")

QGA_OK = 0
QGA_ERR_INVALID_ARG = -1
QGA_ERR_UNSUPPORTED = -2
QGA_ERR_CUDA = -3
QGA_MAX_WORKERS = 64
QGA_DTYPE_F32 = 0
QGA_DTYPE_BF16 = 1

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libqga.so not found at {LIB_PATH}; build it with "
        "`python quantized_gradient_aggregation_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

_i64, _i32, _u64, _f32, _vp = ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p
_VPP = ctypes.POINTER(ctypes.c_void_p)


class qga_bucket_tensor(ctypes.Structure):
    _fields_ = [("grad", ctypes.c_void_p), ("residual", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("neg_threshold", ctypes.c_float), ("pos_threshold", ctypes.c_float)]


_SIGS = {
    "qga_strerror": (ctypes.c_char_p, [_i32]),
    "qga_last_cuda_error": (_i32, []),
    "qga_version": (_i32, []),
    "qga_2bit_words": (_i64, [_i64]),
    "qga_quantize_2bit": (_i32, [_vp, _vp, _vp, _i64, _f32, _f32, _vp]),
    "qga_quantize_2bit_bf16": (_i32, [_vp, _vp, _vp, _i64, _f32, _f32, _vp]),
    "qga_dequantize_2bit": (_i32, [_vp, _vp, _i64, _vp]),
    "qga_dequant_accumulate_2bit": (_i32, [_VPP, _i32, _vp, _i64, _vp]),
    "qga_2bit_bucket_words": (_i64, [ctypes.POINTER(ctypes.c_int64), _i32]),
    "qga_quantize_2bit_bucket": (_i32, [ctypes.POINTER(qga_bucket_tensor), _i32, _i32, _vp, _vp]),
    "qga_dequant_accumulate_2bit_bucket": (_i32, [_VPP, _i32, ctypes.POINTER(ctypes.c_int64), _i32,
                                                  _vp, _vp]),
    "qga_ternary_words": (_i64, [_i64]),
    "qga_quantize_ternary": (_i32, [_vp, _vp, _vp, _i64, _f32, _f32, _vp]),
    "qga_dequantize_ternary": (_i32, [_vp, _vp, _i64, _vp]),
    "qga_dequant_accumulate_ternary": (_i32, [_VPP, _i32, _vp, _i64, _vp]),
    "qga_quantize_merge_2bit": (_i32, [_vp, _vp, _i64, _f32, _f32, _VPP, _i32, _i32, _vp, _vp]),
    "qga_qsgd_words": (_i64, [_i64, _i32]),
    "qga_qsgd_mn_max": (_i32, [_VPP, _i32, _i64, _vp, _vp]),
    "qga_qsgd_mn_quantize": (_i32, [_vp, _vp, _i64, _i32, _u64, _vp, _vp]),
    "qga_qsgd_mn_dequant_accumulate": (_i32, [_VPP, _i32, _vp, _i64, _i32, _vp]),
    "qga_qsgd_mnts_words": (_i64, [_i64, _i32, _i32]),
    "qga_qsgd_mnts_quantize": (_i32, [_vp, _vp, _i64, _i32, _i32, _u64, _vp, _vp]),
    "qga_qsgd_mnts_dequant_accumulate": (_i32, [_VPP, _i32, _vp, _i64, _i32, _i32, _vp]),
    "qga_grandk_mn_max": (_i32, [_VPP, _i32, _i64, _vp, _i64, _vp, _vp]),
    "qga_grandk_mn_quantize": (_i32, [_vp, _i64, _vp, _i64, _vp, _i32, _u64, _vp, _vp]),
    "qga_grandk_mn_dequant_accumulate": (_i32, [_VPP, _i32, _vp, _i64, _vp, _i64, _i32, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def lib():
    """The loaded ctypes library (raw C ABI)."""
    return _lib


class QGAError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.qga_strerror(status).decode()
        if status == QGA_ERR_CUDA:
            msg += f" (cudaError {_lib.qga_last_cuda_error()})"
        super().__init__(f"{where}: status {status}: {msg}")
        self.status = status


def _check(status: int, where: str):
    if status != QGA_OK:
        raise QGAError(status, where)


def _stream(stream, device=None):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t, dtype, numel, what):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{what} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{what}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{what}: {t.numel()} elements, need {numel}")


def _ptr_array(tensors):
    arr = (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])
    return ctypes.cast(arr, _VPP), arr


# =============================================================== 2-bit ====

def qga_2bit_words(n: int) -> int:
    w = _lib.qga_2bit_words(n)
    if w < 0:
        raise QGAError(int(w), "qga_2bit_words")
    return int(w)


def create_2bit(grad: torch.Tensor) -> torch.Tensor:
    """create_2bit(grad) of the MXNet operator API: an uninitialised record
    buffer (uint32 words, held in an int32 tensor) sized for ``grad``."""
    return torch.empty(qga_2bit_words(grad.numel()), dtype=torch.int32, device=grad.device)


def qga_quantize_2bit(grad, residual, compr, neg_threshold, pos_threshold, stream=None):
    """Fused residual add + 2-bit code + residual update + pack (fp32 or bf16 grad)."""
    n = residual.numel()
    _need(residual, torch.float32, None, "residual")
    _need(compr, torch.int32, qga_2bit_words(n), "compr")
    if grad.dtype == torch.bfloat16:
        _need(grad, torch.bfloat16, n, "grad")
        fn, name = _lib.qga_quantize_2bit_bf16, "qga_quantize_2bit_bf16"
    else:
        _need(grad, torch.float32, n, "grad")
        fn, name = _lib.qga_quantize_2bit, "qga_quantize_2bit"
    if grad.numel() != n:
        raise ValueError("grad and residual sizes differ")
    _check(fn(_ptr(grad), _ptr(residual), _ptr(compr), n, float(neg_threshold),
              float(pos_threshold), _stream(stream, residual.device)), name)


def qga_dequantize_2bit(compr, out, stream=None):
    n = out.numel()
    _need(out, torch.float32, None, "out")
    _need(compr, torch.int32, qga_2bit_words(n), "compr")
    _check(_lib.qga_dequantize_2bit(_ptr(compr), _ptr(out), n, _stream(stream, out.device)),
           "qga_dequantize_2bit")


def qga_dequant_accumulate_2bit(comprs, out, stream=None):
    n = out.numel()
    _need(out, torch.float32, None, "out")
    words = qga_2bit_words(n)
    for i, c in enumerate(comprs):
        _need(c, torch.int32, words, f"compr[{i}]")
    arr, keep = _ptr_array(comprs)
    _check(_lib.qga_dequant_accumulate_2bit(arr, len(comprs), _ptr(out), n,
                                            _stream(stream, out.device)),
           "qga_dequant_accumulate_2bit")


def qga_quantize_merge_2bit(grad, residual, comprs, own, neg_threshold, pos_threshold, out,
                            stream=None):
    """The reducing worker's step: quantize worker ``own``'s gradient into
    ``comprs[own]`` and merge all records into ``out``, in one launch."""
    n = residual.numel()
    _need(grad, torch.float32, n, "grad")
    _need(residual, torch.float32, None, "residual")
    _need(out, torch.float32, n, "out")
    words = qga_2bit_words(n)
    for i, c in enumerate(comprs):
        _need(c, torch.int32, words, f"compr[{i}]")
    arr, keep = _ptr_array(comprs)
    _check(_lib.qga_quantize_merge_2bit(_ptr(grad), _ptr(residual), n, float(neg_threshold),
                                        float(pos_threshold), arr, len(comprs), int(own), _ptr(out),
                                        _stream(stream, residual.device)),
           "qga_quantize_merge_2bit")


def qga_2bit_bucket_words(sizes) -> int:
    arr = (ctypes.c_int64 * max(1, len(sizes)))(*sizes)
    w = _lib.qga_2bit_bucket_words(arr, len(sizes))
    if w < 0:
        raise QGAError(int(w), "qga_2bit_bucket_words")
    return int(w)


def make_bucket_table(grads, residuals, neg_thresholds, pos_thresholds):
    """Host descriptor table of a bucket (build once, reuse every step)."""
    T = len(residuals)
    table = (qga_bucket_tensor * max(1, T))()
    for t in range(T):
        n = residuals[t].numel()
        table[t] = qga_bucket_tensor(grads[t].data_ptr() if n else 0,
                                     residuals[t].data_ptr() if n else 0, n,
                                     float(neg_thresholds[t]), float(pos_thresholds[t]))
    return table


def qga_quantize_2bit_bucket(grads, residuals, neg_thresholds, pos_thresholds, compr,
                             stream=None, table=None):
    T = len(residuals)
    dtype = grads[0].dtype if T else torch.float32
    if dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"bucket grad dtype {dtype}")
    sizes = [r.numel() for r in residuals]
    _need(compr, torch.int32, qga_2bit_bucket_words(sizes), "compr")
    if table is None:
        for t in range(T):
            _need(residuals[t], torch.float32, None, f"residual[{t}]")
            _need(grads[t], dtype, sizes[t], f"grad[{t}]")
        table = make_bucket_table(grads, residuals, neg_thresholds, pos_thresholds)
    code = QGA_DTYPE_BF16 if dtype == torch.bfloat16 else QGA_DTYPE_F32
    _check(_lib.qga_quantize_2bit_bucket(table, T, code, _ptr(compr), _stream(stream, compr.device)),
           "qga_quantize_2bit_bucket")


def qga_dequant_accumulate_2bit_bucket(comprs, sizes, out, stream=None):
    words = qga_2bit_bucket_words(sizes)
    _need(out, torch.float32, sum(sizes), "out")
    for i, c in enumerate(comprs):
        _need(c, torch.int32, words, f"compr[{i}]")
    arr, keep = _ptr_array(comprs)
    n = (ctypes.c_int64 * max(1, len(sizes)))(*sizes)
    _check(_lib.qga_dequant_accumulate_2bit_bucket(arr, len(comprs), n, len(sizes), _ptr(out),
                                                   _stream(stream, out.device)),
           "qga_dequant_accumulate_2bit_bucket")


# ======================================================= dense ternary ====

def qga_ternary_words(n: int) -> int:
    w = _lib.qga_ternary_words(n)
    if w < 0:
        raise QGAError(int(w), "qga_ternary_words")
    return int(w)


def qga_quantize_ternary(grad, residual, compr, neg_threshold, pos_threshold, stream=None):
    """The 2-bit error-feedback step written as a dense (5 codes per byte) record."""
    n = residual.numel()
    _need(residual, torch.float32, None, "residual")
    _need(grad, torch.float32, n, "grad")
    _need(compr, torch.int32, qga_ternary_words(n), "compr")
    _check(_lib.qga_quantize_ternary(_ptr(grad), _ptr(residual), _ptr(compr), n,
                                     float(neg_threshold), float(pos_threshold),
                                     _stream(stream, residual.device)), "qga_quantize_ternary")


def qga_dequantize_ternary(compr, out, stream=None):
    n = out.numel()
    _need(out, torch.float32, None, "out")
    _need(compr, torch.int32, qga_ternary_words(n), "compr")
    _check(_lib.qga_dequantize_ternary(_ptr(compr), _ptr(out), n, _stream(stream, out.device)),
           "qga_dequantize_ternary")


def qga_dequant_accumulate_ternary(comprs, out, stream=None):
    n = out.numel()
    _need(out, torch.float32, None, "out")
    words = qga_ternary_words(n)
    for i, c in enumerate(comprs):
        _need(c, torch.int32, words, f"compr[{i}]")
    arr, keep = _ptr_array(comprs)
    _check(_lib.qga_dequant_accumulate_ternary(arr, len(comprs), _ptr(out), n,
                                               _stream(stream, out.device)),
           "qga_dequant_accumulate_ternary")


# ================================================================ QSGD ====

def qga_qsgd_words(n: int, bits: int) -> int:
    w = _lib.qga_qsgd_words(n, bits)
    if w < 0:
        raise QGAError(int(w), "qga_qsgd_words")
    return int(w)


def qga_qsgd_mn_max(grads, max_out, stream=None):
    n = grads[0].numel()
    for i, g in enumerate(grads):
        _need(g, torch.float32, n, f"grad[{i}]")
    _need(max_out, torch.float32, 1, "max_out")
    arr, keep = _ptr_array(grads)
    _check(_lib.qga_qsgd_mn_max(arr, len(grads), n, _ptr(max_out), _stream(stream, max_out.device)),
           "qga_qsgd_mn_max")


def qga_qsgd_mn_quantize(grad, compr, bits, seed, max_in, stream=None):
    n = grad.numel()
    _need(grad, torch.float32, None, "grad")
    _need(compr, torch.int32, qga_qsgd_words(n, bits), "compr")
    _need(max_in, torch.float32, 1, "max_in")
    _check(_lib.qga_qsgd_mn_quantize(_ptr(grad), _ptr(compr), n, bits, seed & ((1 << 64) - 1),
                                     _ptr(max_in), _stream(stream, grad.device)),
           "qga_qsgd_mn_quantize")


def qga_qsgd_mn_dequant_accumulate(comprs, out, bits, stream=None):
    n = out.numel()
    _need(out, torch.float32, None, "out")
    words = qga_qsgd_words(n, bits)
    for i, c in enumerate(comprs):
        _need(c, torch.int32, words, f"compr[{i}]")
    arr, keep = _ptr_array(comprs)
    _check(_lib.qga_qsgd_mn_dequant_accumulate(arr, len(comprs), _ptr(out), n, bits,
                                               _stream(stream, out.device)),
           "qga_qsgd_mn_dequant_accumulate")


# ======================================================= QSGD-MN-TS ====

def qga_qsgd_mnts_words(n: int, bits_coarse: int, bits_fine: int) -> int:
    w = _lib.qga_qsgd_mnts_words(n, bits_coarse, bits_fine)
    if w < 0:
        raise QGAError(int(w), "qga_qsgd_mnts_words")
    return int(w)


def qga_qsgd_mnts_quantize(grad, compr, bits_coarse, bits_fine, seed, max_in, stream=None):
    """Two-scale record of ``grad``: coarse levels on M (``max_in``), fine
    levels on M / s_coarse; see include/qga.h."""
    n = grad.numel()
    _need(grad, torch.float32, None, "grad")
    _need(compr, torch.int32, qga_qsgd_mnts_words(n, bits_coarse, bits_fine), "compr")
    _need(max_in, torch.float32, 1, "max_in")
    _check(_lib.qga_qsgd_mnts_quantize(_ptr(grad), _ptr(compr), n, bits_coarse, bits_fine,
                                       seed & ((1 << 64) - 1), _ptr(max_in),
                                       _stream(stream, grad.device)),
           "qga_qsgd_mnts_quantize")


def qga_qsgd_mnts_dequant_accumulate(comprs, out, bits_coarse, bits_fine, stream=None):
    n = out.numel()
    _need(out, torch.float32, None, "out")
    words = qga_qsgd_mnts_words(n, bits_coarse, bits_fine)
    for i, c in enumerate(comprs):
        _need(c, torch.int32, words, f"compr[{i}]")
    arr, keep = _ptr_array(comprs)
    _check(_lib.qga_qsgd_mnts_dequant_accumulate(arr, len(comprs), _ptr(out), n, bits_coarse,
                                                 bits_fine, _stream(stream, out.device)),
           "qga_qsgd_mnts_dequant_accumulate")


# ======================================================== GRandK-MN ====

def qga_grandk_mn_max(grads, index, max_out, stream=None):
    """M over the kept coordinates ``index`` (int64) of every worker's grad."""
    n = grads[0].numel()
    for i, g in enumerate(grads):
        _need(g, torch.float32, n, f"grad[{i}]")
    _need(index, torch.int64, None, "index")
    _need(max_out, torch.float32, 1, "max_out")
    arr, keep = _ptr_array(grads)
    _check(_lib.qga_grandk_mn_max(arr, len(grads), n, _ptr(index), index.numel(), _ptr(max_out),
                                  _stream(stream, max_out.device)),
           "qga_grandk_mn_max")


def qga_grandk_mn_quantize(grad, index, compr, bits, seed, max_in, stream=None):
    _need(grad, torch.float32, None, "grad")
    _need(index, torch.int64, None, "index")
    _need(compr, torch.int32, qga_qsgd_words(index.numel(), bits), "compr")
    _need(max_in, torch.float32, 1, "max_in")
    _check(_lib.qga_grandk_mn_quantize(_ptr(grad), grad.numel(), _ptr(index), index.numel(),
                                       _ptr(compr), bits, seed & ((1 << 64) - 1), _ptr(max_in),
                                       _stream(stream, grad.device)),
           "qga_grandk_mn_quantize")


def qga_grandk_mn_dequant_accumulate(comprs, index, out, bits, stream=None):
    """Merge into ``out`` (float32[n], overwritten): the scaled level sums at
    the kept coordinates, +0 elsewhere."""
    _need(out, torch.float32, None, "out")
    _need(index, torch.int64, None, "index")
    words = qga_qsgd_words(index.numel(), bits)
    for i, c in enumerate(comprs):
        _need(c, torch.int32, words, f"compr[{i}]")
    arr, keep = _ptr_array(comprs)
    _check(_lib.qga_grandk_mn_dequant_accumulate(arr, len(comprs), _ptr(index), index.numel(),
                                                 _ptr(out), out.numel(), bits,
                                                 _stream(stream, out.device)),
           "qga_grandk_mn_dequant_accumulate")
