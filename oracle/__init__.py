"""CPU oracle for quantized gradient aggregation -- TEST INFRASTRUCTURE ONLY.

The arithmetic lives in ``qga_oracle.c`` (plain single-threaded C, one
binary32 operation per step, no contraction).  This module compiles it with
gcc and exposes it to numpy through ctypes; it adds no arithmetic of its own
beyond allocating output arrays.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The GPU library never does: the two
implementations share no code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qga_oracle.c")
_LIB = os.path.join(_HERE, "libqga_oracle.so")
_CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libqga_oracle.so`` (if stale)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _ptr_array(arrays):
    arr = (ctypes.c_void_p * max(1, len(arrays)))()
    for i, a in enumerate(arrays):
        arr[i] = a.ctypes.data
    return arr


def lib(path: str | None = None):
    """Load (building if needed) the oracle shared library."""
    global _lib
    with _lock:
        if path is not None:
            return _declare(ctypes.CDLL(path))
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
        return _lib


def _declare(L):
    i64, f32, i32, u64, vp = (ctypes.c_int64, ctypes.c_float, ctypes.c_int,
                              ctypes.c_uint64, ctypes.c_void_p)
    L.oracle_2bit_words.restype = i64
    L.oracle_2bit_words.argtypes = [i64]
    L.oracle_quantize_2bit.argtypes = [vp, vp, vp, i64, f32, f32]
    L.oracle_quantize_2bit_bf16.argtypes = [vp, vp, vp, i64, f32, f32]
    L.oracle_dequantize_2bit.argtypes = [vp, vp, i64]
    L.oracle_dequant_accumulate_2bit.argtypes = [vp, i32, vp, i64]
    L.oracle_2bit_bucket_words.restype = i64
    L.oracle_2bit_bucket_words.argtypes = [vp, i32]
    L.oracle_quantize_2bit_bucket.argtypes = [vp, vp, vp, vp, vp, i32, i32, vp]
    L.oracle_dequant_accumulate_2bit_bucket.argtypes = [vp, i32, vp, i32, vp]
    L.oracle_philox4x32_10.argtypes = [vp, vp, vp]
    L.oracle_qsgd_mn_max.restype = f32
    L.oracle_qsgd_mn_max.argtypes = [vp, i32, i64]
    L.oracle_qsgd_uniform.restype = f32
    L.oracle_qsgd_uniform.argtypes = [u64, i64]
    L.oracle_qsgd_level.restype = ctypes.c_int32
    L.oracle_qsgd_level.argtypes = [f32, f32, i32, u64, i64]
    L.oracle_qsgd_words.restype = i64
    L.oracle_qsgd_words.argtypes = [i64, i32]
    L.oracle_qsgd_mn_quantize.argtypes = [vp, vp, i64, i32, u64, f32]
    L.oracle_qsgd_mn_dequant_accumulate.argtypes = [vp, i32, vp, i64, i32]
    L.oracle_ternary_words.restype = i64
    L.oracle_qsgd_mnts_words.restype = i64
    L.oracle_qsgd_mnts_words.argtypes = [i64, i32, i32]
    L.oracle_qsgd_mnts_fine_scale.restype = f32
    L.oracle_qsgd_mnts_fine_scale.argtypes = [f32, i32]
    L.oracle_qsgd_mnts_quantize.argtypes = [vp, vp, i64, i32, i32, u64, f32]
    L.oracle_qsgd_mnts_levels.argtypes = [f32, f32, i32, i32, u64, i64, vp]
    L.oracle_qsgd_mnts_dequant_accumulate.argtypes = [vp, i32, vp, i64, i32, i32]
    L.oracle_grandk_mn_max.restype = f32
    L.oracle_grandk_mn_max.argtypes = [vp, i32, i64, vp, i64]
    L.oracle_grandk_mn_quantize.argtypes = [vp, i64, vp, i64, vp, i32, u64, f32]
    L.oracle_grandk_mn_dequant_accumulate.argtypes = [vp, i32, vp, i64, vp, i64, i32]
    L.oracle_ternary_words.argtypes = [i64]
    L.oracle_quantize_ternary.argtypes = [vp, vp, vp, i64, f32, f32]
    L.oracle_dequantize_ternary.argtypes = [vp, vp, i64]
    L.oracle_dequant_accumulate_ternary.argtypes = [vp, i32, vp, i64]
    return L


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


# ---------------------------------------------------------------- 2-bit ----

def words_2bit(n: int) -> int:
    return int(lib().oracle_2bit_words(n))


def quantize_2bit(grad, residual, neg_thr, pos_thr, L=None):
    """Return (compr, new_residual); the inputs are not modified.

    ``grad`` is float32, or uint16 holding bfloat16 bit patterns.
    """
    L = L or lib()
    grad = np.ascontiguousarray(grad)
    res = _c(residual, np.float32).copy()
    n = res.size
    if grad.size != n:
        raise ValueError("grad and residual sizes differ")
    compr = np.zeros(int(L.oracle_2bit_words(n)), np.uint32)
    if grad.dtype == np.float32:
        L.oracle_quantize_2bit(grad.ctypes.data, res.ctypes.data, compr.ctypes.data, n,
                               float(neg_thr), float(pos_thr))
    elif grad.dtype == np.uint16:
        L.oracle_quantize_2bit_bf16(grad.ctypes.data, res.ctypes.data, compr.ctypes.data, n,
                                    float(neg_thr), float(pos_thr))
    else:
        raise TypeError(f"grad dtype {grad.dtype}")
    return compr, res


def dequantize_2bit(compr, n, L=None):
    L = L or lib()
    compr = _c(compr, np.uint32)
    out = np.empty(n, np.float32)
    L.oracle_dequantize_2bit(compr.ctypes.data, out.ctypes.data, n)
    return out


def dequant_accumulate_2bit(comprs, n, L=None):
    L = L or lib()
    comprs = [_c(c, np.uint32) for c in comprs]
    out = np.empty(n, np.float32)
    L.oracle_dequant_accumulate_2bit(_ptr_array(comprs), len(comprs), out.ctypes.data, n)
    return out


def bucket_words_2bit(sizes) -> int:
    L = lib()
    n = np.asarray(sizes, np.int64)
    return int(L.oracle_2bit_bucket_words(n.ctypes.data, n.size))


def quantize_2bit_bucket(grads, residuals, neg_thr, pos_thr, L=None):
    """Bucket of T tensors; returns (compr, [new residuals])."""
    L = L or lib()
    grads = [np.ascontiguousarray(g) for g in grads]
    is_bf16 = int(grads[0].dtype == np.uint16)
    res = [_c(r, np.float32).copy() for r in residuals]
    n = np.array([r.size for r in res], np.int64)
    neg = np.asarray(neg_thr, np.float32)
    pos = np.asarray(pos_thr, np.float32)
    compr = np.zeros(int(L.oracle_2bit_bucket_words(n.ctypes.data, n.size)), np.uint32)
    L.oracle_quantize_2bit_bucket(_ptr_array(grads), _ptr_array(res), n.ctypes.data,
                                  neg.ctypes.data, pos.ctypes.data, len(grads), is_bf16,
                                  compr.ctypes.data)
    return compr, res


def dequant_accumulate_2bit_bucket(comprs, sizes, L=None):
    L = L or lib()
    comprs = [_c(c, np.uint32) for c in comprs]
    n = np.asarray(sizes, np.int64)
    out = np.empty(int(n.sum()), np.float32)
    L.oracle_dequant_accumulate_2bit_bucket(_ptr_array(comprs), len(comprs), n.ctypes.data,
                                            n.size, out.ctypes.data)
    return out


# ----------------------------------------------------------------- QSGD ----

def philox4x32_10(counter, key, L=None):
    L = L or lib()
    c = np.asarray(counter, np.uint32).copy()
    k = np.asarray(key, np.uint32).copy()
    out = np.zeros(4, np.uint32)
    L.oracle_philox4x32_10(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def qsgd_uniform(seed: int, e: int, L=None) -> float:
    L = L or lib()
    return float(np.float32(L.oracle_qsgd_uniform(seed, e)))


def qsgd_level(grad: float, M: float, b: int, seed: int, e: int, L=None) -> int:
    L = L or lib()
    return int(L.oracle_qsgd_level(float(grad), float(M), b, seed, e))


def qsgd_words(n: int, b: int) -> int:
    return int(lib().oracle_qsgd_words(n, b))


def qsgd_mn_max(grads, L=None) -> np.float32:
    L = L or lib()
    grads = [_c(g, np.float32) for g in grads]
    n = grads[0].size
    return np.float32(L.oracle_qsgd_mn_max(_ptr_array(grads), len(grads), n))


def qsgd_mn_quantize(grad, b, seed, M, L=None):
    L = L or lib()
    grad = _c(grad, np.float32)
    n = grad.size
    compr = np.zeros(int(L.oracle_qsgd_words(n, b)), np.uint32)
    L.oracle_qsgd_mn_quantize(grad.ctypes.data, compr.ctypes.data, n, b, seed, float(M))
    return compr


def qsgd_mn_dequant_accumulate(comprs, n, b, L=None):
    L = L or lib()
    comprs = [_c(c, np.uint32) for c in comprs]
    out = np.empty(n, np.float32)
    L.oracle_qsgd_mn_dequant_accumulate(_ptr_array(comprs), len(comprs), out.ctypes.data, n, b)
    return out


# ----------------------------------------------------------- QSGD-MN-TS ----

def qsgd_mnts_words(n: int, b1: int, b2: int, L=None) -> int:
    L = L or lib()
    return int(L.oracle_qsgd_mnts_words(n, b1, b2))


def qsgd_mnts_fine_scale(M, b1: int, L=None) -> np.float32:
    L = L or lib()
    return np.float32(L.oracle_qsgd_mnts_fine_scale(float(M), b1))


def qsgd_mnts_levels(grad: float, M, b1: int, b2: int, seed: int, e: int, L=None):
    """(coarse level, fine level) of one element at position e."""
    L = L or lib()
    q = np.zeros(2, np.int32)
    L.oracle_qsgd_mnts_levels(float(grad), float(M), b1, b2, seed, e, q.ctypes.data)
    return int(q[0]), int(q[1])


def qsgd_mnts_quantize(grad, b1, b2, seed, M, L=None):
    """Two-scale record: the coarse QSGD-MaxNorm record of b1 bits, then the
    fine one of b2 bits."""
    L = L or lib()
    grad = _c(grad, np.float32)
    n = grad.size
    compr = np.zeros(int(L.oracle_qsgd_mnts_words(n, b1, b2)), np.uint32)
    L.oracle_qsgd_mnts_quantize(grad.ctypes.data, compr.ctypes.data, n, b1, b2, seed, float(M))
    return compr


def qsgd_mnts_dequant_accumulate(comprs, n, b1, b2, L=None):
    L = L or lib()
    comprs = [_c(c, np.uint32) for c in comprs]
    out = np.empty(n, np.float32)
    L.oracle_qsgd_mnts_dequant_accumulate(_ptr_array(comprs), len(comprs), out.ctypes.data, n,
                                          b1, b2)
    return out


# ------------------------------------------------------------ GRandK-MN ----

def grandk_mn_max(grads, index, L=None) -> np.float32:
    """M = max |g_w[index[k]]| over workers and kept coordinates in [0, n)."""
    L = L or lib()
    grads = [_c(g, np.float32) for g in grads]
    index = _c(index, np.int64)
    n = grads[0].size
    return np.float32(L.oracle_grandk_mn_max(_ptr_array(grads), len(grads), n,
                                             index.ctypes.data, index.size))


def grandk_mn_quantize(grad, index, b, seed, M, L=None):
    """One worker's record of its kept coordinates (length K = index.size)."""
    L = L or lib()
    grad = _c(grad, np.float32)
    index = _c(index, np.int64)
    K = index.size
    compr = np.zeros(int(L.oracle_qsgd_words(K, b)), np.uint32)
    L.oracle_grandk_mn_quantize(grad.ctypes.data, grad.size, index.ctypes.data, K,
                                compr.ctypes.data, b, seed, float(M))
    return compr


def grandk_mn_dequant_accumulate(comprs, index, n, b, L=None):
    """The n-element merge: scaled level sums at the kept coordinates, +0 elsewhere."""
    L = L or lib()
    comprs = [_c(c, np.uint32) for c in comprs]
    index = _c(index, np.int64)
    out = np.full(n, np.nan, np.float32)     # an element left unwritten shows as NaN
    L.oracle_grandk_mn_dequant_accumulate(_ptr_array(comprs), len(comprs), index.ctypes.data,
                                          index.size, out.ctypes.data, n, b)
    return out


# -------------------------------------------------------- dense ternary ----

def words_ternary(n: int) -> int:
    return int(lib().oracle_ternary_words(n))


def quantize_ternary(grad, residual, neg_thr, pos_thr, L=None):
    """Return (compr, new_residual) of the dense ternary record."""
    L = L or lib()
    grad = _c(grad, np.float32)
    res = _c(residual, np.float32).copy()
    n = res.size
    compr = np.zeros(int(L.oracle_ternary_words(n)), np.uint32)
    L.oracle_quantize_ternary(grad.ctypes.data, res.ctypes.data, compr.ctypes.data, n,
                              float(neg_thr), float(pos_thr))
    return compr, res


def dequantize_ternary(compr, n, L=None):
    L = L or lib()
    compr = _c(compr, np.uint32)
    out = np.empty(n, np.float32)
    L.oracle_dequantize_ternary(compr.ctypes.data, out.ctypes.data, n)
    return out


def dequant_accumulate_ternary(comprs, n, L=None):
    L = L or lib()
    comprs = [_c(c, np.uint32) for c in comprs]
    out = np.empty(n, np.float32)
    L.oracle_dequant_accumulate_ternary(_ptr_array(comprs), len(comprs), out.ctypes.data, n)
    return out
