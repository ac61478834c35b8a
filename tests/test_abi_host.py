"""Host-side checks of libqga.so that need no GPU.

The library loads, exports every entry point that include/qga.h declares,
answers the size queries, and rejects invalid arguments with a status before
it makes any CUDA call (so none of these calls reaches a GPU, here or on a
GPU machine).
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qga.h")


@pytest.fixture(scope="module")
def qga():
    import __graft_entry__
    __graft_entry__._load_build_module().build()
    import quantized_gradient_aggregation_b200 as q
    return q


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|int64_t|int)\s*(qga_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["qga_2bit_words", "qga_quantize_2bit", "qga_quantize_2bit_bf16",
                 "qga_dequantize_2bit", "qga_dequant_accumulate_2bit", "qga_2bit_bucket_words",
                 "qga_quantize_2bit_bucket", "qga_dequant_accumulate_2bit_bucket",
                 "qga_qsgd_words", "qga_qsgd_mn_max", "qga_qsgd_mn_quantize",
                 "qga_qsgd_mn_dequant_accumulate", "qga_strerror", "qga_last_cuda_error",
                 "qga_version", "qga_ternary_words", "qga_quantize_ternary",
                 "qga_dequantize_ternary", "qga_dequant_accumulate_ternary",
                 "qga_grandk_mn_max", "qga_grandk_mn_quantize",
                 "qga_grandk_mn_dequant_accumulate", "qga_quantize_merge_2bit"]:
        assert want in names, want


def test_library_exports_every_declared_symbol(qga):
    lib = ctypes.CDLL(qga.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", qga.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(qga_\w+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported
    # the binding covers the whole boundary
    assert set(declared_functions()) == set(qga.EXPORTED)


def test_library_does_not_link_the_oracle(qga):
    out = subprocess.run(["nm", "-D", qga.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle_" not in out
    ldd = subprocess.run(["ldd", qga.LIB_PATH], capture_output=True, text=True).stdout
    assert "qga_oracle" not in ldd


def test_size_queries(qga):
    L = qga.lib()
    for n, w in [(0, 3), (1, 4), (16, 4), (17, 5), (138_357_544, 8_647_350), (25_557_032, 1_597_318),
                 (1 << 20, 65_539)]:
        assert L.qga_2bit_words(n) == w
    assert L.qga_2bit_words(-1) == qga.QGA_ERR_INVALID_ARG
    for b, n, w in [(2, 1 << 27, 3 + (1 << 23)), (4, 1 << 27, 3 + (1 << 24)), (8, 5, 5), (2, 0, 3)]:
        assert L.qga_qsgd_words(n, b) == w
    assert L.qga_qsgd_words(10, 3) == qga.QGA_ERR_UNSUPPORTED
    assert L.qga_qsgd_words(-1, 2) == qga.QGA_ERR_INVALID_ARG
    import workloads
    sizes = workloads.bert_base_sizes()
    assert len(sizes) == 197 and sum(sizes) == 109_480_704
    assert all(s % 16 == 0 for s in sizes)
    assert qga.qga_2bit_bucket_words(sizes) == 6_843_135


def test_strerror_and_version(qga):
    L = qga.lib()
    for st in (0, -1, -2, -3, 7):
        assert isinstance(L.qga_strerror(st), bytes) and L.qga_strerror(st)
    assert L.qga_version() >= 10000
    assert L.qga_last_cuda_error() == 0


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def test_invalid_arguments_are_rejected_before_any_cuda_call(qga):
    L = qga.lib()
    E = qga.QGA_ERR_INVALID_ARG
    inf, nan = float("inf"), float("nan")
    # quantize: null/misaligned pointers, negative n, non-finite thresholds
    assert L.qga_quantize_2bit(None, FAKE, FAKE, 16, -1.0, 1.0, None) == E
    assert L.qga_quantize_2bit(FAKE, None, FAKE, 16, -1.0, 1.0, None) == E
    assert L.qga_quantize_2bit(FAKE, FAKE, None, 16, -1.0, 1.0, None) == E
    assert L.qga_quantize_2bit(FAKE, FAKE, FAKE, -5, -1.0, 1.0, None) == E
    assert L.qga_quantize_2bit(FAKE, FAKE, FAKE, 16, nan, 1.0, None) == E
    assert L.qga_quantize_2bit(FAKE, FAKE, FAKE, 16, -1.0, inf, None) == E
    assert L.qga_quantize_2bit(FAKE + 1, FAKE, FAKE, 16, -1.0, 1.0, None) == E
    assert L.qga_quantize_2bit(FAKE, FAKE + 2, FAKE, 16, -1.0, 1.0, None) == E
    assert L.qga_quantize_2bit(FAKE, FAKE, FAKE + 2, 16, -1.0, 1.0, None) == E
    assert L.qga_quantize_2bit_bf16(FAKE + 1, FAKE, FAKE, 16, -1.0, 1.0, None) == E
    # dequantize / merge
    assert L.qga_dequantize_2bit(None, FAKE, 16, None) == E
    assert L.qga_dequantize_2bit(FAKE, None, 16, None) == E
    assert L.qga_dequantize_2bit(FAKE, FAKE + 1, 16, None) == E
    arr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    parr = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    assert L.qga_dequant_accumulate_2bit(parr, 0, FAKE, 16, None) == E
    assert L.qga_dequant_accumulate_2bit(parr, 65, FAKE, 16, None) == E
    assert L.qga_dequant_accumulate_2bit(None, 2, FAKE, 16, None) == E
    assert L.qga_dequant_accumulate_2bit(parr, 2, None, 16, None) == E
    bad = (ctypes.c_void_p * 2)(FAKE, 0)
    assert L.qga_dequant_accumulate_2bit(ctypes.cast(bad, ctypes.POINTER(ctypes.c_void_p)), 2,
                                         FAKE, 16, None) == E
    # quantize + merge of the reducing worker
    assert L.qga_quantize_merge_2bit(FAKE, FAKE, 16, -1.0, 1.0, parr, 2, 2, FAKE, None) == E
    assert L.qga_quantize_merge_2bit(FAKE, FAKE, 16, -1.0, 1.0, parr, 2, -1, FAKE, None) == E
    assert L.qga_quantize_merge_2bit(FAKE, FAKE, 16, nan, 1.0, parr, 2, 0, FAKE, None) == E
    assert L.qga_quantize_merge_2bit(FAKE, FAKE, -1, -1.0, 1.0, parr, 2, 0, FAKE, None) == E
    assert L.qga_quantize_merge_2bit(None, FAKE, 16, -1.0, 1.0, parr, 2, 0, FAKE, None) == E
    assert L.qga_quantize_merge_2bit(FAKE, FAKE, 16, -1.0, 1.0, parr, 2, 0, None, None) == E
    assert L.qga_quantize_merge_2bit(FAKE, FAKE + 2, 16, -1.0, 1.0, parr, 2, 0, FAKE, None) == E
    assert L.qga_quantize_merge_2bit(FAKE, FAKE, 16, -1.0, 1.0, parr, 0, 0, FAKE, None) == E
    assert L.qga_quantize_merge_2bit(FAKE, FAKE, 16, -1.0, 1.0,
                                     ctypes.cast(bad, ctypes.POINTER(ctypes.c_void_p)), 2, 0, FAKE,
                                     None) == E
    # bucket
    T = qga.qga_bucket_tensor
    rows = (T * 2)(T(FAKE, FAKE, 16, -1.0, 1.0), T(FAKE, FAKE, -1, -1.0, 1.0))
    assert L.qga_quantize_2bit_bucket(rows, 2, qga.QGA_DTYPE_F32, FAKE, None) == E
    rows = (T * 1)(T(FAKE, FAKE, 16, nan, 1.0))
    assert L.qga_quantize_2bit_bucket(rows, 1, qga.QGA_DTYPE_F32, FAKE, None) == E
    rows = (T * 1)(T(FAKE, FAKE, 16, -1.0, 1.0))
    assert L.qga_quantize_2bit_bucket(rows, 1, 7, FAKE, None) == qga.QGA_ERR_UNSUPPORTED
    assert L.qga_quantize_2bit_bucket(rows, 1, qga.QGA_DTYPE_F32, None, None) == E
    assert L.qga_quantize_2bit_bucket(rows, -1, qga.QGA_DTYPE_F32, FAKE, None) == E
    sizes = (ctypes.c_int64 * 2)(16, -3)
    assert L.qga_dequant_accumulate_2bit_bucket(parr, 2, sizes, 2, FAKE, None) == E
    assert L.qga_2bit_bucket_words(sizes, 2) == E
    # QSGD
    assert L.qga_qsgd_mn_max(parr, 0, 16, FAKE, None) == E
    assert L.qga_qsgd_mn_max(parr, 2, 16, None, None) == E
    assert L.qga_qsgd_mn_max(parr, 2, 16, FAKE + 1, None) == E
    assert L.qga_qsgd_mn_quantize(FAKE, FAKE, 16, 2, 0, None, None) == E
    assert L.qga_qsgd_mn_quantize(None, FAKE, 16, 2, 0, FAKE, None) == E
    assert L.qga_qsgd_mn_quantize(FAKE, FAKE, -1, 2, 0, FAKE, None) == E
    assert L.qga_qsgd_mn_quantize(FAKE, FAKE, 16, 3, 0, FAKE, None) == qga.QGA_ERR_UNSUPPORTED
    assert L.qga_qsgd_mn_dequant_accumulate(parr, 2, FAKE, 16, 5, None) == qga.QGA_ERR_UNSUPPORTED
    assert L.qga_qsgd_mn_dequant_accumulate(parr, 2, None, 16, 2, None) == E
    assert L.qga_qsgd_mn_dequant_accumulate(parr, 99, FAKE, 16, 2, None) == E
    # GRandK-MN: index is int64 (8-byte aligned), K >= 0
    assert L.qga_grandk_mn_max(parr, 2, 16, FAKE, -1, FAKE, None) == E
    assert L.qga_grandk_mn_max(parr, 2, 16, None, 4, FAKE, None) == E
    assert L.qga_grandk_mn_max(parr, 2, 16, FAKE + 4, 4, FAKE, None) == E
    assert L.qga_grandk_mn_max(parr, 0, 16, FAKE, 4, FAKE, None) == E
    assert L.qga_grandk_mn_max(ctypes.cast(bad, ctypes.POINTER(ctypes.c_void_p)), 2, 16, FAKE, 4,
                               FAKE, None) == E
    assert L.qga_grandk_mn_quantize(FAKE, 16, FAKE + 4, 4, FAKE, 2, 0, FAKE, None) == E
    assert L.qga_grandk_mn_quantize(None, 16, FAKE, 4, FAKE, 2, 0, FAKE, None) == E
    assert L.qga_grandk_mn_quantize(FAKE, 16, FAKE, 4, None, 2, 0, FAKE, None) == E
    assert L.qga_grandk_mn_quantize(FAKE, 16, FAKE, 4, FAKE, 2, 0, None, None) == E
    assert L.qga_grandk_mn_quantize(FAKE, -2, FAKE, 4, FAKE, 2, 0, FAKE, None) == E
    assert L.qga_grandk_mn_quantize(FAKE, 16, FAKE, 4, FAKE, 6, 0, FAKE, None) == qga.QGA_ERR_UNSUPPORTED
    assert L.qga_grandk_mn_dequant_accumulate(parr, 2, FAKE, 4, FAKE, 16, 3, None) == \
        qga.QGA_ERR_UNSUPPORTED
    assert L.qga_grandk_mn_dequant_accumulate(parr, 2, None, 4, FAKE, 16, 2, None) == E
    assert L.qga_grandk_mn_dequant_accumulate(parr, 2, FAKE, 4, None, 16, 2, None) == E
    assert L.qga_grandk_mn_dequant_accumulate(parr, 2, FAKE, -4, FAKE, 16, 2, None) == E
    assert L.qga_grandk_mn_dequant_accumulate(parr, 65, FAKE, 4, FAKE, 16, 2, None) == E
    # dense ternary
    assert L.qga_ternary_words(-1) == E and L.qga_ternary_words(0) == 3 and L.qga_ternary_words(21) == 5
    assert L.qga_quantize_ternary(None, FAKE, FAKE, 16, -1.0, 1.0, None) == E
    assert L.qga_quantize_ternary(FAKE, FAKE, FAKE, 16, nan, 1.0, None) == E
    assert L.qga_quantize_ternary(FAKE + 1, FAKE, FAKE, 16, -1.0, 1.0, None) == E
    assert L.qga_dequantize_ternary(FAKE, None, 16, None) == E
    assert L.qga_dequant_accumulate_ternary(parr, 0, FAKE, 16, None) == E
    assert L.qga_dequant_accumulate_ternary(parr, 2, FAKE + 2, 16, None) == E
    assert L.qga_last_cuda_error() == 0


def test_binding_refuses_cpu_tensors(qga):
    import torch
    g = torch.zeros(16)
    r = torch.zeros(16)
    c = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        qga.qga_quantize_2bit(g, r, c, -1.0, 1.0)
