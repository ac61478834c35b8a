"""The oracle's Philox4x32-10 against cuRAND's (a library implementation,
run on the GPU): raw output words for many seeds and counter blocks,
including counters above 2^32 (their high word set)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def curand_lib(tmp_path_factory):
    so = tmp_path_factory.mktemp("curand") / "libcurand_philox_ref.so"
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                    "-Xcompiler", "-fPIC", "-o", str(so), os.path.join(HERE, "curand_philox_ref.cu")],
                   check=True)
    lib = ctypes.CDLL(str(so))
    lib.curand_philox_blocks.argtypes = [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_void_p]
    return lib


def test_oracle_philox_equals_curand(curand_lib):
    rng = np.random.default_rng(4)
    seeds = [0, 1, 1234, 1241, 0xFFFFFFFF, 1 << 32, 0x0123456789ABCDEF, 2 ** 64 - 1]
    blocks = np.concatenate([np.arange(64), rng.integers(0, 1 << 40, 192),
                             [(1 << 32) - 1, 1 << 32, (1 << 32) + 5]]).astype(np.uint64)
    dev_blocks = torch.from_numpy(blocks.view(np.int64)).cuda()
    out = torch.empty((blocks.size, 4), dtype=torch.int32, device="cuda")
    for seed in seeds:
        st = curand_lib.curand_philox_blocks(seed, dev_blocks.data_ptr(), blocks.size, out.data_ptr())
        assert st == 0
        got = out.cpu().numpy().view(np.uint32)
        for i, blk in enumerate(blocks.tolist()):
            want = oracle.philox4x32_10([blk & 0xFFFFFFFF, blk >> 32, 0, 0],
                                        [seed & 0xFFFFFFFF, seed >> 32])
            assert got[i].tolist() == want.tolist(), (seed, blk)
