"""The compressed all-gather exchange on a one-rank NCCL group (the only GPU
count this test machine offers): quantize, NCCL all-gather, merge, all on the
device, against the oracle.  The multi-rank layout of the gather is tested
with gloo ranks on CPU (test_dist_gloo.py)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from gpu_util import DEV, f32, same_bits_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt", ["2bit", "ternary"])
def test_exchange_one_rank(nccl_group, fmt):
    from quantized_gradient_aggregation_b200.exchange import CompressedAllGather
    n = 1_000_003
    gen = torch.Generator(device=DEV)
    gen.manual_seed(3)
    g = torch.randn(n, device=DEV, generator=gen) * 0.4
    r = torch.zeros(n, device=DEV)
    out = torch.empty(n, device=DEV)
    ex = CompressedAllGather(n, -0.25, 0.25, fmt=fmt)
    g_host = f32(g)
    r_host = np.zeros(n, np.float32)
    for it in range(3):
        ex.step(g, r, out)
        if fmt == "2bit":
            rec, r_host = oracle.quantize_2bit(g_host, r_host, -0.25, 0.25)
            want = oracle.dequant_accumulate_2bit([rec], n)
        else:
            rec, r_host = oracle.quantize_ternary(g_host, r_host, -0.25, 0.25)
            want = oracle.dequant_accumulate_ternary([rec], n)
        assert np.array_equal(ex.gathered.cpu().numpy().view(np.uint32), rec), it
        assert same_bits_f32(f32(r), r_host), it
        assert same_bits_f32(f32(out), want), it
