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


def test_bucketed_exchange_one_rank(nccl_group):
    """Two BERT-like buckets (bf16 gradients), pipelined all-gathers, three
    steps with carried residuals, against the oracle's bucket functions."""
    from quantized_gradient_aggregation_b200.exchange import BucketedCompressedAllGather
    buckets = [[768, 3072, 589_824, 17], [30_000, 5, 768 * 16]]
    neg = [[-2e-3] * len(b) for b in buckets]
    pos = [[2e-3 + 1e-4 * i for i in range(len(b))] for b in buckets]
    gen = torch.Generator(device=DEV)
    gen.manual_seed(12)
    grads = [[(torch.randn(s, device=DEV, generator=gen) * 1e-3).to(torch.bfloat16) for s in b]
             for b in buckets]
    res = [[torch.zeros(s, device=DEV) for s in b] for b in buckets]
    outs = [torch.empty(sum(b), device=DEV) for b in buckets]
    ex = BucketedCompressedAllGather(buckets, neg, pos)
    g_host = [[g.cpu().view(torch.int16).numpy().view(np.uint16) for g in b] for b in grads]
    r_host = [[np.zeros(s, np.float32) for s in b] for b in buckets]
    for it in range(3):
        ex.step(grads, res, outs)
        for b in range(len(buckets)):
            want_c, r_host[b] = oracle.quantize_2bit_bucket(g_host[b], r_host[b], neg[b], pos[b])
            assert np.array_equal(ex.gathered[b].cpu().numpy().view(np.uint32), want_c), (it, b)
            want = oracle.dequant_accumulate_2bit_bucket([want_c], buckets[b])
            assert same_bits_f32(f32(outs[b]), want), (it, b)
            for t in range(len(buckets[b])):
                assert same_bits_f32(f32(res[b][t]), r_host[b][t]), (it, b, t)


@pytest.mark.parametrize("b", [2, 4, 8])
def test_qsgd_exchange_one_rank(nccl_group, b):
    """QSGD-MaxNorm step on a one-rank NCCL group: the local max, its
    all-reduce, the quantize with this rank's seed, the gather and the merge,
    all on the device, against the oracle."""
    from quantized_gradient_aggregation_b200.exchange import QsgdAllGather
    n = 1_000_003
    gen = torch.Generator(device=DEV)
    gen.manual_seed(7 + b)
    ex = QsgdAllGather(n, b, 1234)
    out = torch.empty(n, device=DEV)
    for it in range(2):
        g = torch.randn(n, device=DEV, generator=gen) * 0.3
        ex.step(g, out)
        g_host = f32(g)
        M = oracle.qsgd_mn_max([g_host])
        assert ex.m.item() == M, it
        rec = oracle.qsgd_mn_quantize(g_host, b, 1234, M)
        assert np.array_equal(ex.gathered.cpu().numpy().view(np.uint32), rec), it
        assert same_bits_f32(f32(out), oracle.qsgd_mn_dequant_accumulate([rec], n, b)), it
