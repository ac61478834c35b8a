"""The library calls are stream-ordered, never synchronize and never
allocate: a whole step (W quantizes + the merge; the bucket path; the QSGD
path with its memset) captures into a CUDA graph -- torch captures in the
"global" error mode, where a device allocation or a synchronizing call from
any thread aborts the capture -- and replaying the graph gives the same bits
as running the calls eagerly on the same inputs."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, qga, u32

pytestmark = pytest.mark.gpu


def _step_2bit(q, grads, res, comprs, out):
    for k in range(len(grads)):
        q.qga_quantize_2bit(grads[k], res[k], comprs[k], -0.5, 0.5)
    q.qga_dequant_accumulate_2bit(comprs, out)


def _bits(ts):
    return [t.detach().cpu().numpy().view(np.uint32).copy() for t in ts]


def test_two_bit_step_in_a_cuda_graph():
    q = qga()
    n, W = 300_007, 4
    gen = torch.Generator(device=DEV)
    gen.manual_seed(8)
    grads = [torch.randn(n, device=DEV, generator=gen) for _ in range(W)]
    res0 = [torch.rand(n, device=DEV, generator=gen) - 0.5 for _ in range(W)]
    # eager: three steps; the device's free memory does not move
    res_e = [r.clone() for r in res0]
    comprs_e = [torch.empty(q.qga_2bit_words(n), dtype=torch.int32, device=DEV) for _ in range(W)]
    out_e = torch.empty(n, device=DEV)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        _step_2bit(q, grads, res_e, comprs_e, out_e)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before, "a library call allocated device memory"
    # graph: capture one step, replay three times
    res_g = [r.clone() for r in res0]
    comprs_g = [torch.empty_like(c) for c in comprs_e]
    out_g = torch.empty(n, device=DEV)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            _step_2bit(q, grads, res_g, comprs_g, out_g)
    # capture does not execute: the residuals are still the initial ones
    assert all(np.array_equal(a, b) for a, b in zip(_bits(res_g), _bits(res0)))
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert all(np.array_equal(a, b) for a, b in zip(_bits(res_g), _bits(res_e)))
    assert all(np.array_equal(a, b) for a, b in zip(_bits(comprs_g), _bits(comprs_e)))
    assert np.array_equal(_bits([out_g])[0], _bits([out_e])[0])


def test_reducing_worker_step_in_a_cuda_graph():
    """The bench's step shape: quantizes of workers 1..W-1, then worker 0's
    fused quantize + merge; captured once, replayed, equal to eager calls."""
    q = qga()
    n, W = 200_003, 4
    gen = torch.Generator(device=DEV)
    gen.manual_seed(10)
    grads = [torch.randn(n, device=DEV, generator=gen) for _ in range(W)]
    res0 = [torch.rand(n, device=DEV, generator=gen) - 0.5 for _ in range(W)]

    def step(res, comprs, out):
        for k in range(1, W):
            q.qga_quantize_2bit(grads[k], res[k], comprs[k], -0.5, 0.5)
        q.qga_quantize_merge_2bit(grads[0], res[0], comprs, 0, -0.5, 0.5, out)

    res_e = [r.clone() for r in res0]
    comprs_e = [torch.empty(q.qga_2bit_words(n), dtype=torch.int32, device=DEV) for _ in range(W)]
    out_e = torch.empty(n, device=DEV)
    for _ in range(2):
        step(res_e, comprs_e, out_e)
    res_g = [r.clone() for r in res0]
    comprs_g = [torch.empty_like(c) for c in comprs_e]
    out_g = torch.empty(n, device=DEV)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step(res_g, comprs_g, out_g)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert all(np.array_equal(a, b) for a, b in zip(_bits(res_g), _bits(res_e)))
    assert all(np.array_equal(a, b) for a, b in zip(_bits(comprs_g), _bits(comprs_e)))
    assert np.array_equal(_bits([out_g])[0], _bits([out_e])[0])


def test_bucket_and_qsgd_in_a_cuda_graph():
    q = qga()
    gen = torch.Generator(device=DEV)
    gen.manual_seed(9)
    sizes = [768, 3072, 589_824, 17]
    grads = [(torch.randn(s, device=DEV, generator=gen) * 1e-3).to(torch.bfloat16) for s in sizes]
    res_e = [torch.zeros(s, device=DEV) for s in sizes]
    res_g = [torch.zeros(s, device=DEV) for s in sizes]
    words = q.qga_2bit_bucket_words(sizes)
    c_e = torch.empty(words, dtype=torch.int32, device=DEV)
    c_g = torch.empty(words, dtype=torch.int32, device=DEV)
    neg, pos = [-2e-3] * 4, [2e-3] * 4
    table_g = q.make_bucket_table(grads, res_g, neg, pos)

    n = 500_003
    gq = [torch.randn(n, device=DEV, generator=gen) for _ in range(3)]
    M_e, M_g = torch.empty(1, device=DEV), torch.empty(1, device=DEV)
    rec_e = [torch.empty(q.qga_qsgd_words(n, 4), dtype=torch.int32, device=DEV) for _ in range(3)]
    rec_g = [torch.empty_like(r) for r in rec_e]
    out_e, out_g = torch.empty(n, device=DEV), torch.empty(n, device=DEV)

    def qsgd(M, recs, out):
        q.qga_qsgd_mn_max(gq, M)
        for k in range(3):
            q.qga_qsgd_mn_quantize(gq[k], recs[k], 4, 1234 + k, M)
        q.qga_qsgd_mn_dequant_accumulate(recs, out, 4)

    for _ in range(2):
        q.qga_quantize_2bit_bucket(grads, res_e, neg, pos, c_e)
    qsgd(M_e, rec_e, out_e)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            q.qga_quantize_2bit_bucket(grads, res_g, neg, pos, c_g, table=table_g)
    graph.replay()
    graph.replay()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g2, stream=side):
            qsgd(M_g, rec_g, out_g)
    g2.replay()
    torch.cuda.synchronize()
    assert np.array_equal(u32(c_g), u32(c_e))
    assert all(np.array_equal(a, b) for a, b in zip(_bits(res_g), _bits(res_e)))
    assert M_g.item() == M_e.item()
    assert all(np.array_equal(a, b) for a, b in zip(_bits(rec_g), _bits(rec_e)))
    assert np.array_equal(_bits([out_g])[0], _bits([out_e])[0])
