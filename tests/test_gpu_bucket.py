"""GPU parity of the ragged bucket launcher against the CPU oracle: a bucket
equals its tensors' standalone records one after the other, word for word,
and its merge equals the per-tensor merges."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import AGG_ATOL, AGG_RTOL, DEV, bf16_bits, f32, first_diff, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu


def _quantize_bucket(grads, residuals, neg, pos):
    q = qga()
    sizes = [r.numel() for r in residuals]
    words = q.qga_2bit_bucket_words(sizes)
    compr = torch.full((words + 4,), 0x5A5A5A5A, dtype=torch.int32, device=DEV)
    q.qga_quantize_2bit_bucket(grads, residuals, neg, pos, compr[:words])
    torch.cuda.synchronize()
    assert (u32(compr[words:]) == 0x5A5A5A5A).all()
    return compr[:words]


def _host(g):
    return bf16_bits(g) if g.dtype == torch.bfloat16 else f32(g).copy()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ragged_bucket(dtype):
    sizes = [0, 1, 15, 16, 17, 33, 768, 4095, 8192, 8193, 70_001, 5, 0, 3]
    rng = np.random.default_rng(3)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(5)
    # misaligned tensors: carve them out of one buffer at odd offsets
    offs = np.cumsum([0] + [s + 1 for s in sizes])
    gbuf = (torch.randn(int(offs[-1]), device=DEV, generator=gen) * 0.05).to(dtype)
    rbuf = (torch.rand(int(offs[-1]), device=DEV, generator=gen) - 0.5) * 0.04
    grads = [gbuf[offs[i]:offs[i] + s] for i, s in enumerate(sizes)]
    res = [rbuf[offs[i]:offs[i] + s] for i, s in enumerate(sizes)]
    thr = rng.uniform(0.01, 0.06, len(sizes)).astype(np.float32)
    neg, pos = [-float(t) for t in thr], [float(t) for t in thr]
    g_host = [_host(g) for g in grads]
    r_host = [f32(r).copy() for r in res]
    compr = _quantize_bucket(grads, res, neg, pos)
    want_c, want_r = oracle.quantize_2bit_bucket(g_host, r_host, neg, pos)
    assert np.array_equal(u32(compr), want_c), first_diff(u32(compr), want_c)
    for t in range(len(sizes)):
        assert same_bits_f32(f32(res[t]), want_r[t]), t


def test_bucket_of_more_than_256_tensors():
    """Tables over 256 tensors are split into several launches."""
    sizes = [16 * (1 + (i % 7)) + (i % 5) for i in range(600)]
    gen = torch.Generator(device=DEV)
    gen.manual_seed(11)
    grads = [torch.randn(s, device=DEV, generator=gen) for s in sizes]
    res = [torch.zeros(s, device=DEV) for s in sizes]
    neg = [-0.5 - 0.001 * i for i in range(600)]
    pos = [0.5 + 0.001 * i for i in range(600)]
    g_host = [f32(g) for g in grads]
    compr = _quantize_bucket(grads, res, neg, pos)
    want_c, want_r = oracle.quantize_2bit_bucket(g_host, [np.zeros(s, np.float32) for s in sizes],
                                                 neg, pos)
    assert np.array_equal(u32(compr), want_c)
    comprs = [compr, compr.clone()]
    out = torch.empty(sum(sizes), device=DEV)
    qga().qga_dequant_accumulate_2bit_bucket(comprs, sizes, out)
    want = oracle.dequant_accumulate_2bit_bucket([want_c, want_c], sizes)
    assert same_bits_f32(f32(out), want)


def test_bert_base_bucket_four_workers():
    """The BERT-Base bucket: 197 bf16 tensors (109,480,704 elements), per-tensor
    +-2 sigma thresholds from worker 0's gradient, 4 workers; every word,
    residual and merged value checked."""
    w = workloads.WORKLOADS["bert-bucket-4w"]
    sizes = workloads.bert_base_sizes()
    q = qga()
    words = q.qga_2bit_bucket_words(sizes)
    comprs, want_recs = [], []
    neg = pos = None
    for k in range(w.workers):
        grads = workloads.bert_bucket(w, k, 0, device=DEV)
        if neg is None:
            neg, pos = workloads.bert_thresholds(grads)
        res = [workloads.random_residual(s, 1e-3, 1000 * k + i, device=DEV)
               for i, s in enumerate(sizes)]
        g_host = [bf16_bits(g) for g in grads]
        r_host = [f32(r).copy() for r in res]
        compr = torch.empty(words, dtype=torch.int32, device=DEV)
        q.qga_quantize_2bit_bucket(grads, res, neg, pos, compr)
        want_c, want_r = oracle.quantize_2bit_bucket(g_host, r_host, neg, pos)
        assert np.array_equal(u32(compr), want_c), (k, first_diff(u32(compr), want_c))
        for t in range(len(sizes)):
            assert same_bits_f32(f32(res[t]), want_r[t]), (k, t)
        comprs.append(compr)
        want_recs.append(want_c)
        del grads, res
    out = torch.empty(sum(sizes), device=DEV)
    q.qga_dequant_accumulate_2bit_bucket(comprs, sizes, out)
    want = oracle.dequant_accumulate_2bit_bucket(want_recs, sizes)
    got = f32(out)
    np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
    assert same_bits_f32(got, want)


def test_bucket_equals_standalone_calls():
    """One bucket launch == T single-tensor launches, word for word."""
    sizes = [768, 3072, 17, 589_824, 0, 33]
    gen = torch.Generator(device=DEV)
    gen.manual_seed(21)
    grads = [(torch.randn(s, device=DEV, generator=gen) * 1e-3).to(torch.bfloat16) for s in sizes]
    res_a = [torch.zeros(s, device=DEV) for s in sizes]
    res_b = [torch.zeros(s, device=DEV) for s in sizes]
    neg = [-2e-3] * len(sizes)
    pos = [2e-3] * len(sizes)
    bucket = _quantize_bucket(grads, res_a, neg, pos)
    pieces = []
    for t, s in enumerate(sizes):
        c = torch.empty(qga().qga_2bit_words(s), dtype=torch.int32, device=DEV)
        qga().qga_quantize_2bit(grads[t], res_b[t], c, neg[t], pos[t])
        pieces.append(u32(c))
    assert np.array_equal(u32(bucket), np.concatenate(pieces))
    for t in range(len(sizes)):
        assert same_bits_f32(f32(res_a[t]), f32(res_b[t]))
