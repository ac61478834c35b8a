"""GPU parity of the dense ternary records (5 codes per byte) through the C
ABI against the CPU oracle: record words and residuals bit for bit, merged
values bit for bit and within 1e-6 relative + 1e-7 absolute."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import AGG_ATOL, AGG_RTOL, DEV, f32, first_diff, offset_view, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu

SIZES = [0, 1, 4, 5, 6, 19, 20, 21, 639, 640, 641, 1283, 65_537, (1 << 20) + 3]


def _inputs(n, seed):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    g = torch.randn(n, device=DEV, generator=gen) * 0.7
    r = torch.rand(n, device=DEV, generator=gen) - 0.5
    return g, r


def _quantize(g, r, neg, pos, compr_offset=0):
    q = qga()
    n = r.numel()
    words = q.qga_ternary_words(n)
    base = torch.full((words + compr_offset + 4,), -1, dtype=torch.int32, device=DEV)
    base[words + compr_offset:] = 0x5A5A5A5A
    compr = base[compr_offset:compr_offset + words]
    q.qga_quantize_ternary(g, r, compr, neg, pos)
    torch.cuda.synchronize()
    assert (u32(base[words + compr_offset:]) == 0x5A5A5A5A).all()
    return compr


@pytest.mark.parametrize("n", SIZES)
def test_quantize_ternary(n):
    g, r = _inputs(n, 300 + n)
    g_host, r_host = f32(g).copy(), f32(r).copy()
    compr = _quantize(g, r, -0.5, 0.5)
    want_c, want_r = oracle.quantize_ternary(g_host, r_host, -0.5, 0.5)
    assert np.array_equal(u32(compr), want_c), first_diff(u32(compr), want_c)
    assert same_bits_f32(f32(r), want_r)


@pytest.mark.parametrize("offsets", [(1, 0, 0), (0, 3, 1), (2, 2, 2)])
def test_quantize_ternary_misaligned(offsets):
    n = 4099
    g0, r0 = _inputs(n, 17)
    g = offset_view(n, torch.float32, offsets[0])
    r = offset_view(n, torch.float32, offsets[1])
    g.copy_(g0)
    r.copy_(r0)
    g_host, r_host = f32(g).copy(), f32(r).copy()
    compr = _quantize(g, r, -0.3, 0.8, compr_offset=offsets[2])
    want_c, want_r = oracle.quantize_ternary(g_host, r_host, -0.3, 0.8)
    assert np.array_equal(u32(compr), want_c)
    assert same_bits_f32(f32(r), want_r)


def test_ternary_residual_equals_2bit_residual():
    """Same error feedback as the 2-bit operator, bit for bit."""
    q = qga()
    n = 100_000
    g, r = _inputs(n, 5)
    r2 = r.clone()
    c3 = torch.empty(q.qga_ternary_words(n), dtype=torch.int32, device=DEV)
    c2 = torch.empty(q.qga_2bit_words(n), dtype=torch.int32, device=DEV)
    q.qga_quantize_ternary(g, r, c3, -0.5, 0.5)
    q.qga_quantize_2bit(g, r2, c2, -0.5, 0.5)
    assert same_bits_f32(f32(r), f32(r2))
    out3 = torch.empty(n, device=DEV)
    out2 = torch.empty(n, device=DEV)
    q.qga_dequantize_ternary(c3, out3)
    q.qga_dequantize_2bit(c2, out2)
    assert same_bits_f32(f32(out3), f32(out2))


def _random_record(n, neg, pos, seed):
    rng = np.random.default_rng(seed)
    nbytes = -(-n // 5)
    words = np.zeros(3 + -(-n // 20), np.uint32)
    words[:3] = np.array([neg, pos, n], np.float32).view(np.uint32)
    digits = rng.integers(0, 3, 5 * nbytes)
    digits[n:] = 0
    b = (digits.reshape(-1, 5) * np.array([81, 27, 9, 3, 1])).sum(1).astype(np.uint8)
    words[3:].view(np.uint8)[:nbytes] = b
    return words


@pytest.mark.parametrize("n", [1, 5, 21, 641, 65_537])
@pytest.mark.parametrize("oo", [0, 1])
def test_dequantize_ternary(n, oo):
    rec = _random_record(n, -0.75, 1.25, n)
    out = offset_view(n, torch.float32, oo, fill=float("nan"))
    qga().qga_dequantize_ternary(torch.from_numpy(rec.view(np.int32).copy()).to(DEV), out)
    assert same_bits_f32(f32(out), oracle.dequantize_ternary(rec, n))


@pytest.mark.parametrize("W", [1, 3, 8, 9, 17, 33, 64])
@pytest.mark.parametrize("n", [21, 641, 65_537])
def test_dequant_accumulate_ternary(W, n):
    rng = np.random.default_rng(W + n)
    recs = [_random_record(n, -float(a), float(b), 7 * w + n)
            for w, (a, b) in enumerate(rng.uniform(0.01, 2.0, (W, 2)).astype(np.float32))]
    out = offset_view(n, torch.float32, n % 3, fill=float("nan"))
    qga().qga_dequant_accumulate_ternary(
        [torch.from_numpy(r.view(np.int32).copy()).to(DEV) for r in recs], out)
    want = oracle.dequant_accumulate_ternary(recs, n)
    got = f32(out)
    np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
    assert same_bits_f32(got, want), first_diff(got, want)


def test_ternary_resnet50_four_workers_full():
    """ResNet-50-sized gradients, 4 workers: every word, residual and merged
    value of the dense path checked against the oracle."""
    w = workloads.WORKLOADS["resnet50-4w"]
    n = w.n
    q = qga()
    comprs, want_recs = [], []
    for k in range(w.workers):
        g = workloads.gradient(w, k, 0, device=DEV)
        r = workloads.random_residual(n, w.pos_thr, 50 + k, device=DEV)
        g_host, r_host = f32(g), f32(r).copy()
        c = torch.empty(q.qga_ternary_words(n), dtype=torch.int32, device=DEV)
        q.qga_quantize_ternary(g, r, c, w.neg_thr, w.pos_thr)
        want_c, want_r = oracle.quantize_ternary(g_host, r_host, w.neg_thr, w.pos_thr)
        assert np.array_equal(u32(c), want_c), (k, first_diff(u32(c), want_c))
        assert same_bits_f32(f32(r), want_r), k
        comprs.append(c)
        want_recs.append(want_c)
        del g, r
    out = torch.empty(n, device=DEV)
    q.qga_dequant_accumulate_ternary(comprs, out)
    want = oracle.dequant_accumulate_ternary(want_recs, n)
    assert same_bits_f32(f32(out), want)
