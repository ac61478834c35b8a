"""GPU parity of the 2-bit path through the C ABI against the CPU oracle.

Packed words and residuals must match the oracle bit for bit (NaN compared
as NaN); merged aggregates must be within 1e-6 relative + 1e-7 absolute and,
because the kernel adds workers in the oracle's order, are also checked bit
for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import (AGG_ATOL, AGG_RTOL, DEV, f32, first_diff, gather_elems, offset_view, qga,
                      same_bits_f32, sample_words, u32, bf16_bits)

pytestmark = pytest.mark.gpu

CANARY = 0x5A5A5A5A
RAGGED = [0, 1, 2, 3, 4, 5, 15, 16, 17, 31, 33, 127, 129, 511, 512, 513, 4097, 65_537,
          (1 << 20) - 1, (1 << 20) + 1]
THRESHOLDS = [(-0.5, 0.5), (-0.3, 0.8)]


def _inputs(n, seed, dtype=torch.float32):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    g = torch.randn(n, device=DEV, generator=gen) * 0.7
    r = (torch.rand(n, device=DEV, generator=gen) - 0.5)
    return g.to(dtype), r


def _compr_with_canary(words, extra=8):
    buf = torch.full((words + extra,), -1, dtype=torch.int32, device=DEV)   # garbage 0xFFFFFFFF
    buf[words:] = CANARY
    return buf


def _run_quantize(g, r, neg, pos, compr_offset=0):
    q = qga()
    n = r.numel()
    words = q.qga_2bit_words(n)
    base = _compr_with_canary(words + compr_offset)
    compr = base[compr_offset:compr_offset + words]
    q.qga_quantize_2bit(g, r, compr, neg, pos)
    torch.cuda.synchronize()
    tail = u32(base[compr_offset + words:])
    assert (tail == CANARY).all(), "write past the end of the record"
    return compr


def _check_quantize(g, r, neg, pos, compr_offset=0):
    g_host = bf16_bits(g) if g.dtype == torch.bfloat16 else f32(g).copy()
    r_host = f32(r).copy()
    compr = _run_quantize(g, r, neg, pos, compr_offset)
    want_c, want_r = oracle.quantize_2bit(g_host, r_host, neg, pos)
    got_c = u32(compr)
    assert np.array_equal(got_c, want_c), first_diff(got_c, want_c)
    got_r = f32(r)
    assert same_bits_f32(got_r, want_r), first_diff(got_r, want_r)
    return compr, want_c


@pytest.mark.parametrize("n", RAGGED)
@pytest.mark.parametrize("thr", THRESHOLDS)
def test_quantize_fp32_ragged(n, thr):
    g, r = _inputs(n, 1000 + n)
    _check_quantize(g, r, *thr)


@pytest.mark.parametrize("n", [1, 17, 513, 4097, 65_537])
@pytest.mark.parametrize("offsets", [(1, 0, 0), (0, 1, 0), (0, 0, 1), (3, 2, 1),
                                     # 16- but not 32-byte aligned (group tiles), then
                                     # both 32-byte aligned at an offset (lane-owned words)
                                     (4, 4, 0), (4, 0, 0), (8, 8, 3)])
def test_quantize_fp32_misaligned(n, offsets):
    og, orr, oc = offsets
    g0, r0 = _inputs(n, 7 + n)
    g = offset_view(n, torch.float32, og)
    r = offset_view(n, torch.float32, orr)
    g.copy_(g0)
    r.copy_(r0)
    _check_quantize(g, r, -0.5, 0.5, compr_offset=oc)


@pytest.mark.parametrize("n", [0, 1, 5, 16, 33, 513, 4097, (1 << 20) + 3])
@pytest.mark.parametrize("og", [0, 1, 2])
def test_quantize_bf16(n, og):
    g0, r = _inputs(n, 99 + n, torch.bfloat16)
    g = offset_view(n, torch.bfloat16, og)
    g.copy_(g0)
    _check_quantize(g, r, -0.4, 0.4)


def test_quantize_special_values():
    neg, pos = -2.0, 2.0
    specials = [0.0, -0.0, 2.0, -2.0, np.nextafter(np.float32(2), np.float32(0)),
                np.nextafter(np.float32(-2), np.float32(0)), 4.0, -4.0, np.inf, -np.inf, np.nan,
                1e-45, -1e-45, 1e-38, 3.0e38, -3.0e38, 1.0, -1.0]
    vals = np.array(specials, np.float32)
    gg, rr = np.meshgrid(vals, vals, indexing="ij")
    g = torch.from_numpy(gg.reshape(-1).copy()).to(DEV)
    r = torch.from_numpy(rr.reshape(-1).copy()).to(DEV)
    _check_quantize(g, r, neg, pos)


def test_worked_example_on_gpu():
    g = torch.tensor([1.0, 2.5, -1.0, -3.0, 2.0, 0.5, 0.0, -2.0], device=DEV)
    r = torch.zeros(8, device=DEV)
    compr = _run_quantize(g, r, -2.0, 2.0)
    c = u32(compr)
    assert c[3] == 0x12420000
    assert c[:3].view(np.float32).tolist() == [-2.0, 2.0, 8.0]
    out = torch.empty(8, device=DEV)
    qga().qga_dequantize_2bit(compr, out)
    assert out.cpu().tolist() == [0.0, 2.0, 0.0, -2.0, 2.0, 0.0, 0.0, -2.0]


def test_error_feedback_1M():
    """The 2^20 workload: one generator seeded 0 redrawn for 10 iterations,
    residual from 0, thresholds +-0.5; every iteration's record, residual and
    dequantized vector match the oracle."""
    w = workloads.WORKLOADS["ef2bit-1M"]
    n = w.n
    grads = workloads.gradient_stream(w, w.iterations, device=DEV)
    r = torch.zeros(n, device=DEV)
    r_host = np.zeros(n, np.float32)
    out = torch.empty(n, device=DEV)
    compr = torch.empty(qga().qga_2bit_words(n), dtype=torch.int32, device=DEV)
    for it in range(w.iterations):
        g_host = f32(grads[it])
        qga().qga_quantize_2bit(grads[it], r, compr, w.neg_thr, w.pos_thr)
        qga().qga_dequantize_2bit(compr, out)
        want_c, r_host = oracle.quantize_2bit(g_host, r_host, w.neg_thr, w.pos_thr)
        assert np.array_equal(u32(compr), want_c), (it, first_diff(u32(compr), want_c))
        assert same_bits_f32(f32(r), r_host), it
        assert same_bits_f32(f32(out), oracle.dequantize_2bit(want_c, n)), it


def _random_record(n, neg, pos, seed, with_code_11=False):
    rng = np.random.default_rng(seed)
    words = rng.integers(0, 1 << 32, qga().qga_2bit_words(n), dtype=np.uint64).astype(np.uint32)
    if not with_code_11:
        p = words[3:].astype(np.uint64)
        p ^= (p & (p >> 1) & 0x55555555) << 1
        words[3:] = p.astype(np.uint32)
    words[:3] = np.array([neg, pos, n], np.float32).view(np.uint32)
    return words


def _dev_words(words):
    return torch.from_numpy(words.view(np.int32).copy()).to(DEV)


@pytest.mark.parametrize("n", [1, 15, 16, 17, 129, 513, 4097, (1 << 20) + 5])
@pytest.mark.parametrize("oo", [0, 1])
def test_dequantize(n, oo):
    words = _random_record(n, -0.75, 1.25, n, with_code_11=True)
    out = offset_view(n, torch.float32, oo, fill=float("nan"))
    qga().qga_dequantize_2bit(_dev_words(words), out)
    assert same_bits_f32(f32(out), oracle.dequantize_2bit(words, n))


@pytest.mark.parametrize("W", [1, 2, 3, 8, 9, 10, 17, 33, 64])
@pytest.mark.parametrize("n", [1, 17, 513, 4097, 65_537])
def test_dequant_accumulate(W, n):
    rng = np.random.default_rng(W * 1000 + n)
    recs = [_random_record(n, -float(a), float(b), 31 * w + n)
            for w, (a, b) in enumerate(rng.uniform(0.01, 2.0, (W, 2)).astype(np.float32))]
    out = offset_view(n, torch.float32, n % 3, fill=float("nan"))
    qga().qga_dequant_accumulate_2bit([_dev_words(r) for r in recs], out)
    want = oracle.dequant_accumulate_2bit(recs, n)
    got = f32(out)
    np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
    assert same_bits_f32(got, want), first_diff(got, want)


@pytest.mark.parametrize("W", [1, 2, 5, 8, 9, 16])
def test_dequant_accumulate_code_11_reads_as_zero(W):
    """Records holding the unused code 11 (never written by a quantize): it
    reads as +0 in the merge, for every worker count (the table merge clears
    it before forming an index, the per-worker merge decodes it as 0)."""
    n = 4099
    rng = np.random.default_rng(W)
    recs = [_random_record(n, -float(a), float(b), 77 * w + W, with_code_11=True)
            for w, (a, b) in enumerate(rng.uniform(0.01, 2.0, (W, 2)).astype(np.float32))]
    out = torch.empty(n, device=DEV)
    qga().qga_dequant_accumulate_2bit([_dev_words(r) for r in recs], out)
    want = oracle.dequant_accumulate_2bit(recs, n)
    assert same_bits_f32(f32(out), want), first_diff(f32(out), want)


@pytest.mark.parametrize("W", [2, 8, 9, 16])
def test_dequant_accumulate_shared_and_signed_zero_thresholds(W):
    """Thresholds shared by all workers, and -0 as a negative threshold
    (code 10 then adds -0, which leaves a +0 sum at +0)."""
    n = 1000
    recs = [_random_record(n, -0.0 if w % 2 else -0.5, 0.5, 5 * w) for w in range(W)]
    out = torch.empty(n, device=DEV)
    qga().qga_dequant_accumulate_2bit([_dev_words(r) for r in recs], out)
    want = oracle.dequant_accumulate_2bit(recs, n)
    assert same_bits_f32(f32(out), want), first_diff(f32(out), want)


def test_resnet50_four_workers_full():
    """ResNet-50-sized gradient, 4 workers with their own seeds and
    residuals: every word, residual and merged value checked."""
    w = workloads.WORKLOADS["resnet50-4w"]
    n = w.n
    comprs, want_recs = [], []
    for k in range(w.workers):
        g = workloads.gradient(w, k, 0, device=DEV)
        r = workloads.random_residual(n, w.pos_thr, 77 + k, device=DEV)
        g_host, r_host = f32(g), f32(r).copy()
        compr = torch.empty(qga().qga_2bit_words(n), dtype=torch.int32, device=DEV)
        qga().qga_quantize_2bit(g, r, compr, w.neg_thr, w.pos_thr)
        want_c, want_r = oracle.quantize_2bit(g_host, r_host, w.neg_thr, w.pos_thr)
        assert np.array_equal(u32(compr), want_c), (k, first_diff(u32(compr), want_c))
        assert same_bits_f32(f32(r), want_r), k
        comprs.append(compr)
        want_recs.append(want_c)
        del g, r
    out = torch.empty(n, device=DEV)
    qga().qga_dequant_accumulate_2bit(comprs, out)
    want = oracle.dequant_accumulate_2bit(want_recs, n)
    got = f32(out)
    np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
    assert same_bits_f32(got, want)


def test_vgg16_eight_workers_five_iterations_sampled():
    """The VGG16-sized workload at full size, in the launch configuration the
    benchmark times (8 workers, residual carried over 5 iterations).  A fixed
    sample of words is followed through all iterations: the oracle carries
    its OWN residual for the sampled elements (from the same zero start), and
    the GPU's sampled words, residuals and merged values must match it every
    iteration; the header and the ragged last word are in the sample."""
    w = workloads.WORKLOADS["vgg16-8w"]
    n = w.n
    q = qga()
    words = q.qga_2bit_words(n)
    res = [torch.zeros(n, device=DEV) for _ in range(w.workers)]
    comprs = [torch.empty(words, dtype=torch.int32, device=DEV) for _ in range(w.workers)]
    out = torch.empty(n, device=DEV)
    pick = sample_words(words - 3, 1500, seed=3)
    spans = [(int(k) * 16, min(int(k) * 16 + 16, n)) for k in pick]
    m_total = sum(b - a for a, b in spans)
    r_oracle = [np.zeros(m_total, np.float32) for _ in range(w.workers)]
    header = np.array([w.neg_thr, w.pos_thr, n], np.float32).view(np.uint32)
    for it in range(w.iterations):
        oracle_words = []
        for k in range(w.workers):
            g = workloads.gradient(w, k, it, device=DEV)
            g_s, _ = gather_elems(g, pick, 16, n)
            q.qga_quantize_2bit(g, res[k], comprs[k], w.neg_thr, w.pos_thr)
            r_gpu, _ = gather_elems(res[k], pick, 16, n)
            got_words = u32(comprs[k])
            assert np.array_equal(got_words[:3], header), got_words[:3]
            g_s, r_gpu = g_s.numpy(), r_gpu.numpy()
            rec_words = []
            at = 0
            for i, (a, b) in enumerate(spans):
                m = b - a
                want_c, want_r = oracle.quantize_2bit(g_s[at:at + m], r_oracle[k][at:at + m],
                                                      w.neg_thr, w.pos_thr)
                r_oracle[k][at:at + m] = want_r
                assert got_words[3 + pick[i]] == want_c[3], (it, k, int(pick[i]))
                assert same_bits_f32(r_gpu[at:at + m], want_r), (it, k, int(pick[i]))
                rec_words.append(want_c[3])
                at += m
            oracle_words.append(np.array(rec_words, np.uint32))
            del g
        q.qga_dequant_accumulate_2bit(comprs, out)
        got_out, _ = gather_elems(out, pick, 16, n)
        got_out = got_out.numpy()
        at = 0
        for i, (a, b) in enumerate(spans):
            m = b - a
            mini = [np.concatenate([np.array([w.neg_thr, w.pos_thr, m], np.float32).view(np.uint32),
                                    oracle_words[k][i:i + 1]]) for k in range(w.workers)]
            want = oracle.dequant_accumulate_2bit(mini, m)
            got = got_out[at:at + m]
            np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
            assert same_bits_f32(got, want), (it, int(pick[i]))
            at += m


def test_residual_checkpoint_resume():
    """The only state of the method is the caller's residual: saving it to
    the host mid-run and restoring it into a fresh buffer continues the run
    word for word."""
    q = qga()
    w = workloads.WORKLOADS["ef2bit-1M"]
    n = 100_003
    grads = workloads.gradient_stream(w, 6, device=DEV, n=n)
    words = q.qga_2bit_words(n)
    r = torch.zeros(n, device=DEV)
    c = torch.empty(words, dtype=torch.int32, device=DEV)
    for it in range(3):
        q.qga_quantize_2bit(grads[it], r, c, w.neg_thr, w.pos_thr)
    saved = r.cpu().clone()
    straight = []
    for it in range(3, 6):
        q.qga_quantize_2bit(grads[it], r, c, w.neg_thr, w.pos_thr)
        straight.append(u32(c).copy())
    r2 = saved.to(DEV)
    c2 = torch.empty(words, dtype=torch.int32, device=DEV)
    for k, it in enumerate(range(3, 6)):
        q.qga_quantize_2bit(grads[it], r2, c2, w.neg_thr, w.pos_thr)
        assert np.array_equal(u32(c2), straight[k]), it
    assert same_bits_f32(f32(r2), f32(r))
