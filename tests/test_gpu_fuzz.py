"""Seeded random sweep over the entry points: sizes (log-uniform, with the
ragged ends that exact tile counts never reach), alignments of every
pointer, thresholds (shared, per worker, signed zero), worker counts on both
sides of every kernel boundary (1-8 table merges, 9-16 and beyond), and the
bit widths.  Each case is compared with the oracle bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import DEV, f32, first_diff, offset_view, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu

CASES = 64


def _n(rng):
    return int(np.exp(rng.uniform(0.0, np.log(300_000)))) - 1


def _dev_view(values, dtype, offset):
    t = offset_view(values.size, dtype, offset)
    t.copy_(torch.from_numpy(values))
    return t


@pytest.mark.parametrize("case", range(CASES))
def test_fuzz_2bit_quantize_merge(case):
    q = qga()
    rng = np.random.default_rng(9000 + case)
    n = _n(rng)
    W = int(rng.choice([1, 2, 3, 5, 8, 9, 12, 16, 17, 33]))
    scale = float(10 ** rng.uniform(-4, 0))
    recs, want_recs = [], []
    for w in range(W):
        g = (rng.standard_normal(n) * scale).astype(np.float32)
        r = (rng.standard_normal(n) * scale * 0.3).astype(np.float32)
        pos = float(np.float32(scale * rng.uniform(0.2, 2.0)))
        neg = -0.0 if rng.random() < 0.1 else -float(np.float32(scale * rng.uniform(0.2, 2.0)))
        gd = _dev_view(g, torch.float32, int(rng.integers(0, 8)))
        rd = _dev_view(r, torch.float32, int(rng.integers(0, 8)))
        c = torch.empty(q.qga_2bit_words(n), dtype=torch.int32, device=DEV)
        q.qga_quantize_2bit(gd, rd, c, neg, pos)
        want_c, want_r = oracle.quantize_2bit(g, r, neg, pos)
        assert np.array_equal(u32(c), want_c), (case, w, first_diff(u32(c), want_c))
        assert same_bits_f32(f32(rd), want_r), (case, w)
        recs.append(c)
        want_recs.append(want_c)
    out = offset_view(n, torch.float32, int(rng.integers(0, 8)), fill=float("nan"))
    q.qga_dequant_accumulate_2bit(recs, out)
    want = oracle.dequant_accumulate_2bit(want_recs, n)
    assert same_bits_f32(f32(out), want), (case, n, W, first_diff(f32(out), want))
    q.qga_dequantize_2bit(recs[0], out)
    assert same_bits_f32(f32(out), oracle.dequantize_2bit(want_recs[0], n)), (case, n)


@pytest.mark.parametrize("case", range(CASES))
def test_fuzz_ternary_quantize_merge(case):
    q = qga()
    rng = np.random.default_rng(9100 + case)
    n = _n(rng)
    W = int(rng.choice([1, 2, 4, 7, 8, 9, 13, 16, 20]))
    recs, want_recs = [], []
    for w in range(W):
        g = (rng.standard_normal(n) * 0.5).astype(np.float32)
        r = np.zeros(n, np.float32)
        pos = float(np.float32(rng.uniform(0.1, 1.0)))
        neg = -float(np.float32(rng.uniform(0.1, 1.0)))
        gd = _dev_view(g, torch.float32, int(rng.integers(0, 8)))
        rd = _dev_view(r, torch.float32, int(rng.integers(0, 8)))
        c = torch.empty(q.qga_ternary_words(n), dtype=torch.int32, device=DEV)
        q.qga_quantize_ternary(gd, rd, c, neg, pos)
        want_c, want_r = oracle.quantize_ternary(g, r, neg, pos)
        assert np.array_equal(u32(c), want_c), (case, w)
        assert same_bits_f32(f32(rd), want_r), (case, w)
        recs.append(c)
        want_recs.append(want_c)
    out = offset_view(n, torch.float32, int(rng.integers(0, 8)), fill=float("nan"))
    q.qga_dequant_accumulate_ternary(recs, out)
    want = oracle.dequant_accumulate_ternary(want_recs, n)
    assert same_bits_f32(f32(out), want), (case, n, W, first_diff(f32(out), want))


@pytest.mark.parametrize("case", range(CASES))
def test_fuzz_qsgd(case):
    q = qga()
    rng = np.random.default_rng(9200 + case)
    n = max(1, _n(rng))
    W = int(rng.choice([1, 2, 3, 8, 9, 12, 16, 17, 24]))
    b = int(rng.choice([2, 4, 8]))
    grads = [_dev_view((rng.standard_normal(n) * rng.uniform(0.01, 3.0)).astype(np.float32), torch.float32,
                       int(rng.integers(0, 8))) for _ in range(W)]
    hosts = [f32(g) for g in grads]
    M = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max(grads, M)
    M_host = oracle.qsgd_mn_max(hosts)
    assert M.item() == M_host, case
    recs, want_recs = [], []
    for w in range(W):
        seed = int(rng.integers(0, 1 << 63))
        c = torch.empty(q.qga_qsgd_words(n, b), dtype=torch.int32, device=DEV)
        q.qga_qsgd_mn_quantize(grads[w], c, b, seed, M)
        want_c = oracle.qsgd_mn_quantize(hosts[w], b, seed, M_host)
        assert np.array_equal(u32(c), want_c), (case, w, first_diff(u32(c), want_c))
        recs.append(c)
        want_recs.append(want_c)
    out = offset_view(n, torch.float32, int(rng.integers(0, 8)), fill=float("nan"))
    q.qga_qsgd_mn_dequant_accumulate(recs, out, b)
    want = oracle.qsgd_mn_dequant_accumulate(want_recs, n, b)
    assert same_bits_f32(f32(out), want), (case, n, W, b, first_diff(f32(out), want))


@pytest.mark.parametrize("case", range(CASES))
def test_fuzz_qsgd_two_scales(case):
    q = qga()
    rng = np.random.default_rng(9300 + case)
    n = max(1, _n(rng))
    W = int(rng.choice([1, 2, 4, 8, 9, 16]))
    b1, b2 = (int(x) for x in rng.choice([2, 4, 8], 2))
    grads = [_dev_view((rng.standard_normal(n) * rng.uniform(0.01, 3.0)).astype(np.float32), torch.float32,
                       int(rng.integers(0, 8))) for _ in range(W)]
    hosts = [f32(g) for g in grads]
    M = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max(grads, M)
    M_host = oracle.qsgd_mn_max(hosts)
    recs, want_recs = [], []
    for w in range(W):
        seed = int(rng.integers(0, 1 << 63))
        c = torch.empty(q.qga_qsgd_mnts_words(n, b1, b2), dtype=torch.int32, device=DEV)
        q.qga_qsgd_mnts_quantize(grads[w], c, b1, b2, seed, M)
        want_c = oracle.qsgd_mnts_quantize(hosts[w], b1, b2, seed, M_host)
        assert np.array_equal(u32(c), want_c), (case, w, first_diff(u32(c), want_c))
        recs.append(c)
        want_recs.append(want_c)
    out = offset_view(n, torch.float32, int(rng.integers(0, 8)), fill=float("nan"))
    q.qga_qsgd_mnts_dequant_accumulate(recs, out, b1, b2)
    want = oracle.qsgd_mnts_dequant_accumulate(want_recs, n, b1, b2)
    assert same_bits_f32(f32(out), want), (case, n, W, b1, b2, first_diff(f32(out), want))
