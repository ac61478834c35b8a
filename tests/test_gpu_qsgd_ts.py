"""GPU parity of QSGD-MaxNorm with two scales (QSGD-MN-TS) against the CPU
oracle: both sub-records bit for bit (headers, coarse and fine codes) and the
merged values bit for bit (each scale's level sum is an integer) and within
1e-6 relative + 1e-7 absolute."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import AGG_ATOL, AGG_RTOL, DEV, f32, first_diff, offset_view, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu

PAIRS = [(b1, b2) for b1 in (2, 4, 8) for b2 in (2, 4, 8)]


def _grads(W, n, seed, offsets=None, scale=2.0, outliers=True):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    out = []
    for w in range(W):
        g = offset_view(n, torch.float32, offsets[w] if offsets else 0)
        g.copy_(torch.randn(n, device=DEV, generator=gen) * scale)
        if outliers and n > 50:
            g[::97] = 50.0 * (1 - 2 * (w % 2))
        out.append(g)
    return out


def _max(grads):
    M = torch.empty(1, device=DEV)
    qga().qga_qsgd_mn_max(grads, M)
    want = oracle.qsgd_mn_max([f32(g) for g in grads])
    assert M.item() == want
    return M, want


@pytest.mark.parametrize("b1,b2", PAIRS)
@pytest.mark.parametrize("n", [0, 1, 3, 5, 16, 17, 33, 127, 513, 4097, 65_537, (1 << 20) + 7])
def test_quantize(b1, b2, n):
    q = qga()
    (g,) = _grads(1, n, 300 + n)
    if n:
        M, M_host = _max([g])
    else:
        M, M_host = torch.ones(1, device=DEV), np.float32(1.0)
    seed = 0xFEDC_BA98_7654_3210 + n
    words = q.qga_qsgd_mnts_words(n, b1, b2)
    assert words == oracle.qsgd_mnts_words(n, b1, b2)
    buf = torch.full((words + 4,), -1, dtype=torch.int32, device=DEV)
    buf[words:] = 0x5A5A5A5A
    q.qga_qsgd_mnts_quantize(g, buf[:words], b1, b2, seed, M)
    got = u32(buf)
    assert (got[words:] == 0x5A5A5A5A).all()
    want = oracle.qsgd_mnts_quantize(f32(g), b1, b2, seed, M_host)
    assert np.array_equal(got[:words], want), first_diff(got[:words], want)


@pytest.mark.parametrize("b1,b2", PAIRS)
def test_quantize_boundary_misaligned_and_special(b1, b2):
    """Elements on the scale boundary |g| = M / s1 and one ulp either side,
    level boundaries of both scales, specials; a misaligned gradient."""
    q = qga()
    s1 = 2 ** (b1 - 1) - 1
    M = np.float32(50.0)
    M2 = oracle.qsgd_mnts_fine_scale(M, b1)
    vals = [0.0, -0.0, 50.0, -50.0, 1e-40, -1e-40, M2, -M2, np.nextafter(M2, np.float32(99)),
            np.nextafter(M2, np.float32(0)), -np.nextafter(M2, np.float32(99)), 60.0,
            float("nan"), float("inf"), -float("inf"), 25.0, M2 / 2, M2 / 3]
    rng = np.random.default_rng(b1 * 10 + b2)
    # values whose scaled level lies within 2^-10 of an integer on either scale
    for scale, s in ((M, s1), (M2, 2 ** (b2 - 1) - 1)):
        for j in range(1, s + 1):
            for d in (-1e-3, -1e-5, -1e-7, 1e-7, 1e-5):
                vals.append(float(scale) * (j - 0.5 + d) / s)
    vals = np.array(vals + list(rng.standard_normal(500) * 8), np.float32)
    n = vals.size
    g = offset_view(n, torch.float32, 1)
    g.copy_(torch.from_numpy(vals))
    Md = torch.tensor([M], device=DEV)
    words = q.qga_qsgd_mnts_words(n, b1, b2)
    c = torch.empty(words, dtype=torch.int32, device=DEV)
    for seed in (42, 43, 2 ** 63 + 5):
        q.qga_qsgd_mnts_quantize(g, c, b1, b2, seed, Md)
        want = oracle.qsgd_mnts_quantize(vals, b1, b2, seed, M)
        assert np.array_equal(u32(c), want), first_diff(u32(c), want)
    # M == 0: every level is 0
    Md.zero_()
    q.qga_qsgd_mnts_quantize(g, c, b1, b2, 42, Md)
    assert np.array_equal(u32(c), oracle.qsgd_mnts_quantize(vals, b1, b2, 42, np.float32(0.0)))


@pytest.mark.parametrize("b1,b2", PAIRS)
@pytest.mark.parametrize("W", [1, 2, 3, 5, 8, 9, 13, 16, 17, 64])
@pytest.mark.parametrize("n", [1, 17, 513, 65_537])
def test_merge(b1, b2, W, n):
    q = qga()
    grads = _grads(W, n, 7 * W + n)
    M, M_host = _max(grads)
    words = q.qga_qsgd_mnts_words(n, b1, b2)
    recs, want_recs = [], []
    for w, g in enumerate(grads):
        c = torch.empty(words, dtype=torch.int32, device=DEV)
        q.qga_qsgd_mnts_quantize(g, c, b1, b2, 1234 + w, M)
        want_c = oracle.qsgd_mnts_quantize(f32(g), b1, b2, 1234 + w, M_host)
        assert np.array_equal(u32(c), want_c), w
        recs.append(c)
        want_recs.append(want_c)
    # odd worker counts write an aligned output, even ones a misaligned one
    out = offset_view(n, torch.float32, 0 if W % 2 else 1 + n % 3, fill=float("nan"))
    q.qga_qsgd_mnts_dequant_accumulate(recs, out, b1, b2)
    want = oracle.qsgd_mnts_dequant_accumulate(want_recs, n, b1, b2)
    got = f32(out)
    np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
    assert same_bits_f32(got, want), first_diff(got, want)


@pytest.mark.parametrize("b1,b2", [(2, 4), (4, 8), (8, 2)])
@pytest.mark.parametrize("W", [1, 2, 3, 4, 5, 6, 7, 8, 9, 12, 16, 17])
def test_merge_random_records(b1, b2, W):
    """Arbitrary bit patterns in both sub-records (every level value, both
    signs, on both scales at once) merge as the oracle merges them, for every
    worker count of the compile-time kernels and beyond."""
    q = qga()
    n = 4099 + 32 * W
    rng = np.random.default_rng(b1 * 16 + b2 + 1000 * W)
    words = q.qga_qsgd_mnts_words(n, b1, b2)
    w1 = 3 + -(-(n * b1) // 32)
    recs = []
    for w in range(W):
        r = rng.integers(0, 1 << 32, words, dtype=np.uint64).astype(np.uint32)
        r[0] = np.float32(3.0).view(np.uint32)
        r[1], r[2] = np.float32(b1).view(np.uint32), np.float32(n).view(np.uint32)
        r[w1] = np.float32(3.0 / (2 ** (b1 - 1) - 1)).view(np.uint32)
        r[w1 + 1], r[w1 + 2] = np.float32(b2).view(np.uint32), np.float32(n).view(np.uint32)
        recs.append(r)
    out = torch.empty(n, device=DEV)
    q.qga_qsgd_mnts_dequant_accumulate([torch.from_numpy(r.view(np.int32)).to(DEV) for r in recs],
                                       out, b1, b2)
    want = oracle.qsgd_mnts_dequant_accumulate(recs, n, b1, b2)
    assert same_bits_f32(f32(out), want), first_diff(f32(out), want)


def _levels_of_word(word, b):
    per = 32 // b
    out = []
    for i in range(per):
        d = (int(word) >> (32 - b * (i + 1))) & ((1 << b) - 1)
        out.append(d - (1 << b) if d >= (1 << (b - 1)) else d)
    return out


def _pack(levels, b):
    per = 32 // b
    words = np.zeros(-(-len(levels) // per), np.uint32)
    for e, q in enumerate(levels):
        words[e // per] |= np.uint32((int(q) & ((1 << b) - 1)) << (32 - b * (e % per + 1)))
    return words


def test_workload_sampled():
    """The 8 x 2^27 QSGD workload (0.1% outliers of 50) with (b1, b2) = (4, 8),
    in the bench's launch configuration: M exact; headers; the levels of 300
    sampled 32-element spans of every worker's both sub-records against the
    oracle's per-element levels at those positions; the merged values there
    against the oracle's merge of the sampled levels."""
    q = qga()
    wq = workloads.WORKLOADS["qsgd-128M-8w"]
    n, W, b1, b2 = wq.n, wq.workers, 4, 8
    grads = [workloads.gradient(wq, k, 0, device=DEV) for k in range(W)]
    M = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max(grads, M)
    Mf = np.float32(workloads.QSGD_OUTLIER_MAGNITUDE)
    assert M.item() == Mf
    M2 = oracle.qsgd_mnts_fine_scale(Mf, b1)
    words = q.qga_qsgd_mnts_words(n, b1, b2)
    w1 = 3 + (n * b1 + 31) // 32
    rng = np.random.default_rng(17)
    spans = np.unique(np.concatenate([[0, n // 32 - 1], rng.integers(0, n // 32, 300)]))
    elems = (spans[:, None] * 32 + np.arange(32)[None, :]).reshape(-1)
    idx = torch.from_numpy(elems).to(DEV)
    k1 = (spans[:, None] * (b1 // 1) + np.arange(b1)[None, :]).reshape(-1)   # 32 elements = b1 words
    k2 = (spans[:, None] * b2 + np.arange(b2)[None, :]).reshape(-1)
    recs, minis = [], []
    for w in range(W):
        c = torch.empty(words, dtype=torch.int32, device=DEV)
        seed = workloads.QSGD_SEED_BASE + w
        q.qga_qsgd_mnts_quantize(grads[w], c, b1, b2, seed, M)
        recs.append(c)
        head1 = u32(c[:3])
        head2 = u32(c[w1:w1 + 3])
        assert np.array_equal(head1, np.array([Mf, b1, n], np.float32).view(np.uint32))
        assert np.array_equal(head2, np.array([M2, b2, n], np.float32).view(np.uint32))
        got1 = [lv for wd in u32(c.index_select(0, torch.from_numpy(3 + k1).to(DEV)))
                for lv in _levels_of_word(wd, b1)]
        got2 = [lv for wd in u32(c.index_select(0, torch.from_numpy(w1 + 3 + k2).to(DEV)))
                for lv in _levels_of_word(wd, b2)]
        g_s = f32(grads[w].index_select(0, idx))
        want = [oracle.qsgd_mnts_levels(g_s[i], Mf, b1, b2, seed, int(e)) for i, e in enumerate(elems)]
        want1 = [a for a, _ in want]
        want2 = [b for _, b in want]
        assert got1 == want1, (w, first_diff(np.array(got1), np.array(want1)))
        assert got2 == want2, (w, first_diff(np.array(got2), np.array(want2)))
        m = elems.size
        minis.append(np.concatenate([np.array([Mf, b1, m], np.float32).view(np.uint32), _pack(want1, b1),
                                     np.array([M2, b2, m], np.float32).view(np.uint32), _pack(want2, b2)]))
    assert any(any(lv) for lv in [want1]) and any(want2)
    out = torch.empty(n, device=DEV)
    q.qga_qsgd_mnts_dequant_accumulate(recs, out, b1, b2)
    got = f32(out.index_select(0, idx))
    want = oracle.qsgd_mnts_dequant_accumulate(minis, elems.size, b1, b2)
    np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
    assert same_bits_f32(got, want)
