"""GPU parity of QSGD-MaxNorm (max, b-bit quantize, integer-sum merge)
against the CPU oracle: M exact, codes bit for bit, merged values bit for bit
(the level sum is an integer, so the order of workers cannot matter) and
within 1e-6 relative + 1e-7 absolute."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import AGG_ATOL, AGG_RTOL, DEV, f32, first_diff, offset_view, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu

BITS = [2, 4, 8]


def _grads(W, n, seed, offsets=None, scale=2.0):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    out = []
    for w in range(W):
        g = offset_view(n, torch.float32, offsets[w] if offsets else 0)
        g.copy_(torch.randn(n, device=DEV, generator=gen) * scale)
        out.append(g)
    return out


@pytest.mark.parametrize("W", [1, 3, 8, 64])
@pytest.mark.parametrize("n", [1, 3, 17, 4097, 1_000_003])
def test_max(W, n):
    grads = _grads(W, n, W * 7 + n, offsets=[w % 3 for w in range(W)])
    M = torch.full((1,), -1.0, device=DEV)
    qga().qga_qsgd_mn_max(grads, M)
    want = oracle.qsgd_mn_max([f32(g) for g in grads])
    assert M.item() == want
    assert M.item() == torch.stack([g.abs().max() for g in grads]).max().item()


def test_max_special_values():
    g = torch.tensor([0.0, -0.0, float("nan"), -3.5, 1.0, float("nan")], device=DEV)
    M = torch.zeros(1, device=DEV)
    qga().qga_qsgd_mn_max([g], M)
    assert M.item() == 3.5 == oracle.qsgd_mn_max([f32(g)])
    z = torch.zeros(1000, device=DEV)
    M.fill_(7.0)
    qga().qga_qsgd_mn_max([z, z], M)
    assert M.item() == 0.0


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("n", [0, 1, 3, 4, 5, 15, 16, 17, 31, 33, 127, 129, 513, 4097, 65_537,
                               (1 << 20) + 7])
def test_quantize(b, n):
    q = qga()
    (g,) = _grads(1, n, 100 + n)
    g_host = f32(g)
    M = torch.empty(1, device=DEV)
    if n:
        q.qga_qsgd_mn_max([g], M)
        M_oracle = oracle.qsgd_mn_max([g_host])
        assert M.item() == M_oracle
    else:
        M.fill_(1.0)
        M_oracle = np.float32(1.0)
    seed = 0x1234_5678_9ABC_DEF0 + n
    words = q.qga_qsgd_words(n, b)
    buf = torch.full((words + 4,), -1, dtype=torch.int32, device=DEV)
    buf[words:] = 0x5A5A5A5A
    q.qga_qsgd_mn_quantize(g, buf[:words], b, seed, M)
    got = u32(buf)
    assert (got[words:] == 0x5A5A5A5A).all()
    want = oracle.qsgd_mn_quantize(g_host, b, seed, M_oracle)
    assert np.array_equal(got[:words], want), first_diff(got[:words], want)


@pytest.mark.parametrize("b", BITS)
def test_quantize_misaligned_and_special(b):
    q = qga()
    vals = np.array([0.0, -0.0, 50.0, -50.0, 1e-40, -1e-40, 49.999996, -0.5, 25.0, 12.5, 60.0,
                     float("nan"), float("inf")], np.float32)
    n = vals.size
    g = offset_view(n, torch.float32, 1)
    g.copy_(torch.from_numpy(vals))
    M = torch.tensor([50.0], device=DEV)
    words = q.qga_qsgd_words(n, b)
    c = torch.empty(words, dtype=torch.int32, device=DEV)
    q.qga_qsgd_mn_quantize(g, c, b, 42, M)
    assert np.array_equal(u32(c), oracle.qsgd_mn_quantize(vals, b, 42, np.float32(50.0)))
    # M == 0: every level is 0
    M.zero_()
    q.qga_qsgd_mn_quantize(g, c, b, 42, M)
    assert np.array_equal(u32(c), oracle.qsgd_mn_quantize(vals, b, 42, np.float32(0.0)))
    assert not u32(c)[3:].any()


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("W", [1, 2, 3, 5, 7, 8, 9, 12, 16, 17, 64])
@pytest.mark.parametrize("n", [1, 17, 513, 65_537])
def test_merge(b, W, n):
    q = qga()
    grads = _grads(W, n, 1000 * b + W + n)
    hosts = [f32(g) for g in grads]
    M = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max(grads, M)
    M_oracle = oracle.qsgd_mn_max(hosts)
    assert M.item() == M_oracle
    comprs, want_recs = [], []
    for w, g in enumerate(grads):
        c = torch.empty(q.qga_qsgd_words(n, b), dtype=torch.int32, device=DEV)
        q.qga_qsgd_mn_quantize(g, c, b, 1234 + w, M)
        comprs.append(c)
        want_recs.append(oracle.qsgd_mn_quantize(hosts[w], b, 1234 + w, M_oracle))
        assert np.array_equal(u32(c), want_recs[-1])
    out = offset_view(n, torch.float32, n % 3, fill=float("nan"))
    q.qga_qsgd_mn_dequant_accumulate(comprs, out, b)
    want = oracle.qsgd_mn_dequant_accumulate(want_recs, n, b)
    got = f32(out)
    np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
    assert same_bits_f32(got, want), first_diff(got, want)


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("W", [1, 2, 3, 4, 5, 6, 7, 8, 9, 11, 15, 16, 17, 64])
def test_merge_random_records(b, W):
    """Arbitrary bit patterns as records (every b-bit field value, -2^(b-1)
    included, which no quantize writes) merge as the oracle merges them, for
    every worker count of the compile-time kernels and beyond; n ragged and
    the output misaligned for one worker count."""
    q = qga()
    n = 4099 + 16 * W
    rng = np.random.default_rng(100 * b + W)
    words = q.qga_qsgd_words(n, b)
    recs = []
    for w in range(W):
        r = rng.integers(0, 1 << 32, words, dtype=np.uint64).astype(np.uint32)
        r[0] = np.float32(0.75).view(np.uint32)
        r[1], r[2] = np.float32(b).view(np.uint32), np.float32(n).view(np.uint32)
        recs.append(r)
    out = offset_view(n, torch.float32, 1 if W == 5 else 0, fill=float("nan"))
    q.qga_qsgd_mn_dequant_accumulate([torch.from_numpy(r.view(np.int32)).to(DEV) for r in recs], out, b)
    want = oracle.qsgd_mn_dequant_accumulate(recs, n, b)
    assert same_bits_f32(f32(out), want), first_diff(f32(out), want)


def _levels_of_word(word, b):
    per = 32 // b
    out = []
    for i in range(per):
        d = (int(word) >> (32 - b * (i + 1))) & ((1 << b) - 1)
        out.append(d - (1 << b) if d >= (1 << (b - 1)) else d)
    return out


def _pack_levels(levels, b):
    """Oracle levels -> record words (test plumbing: the layout only)."""
    per = 32 // b
    words = []
    for i in range(0, len(levels), per):
        wd = 0
        for j, lv in enumerate(levels[i:i + per]):
            wd |= (int(lv) & ((1 << b) - 1)) << (32 - b * (j + 1))
        words.append(wd)
    return np.array(words, np.uint32)


def test_qsgd_128M_eight_workers_sampled():
    """The QSGD workload at full size (2^27 elements, 0.1% outliers of 50,
    8 workers, seeds 1234 + w): M is exactly 50 and equals torch's max|g|;
    for b = 2, 4, 8, sampled words decode to the oracle's levels at their
    global element indices, and sampled merged values match the oracle."""
    w = workloads.WORKLOADS["qsgd-128M-8w"]
    n = w.n
    q = qga()
    grads = [workloads.gradient(w, k, 0, device=DEV) for k in range(w.workers)]
    M = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max(grads, M)
    # the planted outliers fix M (an input-recipe value, not a GPU result)
    Mf = np.float32(workloads.QSGD_OUTLIER_MAGNITUDE)
    assert M.item() == Mf
    assert M.item() == max(g.abs().max().item() for g in grads)
    rng = np.random.default_rng(5)
    for b in w.bits:
        per = 32 // b
        nwords = q.qga_qsgd_words(n, b) - 3
        pick = np.unique(np.concatenate([[0, nwords - 1], rng.integers(0, nwords, 300)]))
        elems = (pick[:, None] * per + np.arange(per)[None, :]).reshape(-1)
        idx = torch.from_numpy(elems).to(DEV)
        comprs = []
        mini_records = []
        for k, g in enumerate(grads):
            c = torch.empty(q.qga_qsgd_words(n, b), dtype=torch.int32, device=DEV)
            q.qga_qsgd_mn_quantize(g, c, b, workloads.QSGD_SEED_BASE + k, M)
            comprs.append(c)
            header = u32(c[:3])
            assert np.array_equal(header, np.array([Mf, b, n], np.float32).view(np.uint32))
            words = u32(c.index_select(0, torch.from_numpy(pick + 3).to(DEV)))
            g_s = f32(g.index_select(0, idx))
            got_levels = np.array([lv for wd in words for lv in _levels_of_word(wd, b)])
            want_levels = np.array([oracle.qsgd_level(g_s[i], Mf, b, workloads.QSGD_SEED_BASE + k,
                                                      int(e)) for i, e in enumerate(elems)])
            assert np.array_equal(got_levels, want_levels), (b, k, first_diff(got_levels, want_levels))
            assert np.abs(got_levels).max() <= 2 ** (b - 1) - 1
            packed = _pack_levels(want_levels, b)
            assert [lv for wd in packed for lv in _levels_of_word(wd, b)] == want_levels.tolist()
            head = np.array([Mf, b, elems.size], np.float32).view(np.uint32)
            mini_records.append(np.concatenate([head, packed]))
        out = torch.empty(n, device=DEV)
        q.qga_qsgd_mn_dequant_accumulate(comprs, out, b)
        got = f32(out.index_select(0, idx))
        want = oracle.qsgd_mn_dequant_accumulate(mini_records, elems.size, b)
        np.testing.assert_allclose(got, want, rtol=AGG_RTOL, atol=AGG_ATOL)
        assert same_bits_f32(got, want)
        del comprs


@pytest.mark.parametrize("b", BITS)
def test_quantize_levels_next_to_integer_boundaries(b):
    """Inputs placed so that |g|/M*s + u falls just above or below an integer
    (within 1e-7 .. 2e-4 of it), where a shortcut in the level computation
    would first disagree with the definition's three operations."""
    q = qga()
    s = 2 ** (b - 1) - 1
    M = np.float32(3.0)
    seed = 987654321
    n = 4096
    rng = np.random.default_rng(b)
    # The fast level differs from the definition's t by at most 3.8e-5 and
    # defers to the definition within 2^-14 = 6.1e-5 of an integer: distances
    # below, inside and above that band, and on both sides of the margin.
    deltas = np.array([1e-7, -1e-7, 3e-6, -3e-6, 2e-5, -2e-5, 3.7e-5, -3.7e-5, 3.9e-5, -3.9e-5,
                       4.5e-5, -4.5e-5, 5.5e-5, -5.5e-5, 6.0e-5, -6.0e-5, 6.2e-5, -6.2e-5, 7e-5, -7e-5,
                       1e-4, -2e-4, 1.3e-4, -1.3e-4, 3e-4, -3e-4])
    g = np.empty(n, np.float32)
    for e in range(n):
        u = oracle.qsgd_uniform(seed, e)
        target = rng.integers(0, s + 1) + deltas[e % deltas.size]
        x = np.float32(max(0.0, (target - u)) * float(M) / s)
        g[e] = -x if rng.random() < 0.5 else x
    g[:2] = [float(M), -float(M)]
    dev_g = torch.from_numpy(g).to(DEV)
    Md = torch.tensor([float(M)], device=DEV)
    c = torch.empty(q.qga_qsgd_words(n, b), dtype=torch.int32, device=DEV)
    q.qga_qsgd_mn_quantize(dev_g, c, b, seed, Md)
    want = oracle.qsgd_mn_quantize(g, b, seed, M)
    assert np.array_equal(u32(c), want), first_diff(u32(c), want)


@pytest.mark.parametrize("b", BITS)
def test_quantize_16M_full(b):
    """Every code of 2^24 elements spread over all levels (|g| uniform up to
    M, both signs) against the oracle."""
    q = qga()
    n = 1 << 24
    gen = torch.Generator(device=DEV)
    gen.manual_seed(1000 + b)
    g = (torch.rand(n, device=DEV, generator=gen) * 2 - 1) * 6.0
    M = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max([g], M)
    g_host = f32(g)
    M_or = oracle.qsgd_mn_max([g_host])
    assert M.item() == M_or
    c = torch.empty(q.qga_qsgd_words(n, b), dtype=torch.int32, device=DEV)
    q.qga_qsgd_mn_quantize(g, c, b, 2024 + b, M)
    want = oracle.qsgd_mn_quantize(g_host, b, 2024 + b, M_or)
    assert np.array_equal(u32(c), want), first_diff(u32(c), want)
