"""Sizes past the 32-bit element range: every index of the kernels is 64-bit.
n = 2^31 + 37 elements (8.6 GB per fp32 buffer); sampled words near the
start, around 2^31 and at the ragged end are checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import AGG_ATOL, AGG_RTOL, DEV, f32, gather_elems, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu

N = (1 << 31) + 37


def _pick(nwords):
    k31 = (1 << 31) // 16
    idx = {0, 1, nwords - 1, nwords - 2, k31 - 1, k31, k31 + 1}
    idx |= set(np.random.default_rng(1).integers(0, nwords, 200).tolist())
    return np.array(sorted(i for i in idx if 0 <= i < nwords), np.int64)


@pytest.fixture(scope="module")
def big():
    free, _ = torch.cuda.mem_get_info()
    if free < 40e9:
        pytest.skip("needs 40 GB of free device memory")
    gen = torch.Generator(device=DEV)
    gen.manual_seed(31)
    g = torch.randn(N, device=DEV, generator=gen)
    yield g
    del g
    torch.cuda.empty_cache()


def test_quantize_and_merge_past_2_31(big):
    q = qga()
    g = big
    words = q.qga_2bit_words(N)
    pick = _pick(words - 3)
    spans = [(int(k) * 16, min(int(k) * 16 + 16, N)) for k in pick]
    recs, want_words = [], []
    for w, (neg, pos) in enumerate([(-0.5, 0.5), (-1.0, 0.75)]):
        r = torch.zeros(N, device=DEV)
        c = torch.empty(words, dtype=torch.int32, device=DEV)
        q.qga_quantize_2bit(g, r, c, neg, pos)
        g_s, _ = gather_elems(g, pick, 16, N)
        r_s, _ = gather_elems(r, pick, 16, N)
        got = u32(c.index_select(0, torch.from_numpy(pick + 3).to(DEV)))
        g_s, r_s = g_s.numpy(), r_s.numpy()
        at, mine = 0, []
        for i, (a, b) in enumerate(spans):
            m = b - a
            wc, wr = oracle.quantize_2bit(g_s[at:at + m], np.zeros(m, np.float32), neg, pos)
            assert got[i] == wc[3], (w, int(pick[i]))
            assert same_bits_f32(r_s[at:at + m], wr), (w, int(pick[i]))
            mine.append(wc[3])
            at += m
        want_words.append((neg, pos, np.array(mine, np.uint32)))
        recs.append(c)
        del r
    out = torch.empty(N, device=DEV)
    q.qga_dequant_accumulate_2bit(recs, out)
    o_s, _ = gather_elems(out, pick, 16, N)
    o_s = o_s.numpy()
    at = 0
    for i, (a, b) in enumerate(spans):
        m = b - a
        mini = [np.concatenate([np.array([neg, pos, m], np.float32).view(np.uint32), ww[i:i + 1]])
                for neg, pos, ww in want_words]
        want = oracle.dequant_accumulate_2bit(mini, m)
        np.testing.assert_allclose(o_s[at:at + m], want, rtol=AGG_RTOL, atol=AGG_ATOL)
        assert same_bits_f32(o_s[at:at + m], want), int(pick[i])
        at += m


def test_qsgd_past_2_31(big):
    """QSGD codes at global element indices above 2^31 (the Philox counter
    is the element index divided by 4) against the oracle's levels."""
    q = qga()
    g = big
    b = 2
    M = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max([g], M)
    assert M.item() == g.abs().max().item()
    Mf = np.float32(M.item())
    c = torch.empty(q.qga_qsgd_words(N, b), dtype=torch.int32, device=DEV)
    q.qga_qsgd_mn_quantize(g, c, b, 77, M)
    per = 32 // b
    nwords = q.qga_qsgd_words(N, b) - 3
    pick = np.unique(np.array([0, nwords - 1, (1 << 31) // per, (1 << 31) // per - 1] +
                              np.random.default_rng(2).integers(0, nwords, 100).tolist()))
    elems = (pick[:, None] * per + np.arange(per)[None, :]).reshape(-1)
    elems = elems[elems < N]
    g_s = f32(g.index_select(0, torch.from_numpy(elems).to(DEV)))
    words = u32(c.index_select(0, torch.from_numpy(pick + 3).to(DEV)))
    got = {}
    for wd, k in zip(words, pick):
        for i in range(per):
            d = (int(wd) >> (32 - b * (i + 1))) & ((1 << b) - 1)
            got[int(k) * per + i] = d - (1 << b) if d >= (1 << (b - 1)) else d
    for e, gv in zip(elems, g_s):
        assert got[int(e)] == oracle.qsgd_level(gv, Mf, b, 77, int(e)), int(e)


def test_fused_reducing_step_past_2_31(big):
    """The reducing worker's fused quantize + merge at n = 2^31 + 37: its own
    record words, residuals and the merged values at sampled words near 0,
    around 2^31 and at the ragged end, against the oracle."""
    q = qga()
    g = big
    words = q.qga_2bit_words(N)
    pick = _pick(words - 3)
    spans = [(int(k) * 16, min(int(k) * 16 + 16, N)) for k in pick]
    other_thr, own_thr = (-1.0, 0.75), (-0.5, 0.5)
    # worker 0: a record made by the plain quantize (its words are checked there)
    r0 = torch.zeros(N, device=DEV)
    c0 = torch.empty(words, dtype=torch.int32, device=DEV)
    q.qga_quantize_2bit(g, r0, c0, *other_thr)
    del r0
    # worker 1 reduces: its own quantize (residual starts at 0) + the merge of both
    r1 = torch.zeros(N, device=DEV)
    c1 = torch.empty(words, dtype=torch.int32, device=DEV)
    out = torch.empty(N, device=DEV)
    q.qga_quantize_merge_2bit(g, r1, [c0, c1], 1, *own_thr, out)
    g_s, _ = gather_elems(g, pick, 16, N)
    r_s, _ = gather_elems(r1, pick, 16, N)
    o_s, _ = gather_elems(out, pick, 16, N)
    got1 = u32(c1.index_select(0, torch.from_numpy(pick + 3).to(DEV)))
    g_s, r_s, o_s = g_s.numpy(), r_s.numpy(), o_s.numpy()
    at = 0
    for i, (a, b) in enumerate(spans):
        m = b - a
        w0, _ = oracle.quantize_2bit(g_s[at:at + m], np.zeros(m, np.float32), *other_thr)
        w1, wr = oracle.quantize_2bit(g_s[at:at + m], np.zeros(m, np.float32), *own_thr)
        assert got1[i] == w1[3], int(pick[i])
        assert same_bits_f32(r_s[at:at + m], wr), int(pick[i])
        want = oracle.dequant_accumulate_2bit([w0, w1], m)
        assert same_bits_f32(o_s[at:at + m], want), int(pick[i])
        at += m
    del r1, c1, c0, out


def test_grandk_coordinates_past_2_31(big):
    """GRandK-MaxNorm with kept coordinates on both sides of 2^31."""
    q = qga()
    g = big
    rng = np.random.default_rng(3)
    index = np.unique(np.concatenate([rng.integers(0, N, 600), (1 << 31) + np.arange(-20, 20),
                                      [N - 1, 0]])).astype(np.int64)
    rng.shuffle(index)
    idx = torch.from_numpy(index).to(DEV)
    M = torch.empty(1, device=DEV)
    q.qga_grandk_mn_max([g], idx, M)
    kept = f32(g.index_select(0, idx))
    ident = np.arange(index.size, dtype=np.int64)
    want_M = oracle.grandk_mn_max([kept], ident)
    assert M.item() == want_M
    for b in (2, 8):
        c = torch.empty(q.qga_qsgd_words(index.size, b), dtype=torch.int32, device=DEV)
        q.qga_grandk_mn_quantize(g, idx, c, b, 99, M)
        want = oracle.grandk_mn_quantize(kept, ident, b, 99, want_M)
        assert np.array_equal(u32(c), want), b
