"""GPU parity of the reducing worker's fused step (quantize its own gradient,
merge all W records, one launch) through the C ABI: the own record and
residual bit for bit against the oracle's quantize, the aggregate bit for
bit against the oracle's merge of all W records, the other records left
untouched, and equality with the library's two separate calls."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import DEV, f32, first_diff, offset_view, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu


def _record(n, neg, pos, seed):
    rng = np.random.default_rng(seed)
    words = rng.integers(0, 1 << 32, 3 + (n + 15) // 16, dtype=np.uint64).astype(np.uint32)
    words[:3] = np.array([neg, pos, n], np.float32).view(np.uint32)
    return words


def _dev(words):
    return torch.from_numpy(words.view(np.int32).copy()).to(DEV)


def _case(n, W, own, seed, offsets=(0, 0, 0)):
    q = qga()
    rng = np.random.default_rng(seed)
    thr = rng.uniform(0.05, 1.5, (W, 2)).astype(np.float32)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    g = offset_view(n, torch.float32, offsets[0])
    r = offset_view(n, torch.float32, offsets[1])
    g.copy_(torch.randn(n, device=DEV, generator=gen) * 0.8)
    r.copy_(torch.rand(n, device=DEV, generator=gen) - 0.5)
    g_host, r_host = f32(g).copy(), f32(r).copy()
    recs = [_record(n, -float(thr[w, 0]), float(thr[w, 1]), seed * 100 + w) for w in range(W)]
    dev_recs = [_dev(x) for x in recs]
    out = offset_view(n, torch.float32, offsets[2], fill=float("nan"))
    neg, pos = -float(thr[own, 0]), float(thr[own, 1])
    q.qga_quantize_merge_2bit(g, r, dev_recs, own, neg, pos, out)
    torch.cuda.synchronize()
    want_c, want_r = oracle.quantize_2bit(g_host, r_host, neg, pos)
    got_c = u32(dev_recs[own])
    assert np.array_equal(got_c, want_c), first_diff(got_c, want_c)
    assert same_bits_f32(f32(r), want_r), first_diff(f32(r), want_r)
    for w in range(W):
        if w != own:
            assert np.array_equal(u32(dev_recs[w]), recs[w]), w
    merged = list(recs)
    merged[own] = want_c
    want = oracle.dequant_accumulate_2bit(merged, n)
    got = f32(out)
    assert same_bits_f32(got, want), first_diff(got, want)


@pytest.mark.parametrize("n", [1, 15, 16, 17, 1023, 1024, 1025, 65_537, (1 << 20) + 3])
@pytest.mark.parametrize("W,own", [(1, 0), (2, 1), (3, 0), (8, 0), (8, 5), (9, 8), (17, 3)])
def test_quantize_merge(n, W, own):
    _case(n, W, own, seed=n * 31 + W * 7 + own)


@pytest.mark.parametrize("offsets", [(1, 0, 0), (0, 2, 0), (0, 0, 3), (4, 4, 0)])
def test_quantize_merge_misaligned(offsets):
    # (4, 4, 0): 16-byte but not 32-byte aligned gradient and residual
    _case(70_001, 8, 2, seed=sum(offsets) + 5, offsets=offsets)


def test_quantize_merge_empty():
    q = qga()
    rec = torch.full((q.qga_2bit_words(0),), -1, dtype=torch.int32, device=DEV)
    other = _dev(_record(0, -1.0, 1.0, 3))
    e = torch.empty(0, device=DEV)
    q.qga_quantize_merge_2bit(e, torch.empty(0, device=DEV), [other, rec], 1, -0.25, 0.5, e)
    torch.cuda.synchronize()
    assert u32(rec).tolist() == list(np.array([-0.25, 0.5, 0.0], np.float32).view(np.uint32))


def test_quantize_merge_equals_two_calls_vgg16():
    """The VGG16-sized workload, 8 workers, worker 0 reducing: the fused step
    gives the same residual, record and aggregate bits as qga_quantize_2bit
    followed by qga_dequant_accumulate_2bit, and sampled whole words match
    the oracle run on the same sampled inputs (the operation is elementwise
    per word, so a record of the sampled words is what the oracle needs)."""
    q = qga()
    w = workloads.WORKLOADS["vgg16-8w"]
    n, W = w.n, w.workers
    rng = np.random.default_rng(8)
    nwords = (n + 15) // 16
    pick = np.unique(np.concatenate([np.arange(4), nwords - 1 - np.arange(4),
                                     rng.integers(0, nwords, 400)]))
    elems = (pick[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    keep = elems < n
    idx = torch.from_numpy(np.minimum(elems, n - 1)).to(DEV)
    samples = []                       # (g, r) of every worker at the sampled elements

    def sample(g, r):
        gs, rs = f32(g.index_select(0, idx)).copy(), f32(r.index_select(0, idx)).copy()
        gs[~keep] = 0.0                # elements past n: no input (their codes are 00)
        rs[~keep] = 0.0
        samples.append((gs, rs))

    others = []
    for k in range(1, W):
        g = workloads.gradient(w, k, 0, device=DEV)
        r = workloads.random_residual(n, w.pos_thr, 300 + k, device=DEV)
        sample(g, r)
        c = torch.empty(q.qga_2bit_words(n), dtype=torch.int32, device=DEV)
        q.qga_quantize_2bit(g, r, c, w.neg_thr, w.pos_thr)
        others.append(c)
        del g, r
    g0 = workloads.gradient(w, 0, 0, device=DEV)
    r_fused = workloads.random_residual(n, w.pos_thr, 300, device=DEV)
    sample(g0, r_fused)
    samples = [samples[-1]] + samples[:-1]     # worker order 0..7
    r_two = r_fused.clone()
    c_fused = torch.empty(q.qga_2bit_words(n), dtype=torch.int32, device=DEV)
    c_two = torch.empty_like(c_fused)
    out_fused = torch.empty(n, device=DEV)
    out_two = torch.empty(n, device=DEV)
    q.qga_quantize_2bit(g0, r_two, c_two, w.neg_thr, w.pos_thr)
    q.qga_dequant_accumulate_2bit([c_two] + others, out_two)
    q.qga_quantize_merge_2bit(g0, r_fused, [c_fused] + others, 0, w.neg_thr, w.pos_thr, out_fused)
    torch.cuda.synchronize()
    assert torch.equal(c_fused, c_two)
    assert torch.equal(r_fused.view(torch.int32), r_two.view(torch.int32))
    assert torch.equal(out_fused.view(torch.int32), out_two.view(torch.int32))

    m = elems.size
    mini = [oracle.quantize_2bit(gs, rs, w.neg_thr, w.pos_thr) for gs, rs in samples]
    got_words = u32(c_fused.index_select(0, torch.from_numpy(pick + 3).to(DEV)))
    last_ok = keep.reshape(-1, 16).all(axis=1)     # the ragged last word is checked by value below
    assert np.array_equal(got_words[last_ok], mini[0][0][3:][last_ok])
    assert same_bits_f32(f32(r_fused.index_select(0, idx))[keep], mini[0][1][keep])
    want = oracle.dequant_accumulate_2bit([c for c, _ in mini], m)
    assert same_bits_f32(f32(out_fused.index_select(0, idx))[keep], want[keep])
