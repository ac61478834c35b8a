"""GPU parity of GRandK-MaxNorm (QSGD-MaxNorm of K shared coordinates)
through the C ABI against the CPU oracle: M, every record word and every
merged element bit for bit, on ragged sizes, out-of-range coordinates,
K = 0 and the full 2^27-element, 8-worker workload with K = 10000."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import DEV, f32, first_diff, qga, same_bits_f32, u32

pytestmark = pytest.mark.gpu


def _grads(n, W, seed, outliers=True):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    gs = [torch.randn(n, device=DEV, generator=gen) * 2 for _ in range(W)]
    if outliers and n > 10:
        gs[W - 1][n // 3] = -40.0
    return gs


def _run(gs, index, b, seed_base=1234):
    q = qga()
    n, K = gs[0].numel(), index.size
    idx = torch.from_numpy(index).to(DEV)
    M = torch.full((1,), float("nan"), device=DEV)
    q.qga_grandk_mn_max(gs, idx, M)
    comprs = []
    for w, g in enumerate(gs):
        c = torch.full((q.qga_qsgd_words(K, b) + 2,), -1, dtype=torch.int32, device=DEV)
        q.qga_grandk_mn_quantize(g, idx, c, b, seed_base + w, M)
        assert (u32(c[-2:]) == 0xFFFFFFFF).all()          # nothing past the record
        comprs.append(c[:-2])
    out = torch.full((n + 1,), float("nan"), device=DEV)
    q.qga_grandk_mn_dequant_accumulate(comprs, idx, out[:n], b)
    torch.cuda.synchronize()
    assert np.isnan(f32(out[n:])).all()                     # nothing past out
    return M, comprs, out[:n]


def _check(gs, index, b, seed_base=1234):
    M, comprs, out = _run(gs, index, b, seed_base)
    hosts = [f32(g) for g in gs]
    want_M = oracle.grandk_mn_max(hosts, index)
    assert M.item() == want_M
    want_recs = []
    for w, h in enumerate(hosts):
        want = oracle.grandk_mn_quantize(h, index, b, seed_base + w, want_M)
        got = u32(comprs[w])
        assert np.array_equal(got, want), (b, w, first_diff(got, want))
        want_recs.append(want)
    want_out = oracle.grandk_mn_dequant_accumulate(want_recs, index, hosts[0].size, b)
    assert same_bits_f32(f32(out), want_out), first_diff(f32(out), want_out)


@pytest.mark.parametrize("b", [2, 4, 8])
@pytest.mark.parametrize("n,K,W", [(5003, 777, 3), (100, 100, 2), (1 << 20, 10_000, 8),
                                   (4099, 1, 1), (70_001, 33, 5), (1000, 31, 17)])
def test_grandk_matches_oracle(b, n, K, W):
    gs = _grads(n, W, 11 * n + K + b)
    index = np.random.default_rng(n + K).choice(n, size=K, replace=False).astype(np.int64)
    _check(gs, index, b)


@pytest.mark.parametrize("b", [2, 8])
def test_grandk_sorted_and_identity_index(b):
    n = 20_000
    gs = _grads(n, 4, 3)
    index = np.sort(np.random.default_rng(1).choice(n, size=4_321, replace=False)).astype(np.int64)
    _check(gs, index, b)
    _check(gs, np.arange(n, dtype=np.int64), b)


def test_grandk_identity_equals_dense_qsgd():
    """Keeping every coordinate in order gives the dense QSGD-MaxNorm
    results of the same library, bit for bit."""
    q = qga()
    n, b = 33_333, 4
    gs = _grads(n, 3, 8)
    M, comprs, out = _run(gs, np.arange(n, dtype=np.int64), b)
    Md = torch.empty(1, device=DEV)
    q.qga_qsgd_mn_max(gs, Md)
    dense = []
    for w, g in enumerate(gs):
        c = torch.empty(q.qga_qsgd_words(n, b), dtype=torch.int32, device=DEV)
        q.qga_qsgd_mn_quantize(g, c, b, 1234 + w, Md)
        dense.append(c)
    outd = torch.empty(n, device=DEV)
    q.qga_qsgd_mn_dequant_accumulate(dense, outd, b)
    assert M.item() == Md.item()
    assert all(np.array_equal(u32(a), u32(d)) for a, d in zip(comprs, dense))
    assert same_bits_f32(f32(out), f32(outd))


@pytest.mark.parametrize("b", [2, 4, 8])
def test_grandk_out_of_range_coordinates_are_skipped(b):
    n = 3001
    gs = _grads(n, 3, 21)
    index = np.random.default_rng(2).choice(n, size=64, replace=False).astype(np.int64)
    index[[0, 7, 31, 63]] = [-1, n, 1 << 40, -(1 << 62)]
    _check(gs, index, b)


@pytest.mark.parametrize("b", [2, 8])
def test_grandk_empty_index(b):
    q = qga()
    n = 1000
    gs = _grads(n, 2, 4)
    M, comprs, out = _run(gs, np.zeros(0, np.int64), b)
    assert M.item() == 0.0
    assert u32(comprs[0]).tolist() == [0, np.float32(b).view(np.uint32), 0]
    assert not u32(out).any()                                # all +0
    assert q.qga_qsgd_words(0, b) == 3


def test_grandk_full_size_eight_workers():
    """The QSGD workload's 2^27-element gradients of 8 workers, K = 10000
    shared coordinates: M, all 8 records and all 2^27 merged elements per b
    against the oracle."""
    w = workloads.WORKLOADS["qsgd-128M-8w"]
    n, W = w.n, w.workers
    index = workloads.grandk_index(n)
    q = qga()
    idx = torch.from_numpy(index).to(DEV)
    grads = [workloads.gradient(w, k, 0, device=DEV) for k in range(W)]
    M = torch.empty(1, device=DEV)
    q.qga_grandk_mn_max(grads, idx, M)
    # the oracle reads the kept values only: gather them (torch indexing),
    # then the oracle's identity selection is the same computation (pinned)
    kept = [f32(g.index_select(0, idx)) for g in grads]
    ident = np.arange(index.size, dtype=np.int64)
    want_M = oracle.grandk_mn_max(kept, ident)
    assert M.item() == want_M
    for b in w.bits:
        comprs, want_recs = [], []
        for k, g in enumerate(grads):
            c = torch.empty(q.qga_qsgd_words(index.size, b), dtype=torch.int32, device=DEV)
            q.qga_grandk_mn_quantize(g, idx, c, b, workloads.QSGD_SEED_BASE + k, M)
            want = oracle.grandk_mn_quantize(kept[k], ident, b, workloads.QSGD_SEED_BASE + k, want_M)
            assert np.array_equal(u32(c), want), (b, k)
            comprs.append(c)
            want_recs.append(want)
        out = torch.full((n,), float("nan"), device=DEV)
        q.qga_grandk_mn_dequant_accumulate(comprs, idx, out, b)
        vals = oracle.grandk_mn_dequant_accumulate(want_recs, ident, index.size, b)
        got = f32(out)
        assert same_bits_f32(got[index], vals)
        rest = np.ones(n, bool)
        rest[index] = False
        assert not got[rest].view(np.uint32).any()           # +0 everywhere else
        del out, got, rest
