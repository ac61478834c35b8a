"""Concurrent callers: the entry points keep no device state between calls,
so calls from several host threads, each on its own stream, must give the
same bits as the oracle.  Each thread repeats its merges many times on its
own records and output (including the first calls of the merges that set a
kernel attribute on first use, W > 8), and every result is checked."""
import threading

import numpy as np
import pytest
import torch

import oracle
from gpu_util import DEV, f32, qga, same_bits_f32

pytestmark = pytest.mark.gpu


def _records_2bit(n, W, seed):
    q = qga()
    rng = np.random.default_rng(seed)
    recs = []
    for w in range(W):
        words = rng.integers(0, 1 << 32, q.qga_2bit_words(n), dtype=np.uint64).astype(np.uint32)
        words[:3] = np.array([-0.25 - 0.01 * w, 0.5 + 0.01 * w, n], np.float32).view(np.uint32)
        recs.append(words)
    return recs


def _records_qsgd(n, W, b, seed):
    q = qga()
    rng = np.random.default_rng(seed)
    recs = []
    for _ in range(W):
        words = rng.integers(0, 1 << 32, q.qga_qsgd_words(n, b), dtype=np.uint64).astype(np.uint32)
        words[:3] = np.array([1.5, b, n], np.float32).view(np.uint32)
        recs.append(words)
    return recs


def _dev(words):
    return torch.from_numpy(words.view(np.int32).copy()).to(DEV)


@pytest.mark.parametrize("threads", [2, 4])
def test_merges_from_concurrent_threads_and_streams(threads):
    q = qga()
    n, reps = 200_003, 12
    jobs = []
    for t in range(threads):
        W = (8, 9, 13, 3)[t % 4]
        r2 = _records_2bit(n, W, 10 + t)
        b = (2, 4, 8)[t % 3]
        rq = _records_qsgd(n, 8, b, 20 + t)
        jobs.append({
            "W": W, "b": b,
            "r2": [_dev(r) for r in r2], "rq": [_dev(r) for r in rq],
            "want2": oracle.dequant_accumulate_2bit(r2, n),
            "wantq": oracle.qsgd_mn_dequant_accumulate(rq, n, b),
            "out2": torch.empty(n, device=DEV), "outq": torch.empty(n, device=DEV),
            "stream": torch.cuda.Stream(device=DEV), "bad": [],
        })
    torch.cuda.synchronize()
    start = threading.Barrier(threads)

    def work(job):
        start.wait()
        with torch.cuda.stream(job["stream"]):
            for i in range(reps):
                job["out2"].fill_(float("nan"))
                job["outq"].fill_(float("nan"))
                q.qga_dequant_accumulate_2bit(job["r2"], job["out2"])
                q.qga_qsgd_mn_dequant_accumulate(job["rq"], job["outq"], job["b"])
                job["stream"].synchronize()
                if not same_bits_f32(f32(job["out2"]), job["want2"]):
                    job["bad"].append(("2bit", i))
                if not same_bits_f32(f32(job["outq"]), job["wantq"]):
                    job["bad"].append(("qsgd", i))

    pool = [threading.Thread(target=work, args=(job,)) for job in jobs]
    for th in pool:
        th.start()
    for th in pool:
        th.join(timeout=300)
        assert not th.is_alive()
    for job in jobs:
        assert not job["bad"], (job["W"], job["b"], job["bad"][:3])
