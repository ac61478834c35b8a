"""The compressed all-gather exchange across real ranks: one process per GPU,
an NCCL group, every rank quantizing its OWN seeded gradient with the
library's kernels.  Every rank must hold each rank's record in its row of
the gathered buffer, the merge of all records in rank order, and its own
carried residual, all bit for bit against the oracle, over three steps.

It needs at least two GPUs and is skipped otherwise.  NCCL's NVLink
SHARP path is switched off (plain all-gather over peer links), and the
group's timeout is short, so that a rank that fails ends the others'
collective with an error instead of a wait.
"""
import os
import socket
import subprocess
import sys
import textwrap

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_gpu_ranks(body, world, timeout=300):
    port = _free_port()
    script = textwrap.dedent(f"""
        import os, sys, datetime
        sys.path.insert(0, {ROOT!r})
        sys.path.insert(0, {TESTS!r})
        import torch
        import torch.distributed as dist
        rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
        dev = torch.device("cuda", rank)
        torch.cuda.set_device(dev)
        dist.init_process_group("nccl", rank=rank, world_size=world, device_id=dev,
                                timeout=datetime.timedelta(seconds=60))
        try:
    """) + textwrap.indent(textwrap.dedent(body), "    ") + textwrap.dedent("""
            torch.cuda.synchronize()
        finally:
            dist.destroy_process_group()
    """)
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            p.kill()
            o, e = p.communicate()
        assert p.returncode == 0, e[-4000:]
        outs.append(o)
    return outs


def _worlds():
    n = torch.cuda.device_count() if torch.cuda.is_available() else 0
    return [w for w in (2, 4) if w <= n] or [2]


_PRELUDE = """
    import numpy as np
    import oracle
    from quantized_gradient_aggregation_b200.exchange import (
        BucketedCompressedAllGather, CompressedAllGather)

    def u32(t):
        return t.cpu().numpy().view(np.uint32)

    def grad_of(seed, step, n, scale=0.4):
        g = np.random.default_rng(1000 * seed + step).standard_normal(n) * scale
        return g.astype(np.float32)
"""


@pytest.mark.parametrize("world", _worlds())
@pytest.mark.parametrize("fmt", ["2bit", "ternary"])
def test_exchange_step_across_gpus(world, fmt):
    if torch.cuda.device_count() < world:
        pytest.skip(f"needs {world} GPUs")
    outs = _run_gpu_ranks(_PRELUDE + f"""
    fmt = {fmt!r}
    n, neg, pos = 1_000_003, -0.25, 0.25
    quant = oracle.quantize_2bit if fmt == "2bit" else oracle.quantize_ternary
    merge = oracle.dequant_accumulate_2bit if fmt == "2bit" else oracle.dequant_accumulate_ternary
    ex = CompressedAllGather(n, neg, pos, fmt=fmt)
    r = torch.zeros(n, device=dev)
    out = torch.empty(n, device=dev)
    res_all = [np.zeros(n, np.float32) for _ in range(world)]
    for step in range(3):
        ex.step(torch.from_numpy(grad_of(rank, step, n)).to(dev), r, out)
        torch.cuda.synchronize()
        recs = []
        for k in range(world):
            c, res_all[k] = quant(grad_of(k, step, n), res_all[k], neg, pos)
            recs.append(c)
        rows = u32(ex.gathered).reshape(world, -1)
        for k in range(world):
            assert np.array_equal(rows[k], recs[k]), (step, k)
        assert np.array_equal(u32(r), res_all[rank].view(np.uint32)), step
        assert np.array_equal(u32(out), merge(recs, n).view(np.uint32)), step
    print("ok", float(out.abs().sum()))
    """, world)
    sums = {o.strip().splitlines()[-1] for o in outs}
    assert len(sums) == 1 and next(iter(sums)).startswith("ok")


@pytest.mark.parametrize("world", _worlds())
def test_bucketed_exchange_across_gpus(world):
    if torch.cuda.device_count() < world:
        pytest.skip(f"needs {world} GPUs")
    outs = _run_gpu_ranks(_PRELUDE + """
    buckets = [[768, 3072, 589_824, 17], [30_000, 5, 768 * 16]]
    neg = [[-2e-3] * len(b) for b in buckets]
    pos = [[2e-3 + 1e-4 * i for i in range(len(b))] for b in buckets]

    def bucket_grads(seed, step):
        return [[grad_of(100 * seed + 10 * b + t, step, s, 1e-3) for t, s in enumerate(sizes)]
                for b, sizes in enumerate(buckets)]

    ex = BucketedCompressedAllGather(buckets, neg, pos)
    res = [[torch.zeros(s, device=dev) for s in b] for b in buckets]
    outs_ = [torch.empty(sum(b), device=dev) for b in buckets]
    res_all = [[[np.zeros(s, np.float32) for s in b] for b in buckets] for _ in range(world)]
    for step in range(3):
        mine = [[torch.from_numpy(g).to(dev) for g in b] for b in bucket_grads(rank, step)]
        ex.step(mine, res, outs_)
        torch.cuda.synchronize()
        for b, sizes in enumerate(buckets):
            recs = []
            for k in range(world):
                c, res_all[k][b] = oracle.quantize_2bit_bucket(bucket_grads(k, step)[b], res_all[k][b],
                                                               neg[b], pos[b])
                recs.append(c)
            rows = u32(ex.gathered[b]).reshape(world, -1)
            for k in range(world):
                assert np.array_equal(rows[k], recs[k]), (step, b, k)
            want = oracle.dequant_accumulate_2bit_bucket(recs, sizes)
            assert np.array_equal(u32(outs_[b]), want.view(np.uint32)), (step, b)
            for t in range(len(sizes)):
                assert np.array_equal(u32(res[b][t]), res_all[rank][b][t].view(np.uint32)), (step, b, t)
    print("ok", sum(float(o.abs().sum()) for o in outs_))
    """, world)
    sums = {o.strip().splitlines()[-1] for o in outs}
    assert len(sums) == 1 and next(iter(sums)).startswith("ok")


@pytest.mark.parametrize("world", _worlds())
@pytest.mark.parametrize("b", [2, 8])
def test_qsgd_exchange_across_gpus(world, b):
    if torch.cuda.device_count() < world:
        pytest.skip(f"needs {world} GPUs")
    outs = _run_gpu_ranks(_PRELUDE + f"""
    from quantized_gradient_aggregation_b200.exchange import QsgdAllGather
    b, n, seed_base = {b}, 1_000_003, 1234
    ex = QsgdAllGather(n, b, seed_base)
    out = torch.empty(n, device=dev)
    for step in range(2):
        ex.step(torch.from_numpy(grad_of(rank, step, n)).to(dev), out)
        torch.cuda.synchronize()
        M = oracle.qsgd_mn_max([grad_of(k, step, n) for k in range(world)])
        assert float(ex.m.item()) == float(M), step
        recs = [oracle.qsgd_mn_quantize(grad_of(k, step, n), b, seed_base + k, M) for k in range(world)]
        rows = u32(ex.gathered).reshape(world, -1)
        for k in range(world):
            assert np.array_equal(rows[k], recs[k]), (step, k)
        want = oracle.qsgd_mn_dequant_accumulate(recs, n, b)
        assert np.array_equal(u32(out), want.view(np.uint32)), step
    print("ok", float(out.abs().sum()))
    """, world)
    sums = {o.strip().splitlines()[-1] for o in outs}
    assert len(sums) == 1 and next(iter(sums)).startswith("ok")
