"""The benchmark's multi-rank host logic on CPU: two gloo ranks.

With N GPUs the benchmark runs one replica of the step per rank (every
worker and element is independent, so there is no collective on the data
path); the only cross-rank step is the max of the timings, taken as the
job's time.  These tests run that logic with world size 2 on the gloo
backend, and check that the reference arm does its work on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(body, world=2, timeout=120):
    port = _free_port()
    script = textwrap.dedent(f"""
        import os, sys, json, datetime
        sys.path.insert(0, {ROOT!r})
        import torch.distributed as dist
        rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        try:
    """) + textwrap.indent(textwrap.dedent(body), "    ") + textwrap.dedent("""
        finally:
            dist.destroy_process_group()
    """)
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            p.kill()
            o, e = p.communicate()
        assert p.returncode == 0, e
        outs.append(o)
    return outs


def test_max_over_ranks_takes_the_slowest_rank():
    outs = _run_ranks("""
        import bench
        mine = [10.0 + rank, 5.0 - rank, 7.0 * (rank + 1)]
        print(json.dumps(bench.max_over_ranks(mine, world)))
    """)
    for o in outs:
        assert json.loads(o.strip().splitlines()[-1]) == [11.0, 5.0, 14.0]


def test_job_throughput_counts_every_rank():
    import bench
    # 2 ranks x 8 workers x 1000 elements x 10 steps in 2 ms
    assert bench.job_gelem_per_s(2, 8, 1000, 10, 2.0) == pytest.approx(2 * 8 * 1000 * 10 / 2e-3 / 1e9)
    outs = _run_ranks("""
        import bench
        ms = bench.max_over_ranks([1.0 + rank], world)[0]
        print(json.dumps(bench.job_gelem_per_s(world, 8, 1000, 10, ms)))
    """)
    vals = [json.loads(o.strip().splitlines()[-1]) for o in outs]
    assert vals[0] == vals[1] == pytest.approx(2 * 8 * 1000 * 10 / 2e-3 / 1e9)


def test_reference_arm_runs_on_rank_zero_only():
    outs = _run_ranks("""
        import bench, argparse
        args = argparse.Namespace(gpus=world, steps=1, warmup=0)
        bench.run_reference(args, rank, world)
    """, timeout=300)
    line = json.loads(outs[0].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert outs[1].strip() == ""


def test_record_gather_layout_on_two_and_three_ranks():
    """The exchange's gather step: every rank ends up with the same buffer,
    rank r's record in row r (the merge then adds the rows in rank order).
    The records here are synthetic words, so no GPU is needed."""
    for world in (2, 3):
        outs = _run_ranks("""
            import torch, hashlib
            from quantized_gradient_aggregation_b200.exchange import gather_records
            words = 37
            local = torch.arange(words, dtype=torch.int32) * 1000 + rank
            gathered = torch.empty(world * words, dtype=torch.int32)
            rows = gather_records(local, gathered)
            assert len(rows) == world
            for r, row in enumerate(rows):
                assert row.tolist() == [w * 1000 + r for w in range(words)], r
            print(hashlib.sha256(gathered.numpy().tobytes()).hexdigest())
        """, world=world)
        digests = {o.strip().splitlines()[-1] for o in outs}
        assert len(digests) == 1


# The exchange steps end to end on gloo ranks: every rank quantizes its OWN
# seeded gradient, the records cross the process group, and every rank must
# hold the merge of all ranks' records in rank order, with its residual
# carried over three steps.  The arithmetic is the oracle's (injected through
# the classes' ``ops``, on host tensors); what is under test is the classes'
# ordering: quantize, gather, merge rows in rank order, buffers reused.
_EXCHANGE_PRELUDE = """
    import numpy as np, torch, oracle
    from quantized_gradient_aggregation_b200.exchange import (
        BucketedCompressedAllGather, CompressedAllGather)

    def as_u32(t):
        return t.numpy().view(np.uint32)

    def q2(grad, residual, compr, neg, pos):
        c, r = oracle.quantize_2bit(grad.numpy(), residual.numpy(), neg, pos)
        compr.copy_(torch.from_numpy(c.view(np.int32)))
        residual.copy_(torch.from_numpy(r))

    def m2(records, out):
        out.copy_(torch.from_numpy(oracle.dequant_accumulate_2bit(
            [as_u32(r) for r in records], out.numel())))

    def qt(grad, residual, compr, neg, pos):
        c, r = oracle.quantize_ternary(grad.numpy(), residual.numpy(), neg, pos)
        compr.copy_(torch.from_numpy(c.view(np.int32)))
        residual.copy_(torch.from_numpy(r))

    def mt(records, out):
        out.copy_(torch.from_numpy(oracle.dequant_accumulate_ternary(
            [as_u32(r) for r in records], out.numel())))

    def grad_of(rank_, step, n):
        g = np.random.default_rng(1000 * rank_ + step).standard_normal(n) * 0.4
        return g.astype(np.float32)
"""


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("fmt", ["2bit", "ternary"])
def test_exchange_step_distinct_ranks(world, fmt):
    outs = _run_ranks(_EXCHANGE_PRELUDE + f"""
    fmt = {fmt!r}
    n, neg, pos = 10_007, -0.25, 0.25
    ops = (oracle.words_2bit, q2, m2) if fmt == "2bit" else (oracle.words_ternary, qt, mt)
    quant = oracle.quantize_2bit if fmt == "2bit" else oracle.quantize_ternary
    merge = oracle.dequant_accumulate_2bit if fmt == "2bit" else oracle.dequant_accumulate_ternary
    ex = CompressedAllGather(n, neg, pos, fmt=fmt, device="cpu", ops=ops)
    r = torch.zeros(n)
    out = torch.empty(n)
    res_all = [np.zeros(n, np.float32) for _ in range(world)]
    for step in range(3):
        ex.step(torch.from_numpy(grad_of(rank, step, n)), r, out)
        recs = []
        for k in range(world):  # every rank's record, recomputed from its seed
            c, res_all[k] = quant(grad_of(k, step, n), res_all[k], neg, pos)
            recs.append(c)
        rows = as_u32(ex.gathered).reshape(world, -1)
        for k in range(world):
            assert np.array_equal(rows[k], recs[k]), (step, k)
        assert np.array_equal(r.numpy().view(np.uint32), res_all[rank].view(np.uint32)), step
        want = merge(recs, n)
        assert np.array_equal(out.numpy().view(np.uint32), want.view(np.uint32)), step
    assert len({{bytes(as_u32(ex.gathered))}}) == 1
    print("ok", float(out.abs().sum()))
    """, world=world)
    sums = {o.strip().splitlines()[-1] for o in outs}
    assert len(sums) == 1 and next(iter(sums)).startswith("ok")


@pytest.mark.parametrize("world", [2, 3])
def test_bucketed_exchange_distinct_ranks(world):
    outs = _run_ranks(_EXCHANGE_PRELUDE + """
    buckets = [[768, 3072, 4099, 17], [3000, 5, 768 * 4]]
    neg = [[-2e-3] * len(b) for b in buckets]
    pos = [[2e-3 + 1e-4 * i for i in range(len(b))] for b in buckets]

    def qb(grads, residuals, neg_, pos_, compr, table=None):
        assert table == ("table", len(grads))
        c, rs = oracle.quantize_2bit_bucket([g.numpy() for g in grads],
                                            [r.numpy() for r in residuals], neg_, pos_)
        compr.copy_(torch.from_numpy(c.view(np.int32)))
        for r, new in zip(residuals, rs):
            r.copy_(torch.from_numpy(new))

    def mb(records, sizes, out):
        out.copy_(torch.from_numpy(oracle.dequant_accumulate_2bit_bucket(
            [as_u32(r) for r in records], sizes)))

    ops = (oracle.bucket_words_2bit, lambda g, r, a, b: ("table", len(g)), qb, mb)
    ex = BucketedCompressedAllGather(buckets, neg, pos, device="cpu", ops=ops)

    def bucket_grads(rank_, step):
        return [[torch.from_numpy(grad_of(100 * rank_ + 10 * b + t, step, s) * 1e-2)
                 for t, s in enumerate(sizes)] for b, sizes in enumerate(buckets)]

    res = [[torch.zeros(s) for s in b] for b in buckets]
    outs_ = [torch.empty(sum(b)) for b in buckets]
    res_all = [[[np.zeros(s, np.float32) for s in b] for b in buckets] for _ in range(world)]
    for step in range(3):
        ex.step(bucket_grads(rank, step), res, outs_)
        for b, sizes in enumerate(buckets):
            recs = []
            for k in range(world):
                g_k = [x.numpy() for x in bucket_grads(k, step)[b]]
                c, res_all[k][b] = oracle.quantize_2bit_bucket(g_k, res_all[k][b], neg[b], pos[b])
                recs.append(c)
            rows = as_u32(ex.gathered[b]).reshape(world, -1)
            for k in range(world):
                assert np.array_equal(rows[k], recs[k]), (step, b, k)
            want = oracle.dequant_accumulate_2bit_bucket(recs, sizes)
            assert np.array_equal(outs_[b].numpy().view(np.uint32), want.view(np.uint32)), (step, b)
            for t in range(len(sizes)):
                assert np.array_equal(res[b][t].numpy(), res_all[rank][b][t]), (step, b, t)
    print("ok", sum(float(o.abs().sum()) for o in outs_))
    """, world=world)
    sums = {o.strip().splitlines()[-1] for o in outs}
    assert len(sums) == 1 and next(iter(sums)).startswith("ok")


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("b", [2, 8])
def test_qsgd_exchange_distinct_ranks(world, b):
    """QSGD-MaxNorm across gloo ranks: every rank's local max, the all-reduce
    MAX, each rank's own seed, the gather in rank order and the merge, with
    the oracle's arithmetic injected (host tensors)."""
    outs = _run_ranks(_EXCHANGE_PRELUDE + f"""
    from quantized_gradient_aggregation_b200.exchange import QsgdAllGather
    b, n, seed_base = {b}, 10_007, 1234

    def local_max(g, m):
        m.fill_(float(oracle.qsgd_mn_max([g.numpy()])))

    def quantize(g, compr, bits, seed, m):
        c = oracle.qsgd_mn_quantize(g.numpy(), bits, seed, np.float32(m.item()))
        compr.copy_(torch.from_numpy(c.view(np.int32)))

    def merge(records, out, bits):
        out.copy_(torch.from_numpy(oracle.qsgd_mn_dequant_accumulate([as_u32(r) for r in records],
                                                                   out.numel(), bits)))

    ex = QsgdAllGather(n, b, seed_base, device="cpu", ops=(oracle.qsgd_words, local_max, quantize, merge))
    out = torch.empty(n)
    for step in range(2):
        ex.step(torch.from_numpy(grad_of(rank, step, n)), out)
        M = oracle.qsgd_mn_max([grad_of(k, step, n) for k in range(world)])
        assert float(ex.m.item()) == float(M), step
        recs = [oracle.qsgd_mn_quantize(grad_of(k, step, n), b, seed_base + k, M) for k in range(world)]
        rows = as_u32(ex.gathered).reshape(world, -1)
        for k in range(world):
            assert np.array_equal(rows[k], recs[k]), (step, k)
        want = oracle.qsgd_mn_dequant_accumulate(recs, n, b)
        assert np.array_equal(out.numpy().view(np.uint32), want.view(np.uint32)), step
    print("ok", float(out.abs().sum()))
    """, world=world)
    sums = {o.strip().splitlines()[-1] for o in outs}
    assert len(sums) == 1 and next(iter(sums)).startswith("ok")
