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
