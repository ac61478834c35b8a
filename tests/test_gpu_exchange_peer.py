"""The exchange whose merge reads every rank's record in place (CUDA IPC
mappings of the peers' record buffers): W processes, each quantizing its
OWN seeded gradient with the library's kernels, a gloo group for the host
barriers.  Rank r runs on GPU r mod (GPUs present), so on a one-GPU machine
all ranks share one device (the mappings are then same-device IPC; no kernel
waits on another process, only the host barrier orders the steps), and on a
machine with enough GPUs the merges read their peers' GPUs over NVLink.
Every rank must hold the merge of all ranks' records in rank order and its
own carried residual, bit for bit against the oracle, over four steps (both
record sets of the double buffer, twice).
"""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(body, world, timeout=300):
    port = _free_port()
    script = textwrap.dedent(f"""
        import os, sys, datetime
        sys.path.insert(0, {ROOT!r})
        sys.path.insert(0, {TESTS!r})
        import numpy as np
        import torch
        import torch.distributed as dist
        import oracle
        from quantized_gradient_aggregation_b200.exchange import PeerMergeExchange
        rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
        dev = torch.device("cuda", rank % torch.cuda.device_count())
        torch.cuda.set_device(dev)
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
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
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


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("fmt", ["2bit", "ternary"])
def test_peer_merge_exchange(world, fmt):
    outs = _run(f"""
    fmt = {fmt!r}
    n, neg, pos = 1_000_003, -0.25, 0.25
    quant = oracle.quantize_2bit if fmt == "2bit" else oracle.quantize_ternary
    merge = oracle.dequant_accumulate_2bit if fmt == "2bit" else oracle.dequant_accumulate_ternary

    def grad_of(seed, step):
        return (np.random.default_rng(1000 * seed + step).standard_normal(n) * 0.4).astype(np.float32)

    ex = PeerMergeExchange(n, neg, pos, fmt=fmt)
    r = torch.zeros(n, device=dev)
    out = torch.empty(n, device=dev)
    res_all = [np.zeros(n, np.float32) for _ in range(world)]
    for step in range(4):
        ex.step(torch.from_numpy(grad_of(rank, step)).to(dev), r, out)
        torch.cuda.synchronize()
        recs = []
        for k in range(world):
            c, res_all[k] = quant(grad_of(k, step), res_all[k], neg, pos)
            recs.append(c)
        assert np.array_equal(r.cpu().numpy().view(np.uint32), res_all[rank].view(np.uint32)), step
        want = merge(recs, n)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32)), step
    ex.close()
    print("ok", float(out.abs().sum()))
    """, world)
    sums = {o.strip().splitlines()[-1] for o in outs}
    assert len(sums) == 1 and next(iter(sums)).startswith("ok")
