"""Data-parallel exchange of compressed gradients across ranks.

The receiver-side merge of MXNet pull request #8342 "[WIP] 2bit gradient
compression" ("Local kvstore": every device quantizes its gradient, the
compressed arrays travel to the device that reduces, which dequantizes and
sums them), made symmetric for one process per GPU: every rank quantizes
its own gradient with error feedback, the W records are all-gathered into
one contiguous buffer (NCCL over NVLink / NVSwitch; a record is 1/16 of the
fp32 gradient), and every rank merges the same W records in rank order, so
all ranks hold the same aggregate bit for bit without a second exchange.
The gathered buffer holds W records of ``words`` int32 each, rank r's record
in row r.

Every arithmetic step runs in the library's CUDA kernels; this module only
orders them around one collective on the current stream.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (qga_2bit_words, qga_dequant_accumulate_2bit, qga_dequant_accumulate_ternary,
               qga_quantize_2bit, qga_quantize_ternary, qga_ternary_words)

_FORMATS = {
    "2bit": (qga_2bit_words, qga_quantize_2bit, qga_dequant_accumulate_2bit),
    "ternary": (qga_ternary_words, qga_quantize_ternary, qga_dequant_accumulate_ternary),
}


def gather_records(local: torch.Tensor, gathered: torch.Tensor, group=None):
    """All-gather one record per rank into ``gathered`` (world * words
    int32) and return its rows, row r = rank r's record."""
    world = dist.get_world_size(group)
    words = local.numel()
    if gathered.numel() != world * words:
        raise ValueError(f"gathered holds {gathered.numel()} words, need {world} x {words}")
    dist.all_gather_into_tensor(gathered, local, group=group)
    return list(gathered.view(world, words).unbind(0))


class CompressedAllGather:
    """One compressed all-gather step for an n-element gradient.

    ``step(grad, residual, out)`` quantizes ``grad`` against ``residual``
    (updated in place) with the thresholds given here, all-gathers the
    records of the ``group``'s ranks and writes their merge (worker order =
    rank order) into ``out``.  The two record buffers are allocated once,
    here, on ``device`` (default: the current CUDA device).

    ``ops`` replaces the format's three library calls by a triple
    ``(words(n), quantize(grad, residual, compr, neg, pos), merge(records,
    out))`` with the same arguments; it exists so that the step's ordering
    (quantize, gather, merge in rank order, residual carried) can be driven
    on a CPU process group with stand-in arithmetic.
    """

    def __init__(self, n: int, neg_threshold: float, pos_threshold: float, group=None,
                 fmt: str = "2bit", *, device=None, ops=None):
        if fmt not in _FORMATS:
            raise ValueError(f"format {fmt!r}: one of {sorted(_FORMATS)}")
        self.n = int(n)
        self.neg = float(neg_threshold)
        self.pos = float(pos_threshold)
        self.group = group
        self.world = dist.get_world_size(group)
        words_fn, self._quantize, self._merge = _FORMATS[fmt] if ops is None else ops
        self.words = int(words_fn(self.n))
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.local = torch.empty(self.words, dtype=torch.int32, device=device)
        self.gathered = torch.empty(self.world * self.words, dtype=torch.int32, device=device)

    def step(self, grad: torch.Tensor, residual: torch.Tensor, out: torch.Tensor) -> None:
        self._quantize(grad, residual, self.local, self.neg, self.pos)
        records = gather_records(self.local, self.gathered, self.group)
        self._merge(records, out)


class BucketedCompressedAllGather:
    """The exchange over a list of buckets (each a list of tensors quantized
    by one bucket launch), pipelined: bucket b's records are all-gathered by
    NCCL while the current stream already quantizes bucket b + 1, and each
    bucket's merge waits only for its own all-gather.

    ``buckets``: per bucket, the tensor sizes; ``neg`` / ``pos``: per bucket,
    per-tensor thresholds.  ``step(grads, residuals, outs)`` takes per bucket
    the gradient tensors (fp32 or bf16, one dtype per bucket), the fp32
    residuals (updated in place) and one flat fp32 output holding the
    bucket's merged tensors one after the other.  Record buffers live on
    ``device`` (default: the current CUDA device).

    ``ops`` replaces the four library calls by ``(words(sizes),
    make_table(grads, residuals, neg, pos), quantize(grads, residuals, neg,
    pos, compr, table=...), merge(records, sizes, out))`` with the same
    arguments, so that the pipeline's ordering can be driven on a CPU
    process group with stand-in arithmetic.
    """

    def __init__(self, buckets, neg, pos, group=None, *, device=None, ops=None):
        from . import (make_bucket_table, qga_2bit_bucket_words, qga_dequant_accumulate_2bit_bucket,
                       qga_quantize_2bit_bucket)
        if ops is None:
            ops = (qga_2bit_bucket_words, make_bucket_table, qga_quantize_2bit_bucket,
                   qga_dequant_accumulate_2bit_bucket)
        words_fn, self._make_table, self._quantize, self._merge = ops
        self.sizes = [list(map(int, b)) for b in buckets]
        self.neg = [list(map(float, x)) for x in neg]
        self.pos = [list(map(float, x)) for x in pos]
        self.group = group
        self.world = dist.get_world_size(group)
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.words = [int(words_fn(s)) for s in self.sizes]
        self.local = [torch.empty(w, dtype=torch.int32, device=device) for w in self.words]
        self.gathered = [torch.empty(self.world * w, dtype=torch.int32, device=device)
                         for w in self.words]
        self._tables = None
        self._table_key = None

    def records(self, b):
        return list(self.gathered[b].view(self.world, self.words[b]).unbind(0))

    def step(self, grads, residuals, outs) -> None:
        key = tuple((g.data_ptr(), r.data_ptr()) for bg, br in zip(grads, residuals)
                    for g, r in zip(bg, br))
        if key != self._table_key:  # descriptor tables: rebuilt only when a buffer moved
            self._tables = [self._make_table(grads[b], residuals[b], self.neg[b], self.pos[b])
                            for b in range(len(self.sizes))]
            self._table_key = key
        works = []
        for b in range(len(self.sizes)):
            self._quantize(grads[b], residuals[b], self.neg[b], self.pos[b], self.local[b],
                           table=self._tables[b])
            # NCCL orders the collective after the work already on the current
            # stream, and runs it beside the next bucket's quantize
            works.append(dist.all_gather_into_tensor(self.gathered[b], self.local[b],
                                                     group=self.group, async_op=True))
        for b, work in enumerate(works):
            work.wait()  # the current stream waits for bucket b's records only
            self._merge(self.records(b), self.sizes[b], outs[b])


class PeerMergeExchange:
    """The exchange with the merge reading every rank's record where it lies.

    Each rank quantizes into a record buffer of its own.  The buffers are
    opened in every other rank by CUDA IPC (mappings of the owners' device
    memory), so each rank's merge kernel loads all W records directly: the
    peers' words cross NVLink / NVSwitch as plain loads inside the merge,
    once, overlapped with its arithmetic and output stores, and no
    all-gathered copy is written or read back.  The kernels are the
    library's ordinary merges; a peer's buffer is just another record
    pointer (plain loads only; nothing multicast).

    Ordering across ranks is one host barrier per step: a rank synchronizes
    its stream after its quantize, then waits for the group, then merges.
    Record buffers alternate between two sets, so a rank overwrites set
    s % 2 only at step s + 2, after the barrier of step s + 1, which every
    rank reaches only after its merge of step s is complete.

    ``close()`` releases the mappings of the peers' buffers (call it on
    every rank before the group is destroyed).  Same arguments and formats
    as ``CompressedAllGather``.
    """

    def __init__(self, n: int, neg_threshold: float, pos_threshold: float, group=None,
                 fmt: str = "2bit", *, device=None):
        from torch.multiprocessing.reductions import reduce_tensor
        if fmt not in _FORMATS:
            raise ValueError(f"format {fmt!r}: one of {sorted(_FORMATS)}")
        self.n = int(n)
        self.neg = float(neg_threshold)
        self.pos = float(pos_threshold)
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        words_fn, self._quantize, self._merge = _FORMATS[fmt]
        self.words = int(words_fn(self.n))
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.local = [torch.zeros(self.words, dtype=torch.int32, device=device) for _ in range(2)]
        torch.cuda.synchronize(device)
        specs = [reduce_tensor(buf) for buf in self.local]
        everyone = [None] * self.world
        dist.all_gather_object(everyone, specs, group=self.group)
        # records[k][r]: rank r's buffer of set k (this rank's own, or a mapping of a peer's)
        self.records = [[self.local[k] if r == self.rank else everyone[r][k][0](*everyone[r][k][1])
                         for r in range(self.world)] for k in range(2)]
        self._step = 0

    def step(self, grad: torch.Tensor, residual: torch.Tensor, out: torch.Tensor) -> None:
        k = self._step & 1
        self._quantize(grad, residual, self.local[k], self.neg, self.pos)
        torch.cuda.current_stream(self.local[k].device).synchronize()
        dist.barrier(group=self.group)  # every rank's record of this step is complete
        self._merge(self.records[k], out)
        self._step += 1

    def close(self) -> None:
        torch.cuda.current_stream(self.local[0].device).synchronize()
        dist.barrier(group=self.group)  # no rank still reads a peer's buffer
        self.records = None
        torch.cuda.synchronize(self.local[0].device)
        dist.barrier(group=self.group)


class QsgdAllGather:
    """One QSGD-MaxNorm exchange step across ranks, b bits per element.

    ``step(grad, out)``: the local max |g| (``qga_qsgd_mn_max`` on this
    rank's gradient), an all-reduce MAX of that one float, so that every rank
    quantizes on the same global M; the quantize of this rank's gradient
    with the seed ``seed_base + rank``; an all-gather of the W records; and
    the integer-sum merge of the records in rank order into ``out``.  Every
    rank ends with the same aggregate bit for bit.  QSGD-MaxNorm keeps no
    residual.

    ``ops`` replaces the library calls by ``(words(n, b), local_max(grad,
    m_out), quantize(grad, compr, b, seed, m), merge(records, out, b))`` with
    the same arguments, so that the step's ordering can be driven on a CPU
    process group with stand-in arithmetic.
    """

    def __init__(self, n: int, bits: int, seed_base: int, group=None, *, device=None, ops=None):
        from . import qga_qsgd_mn_dequant_accumulate, qga_qsgd_mn_max, qga_qsgd_mn_quantize, qga_qsgd_words
        if ops is None:
            ops = (qga_qsgd_words, lambda g, m: qga_qsgd_mn_max([g], m), qga_qsgd_mn_quantize,
                   qga_qsgd_mn_dequant_accumulate)
        words_fn, self._max, self._quantize, self._merge = ops
        self.n = int(n)
        self.bits = int(bits)
        self.group = group
        self.world = dist.get_world_size(group)
        self.seed = int(seed_base) + dist.get_rank(group)
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.words = int(words_fn(self.n, self.bits))
        self.m = torch.zeros(1, dtype=torch.float32, device=device)
        self.local = torch.empty(self.words, dtype=torch.int32, device=device)
        self.gathered = torch.empty(self.world * self.words, dtype=torch.int32, device=device)

    def step(self, grad: torch.Tensor, out: torch.Tensor) -> None:
        self._max(grad, self.m)
        dist.all_reduce(self.m, op=dist.ReduceOp.MAX, group=self.group)
        self._quantize(grad, self.local, self.bits, self.seed, self.m)
        records = gather_records(self.local, self.gathered, self.group)
        self._merge(records, out, self.bits)
