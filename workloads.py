"""Seeded synthetic inputs for the tests and the benchmark.

This module only draws numbers: gradients of the shapes and distributions of
the five workloads below, residual initial values, outlier placement, the
kept coordinates of the sparsified (GRandK) variant and the
per-tensor thresholds of the bucket workload (a statistic of the drawn input,
fixed before any quantization runs).  It holds none of the quantization
arithmetic and imports neither the oracle nor the GPU library, so both sides
can be fed from it.

The workloads stand in for the gradients of the models the source pages train
(ResNet-50 and VGG16 on CIFAR-10 in the gradient-compression README, BERT-Base
in the Birder README): the sizes are those models' parameter counts, the
values are random draws.  No dataset or trained weight is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# --------------------------------------------------------------------------
# Workload table
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    n: int                     # elements per worker (sum over tensors for a bucket)
    workers: int               # simulated data-parallel workers
    dist: str                  # "normal" | "laplace" | "normal+outliers" | "bert-bucket"
    scale: float               # std (normal) or b (laplace)
    neg_thr: float = 0.0
    pos_thr: float = 0.0
    iterations: int = 1
    seed_base: int = 0
    bits: tuple = field(default_factory=tuple)   # QSGD b values


WORKLOADS = {
    # 2-bit with error feedback on one 2^20 vector, thresholds +-0.5, 10 iterations.
    "ef2bit-1M": Workload("ef2bit-1M", 1 << 20, 1, "normal", 1.0, -0.5, 0.5, 10, 0),
    # ResNet-50-sized flat gradient, 4 workers, thresholds +-0.01.
    "resnet50-4w": Workload("resnet50-4w", 25_557_032, 4, "normal", 0.01, -0.01, 0.01, 1, 200),
    # VGG16-sized flat gradient, Laplace(0, 1e-3), thresholds +-2e-3, 8 workers, 5 iterations.
    "vgg16-8w": Workload("vgg16-8w", 138_357_544, 8, "laplace", 1e-3, -2e-3, 2e-3, 5, 300),
    # BERT-Base bucket of 197 bf16 tensors, per-tensor +-2 sigma thresholds, 4 workers.
    "bert-bucket-4w": Workload("bert-bucket-4w", 109_480_704, 4, "bert-bucket", 1e-3, 0.0, 0.0, 1, 400),
    # QSGD-MaxNorm: 2^27 N(0,1) plus 0.1% outliers of magnitude 50, 8 workers.
    "qsgd-128M-8w": Workload("qsgd-128M-8w", 1 << 27, 8, "normal+outliers", 1.0, 0.0, 0.0, 1, 500,
                             (2, 4, 8)),
}

QSGD_OUTLIER_MAGNITUDE = 50.0
QSGD_OUTLIER_FRACTION = 0.001
QSGD_SEED_BASE = 1234          # Philox seed of worker w is QSGD_SEED_BASE + w

# GRandK-MaxNorm keeps K = 10000 coordinates (the value the gradient-compression
# README's "Results" uses for every sparsified run) of the QSGD workload's
# gradients; the shared index is drawn once from its own seed.
GRANDK_K = 10_000
GRANDK_INDEX_SEED = 4321


def bert_base_shapes():
    """The 197 parameter tensors of BERT-Base, in model order."""
    shapes = [(30522, 768), (512, 768), (2, 768)]
    for _ in range(12):
        for _ in range(4):                       # Q, K, V, attention output
            shapes += [(768, 768), (768,)]
        shapes += [(768, 3072), (3072,), (3072, 768), (768,)]
        shapes += [(768,), (768,), (768,), (768,)]   # 2 x LayerNorm gamma, beta
    shapes += [(768, 768), (768,)]               # pooler
    return shapes


def bert_base_sizes():
    return [math.prod(s) for s in bert_base_shapes()]


# --------------------------------------------------------------------------
# Seeds and draws
# --------------------------------------------------------------------------

def input_seed(w: Workload, worker: int, iteration: int) -> int:
    """Seed of the torch generator that draws (worker, iteration)'s gradient."""
    return w.seed_base * 1_000_000 + worker * 1_000 + iteration


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(n: int, std: float, gen: torch.Generator, device, dtype=torch.float32):
    x = torch.empty(n, dtype=torch.float32, device=device)
    x.normal_(0.0, std, generator=gen)
    return x.to(dtype)


def laplace(n: int, b: float, gen: torch.Generator, device):
    """Laplace(0, b) by inverting its CDF on a uniform draw in (-1/2, 1/2)."""
    u = torch.rand(n, dtype=torch.float32, device=device, generator=gen) - 0.5
    u = u.clamp(-0.5 + 2**-25, 0.5 - 2**-25)
    x = -b * torch.sign(u) * torch.log1p(-2.0 * u.abs())
    return x.to(torch.float32)


def gradient(w: Workload, worker: int, iteration: int, device="cpu", n: int | None = None):
    """One flat fp32 gradient of workload ``w`` (first ``n`` elements if given)."""
    n = w.n if n is None else n
    gen = _gen(input_seed(w, worker, iteration), device)
    if w.dist == "normal":
        return normal(n, w.scale, gen, device)
    if w.dist == "laplace":
        return laplace(n, w.scale, gen, device)
    if w.dist == "normal+outliers":
        return qsgd_gradient(n, gen, device)
    raise ValueError(w.dist)


def gradient_stream(w: Workload, iterations: int, device="cpu", n: int | None = None):
    """Gradients of worker 0 for a workload drawn from ONE generator, one draw
    per iteration (the 2^20 error-feedback workload)."""
    n = w.n if n is None else n
    gen = _gen(input_seed(w, 0, 0), device)
    return [normal(n, w.scale, gen, device) for _ in range(iterations)]


def qsgd_gradient(n: int, gen: torch.Generator, device):
    """N(0,1) with round(0.001 n) positions (uniform, without replacement)
    set to +-50 with a random sign."""
    x = normal(n, 1.0, gen, device)
    k = int(round(QSGD_OUTLIER_FRACTION * n))
    if k:
        idx = torch.randperm(n, generator=gen, device=device)[:k]
        sign = torch.randint(0, 2, (k,), generator=gen, device=device).to(torch.float32) * 2 - 1
        x[idx] = sign * QSGD_OUTLIER_MAGNITUDE
    return x


def grandk_index(n: int, K: int = GRANDK_K, seed: int = GRANDK_INDEX_SEED):
    """K distinct coordinates of [0, n), uniform without replacement, in draw
    order: the index every worker keeps (int64 numpy array)."""
    import numpy as np
    return np.random.default_rng(seed).choice(n, size=K, replace=False).astype(np.int64)


def bert_bucket(w: Workload, worker: int, iteration: int, device="cpu", sizes=None):
    """The bf16 gradient tensors (flattened) of one worker's BERT-Base bucket."""
    sizes = bert_base_sizes() if sizes is None else sizes
    gen = _gen(input_seed(w, worker, iteration), device)
    return [normal(s, w.scale, gen, device, dtype=torch.bfloat16) for s in sizes]


def bert_thresholds(worker0_iter0_tensors):
    """Per-tensor thresholds +-2 sigma: sigma is the population standard
    deviation of worker 0's first gradient of that tensor, computed in fp64
    and rounded to fp32 once (2 sigma is exact in binary)."""
    neg, pos = [], []
    for t in worker0_iter0_tensors:
        x = t.detach().to("cpu", torch.float64)
        sigma = x.std(unbiased=False).item()
        p = float(torch.tensor(2.0 * sigma, dtype=torch.float32).item())
        neg.append(-p)
        pos.append(p)
    return neg, pos


def random_residual(n: int, scale: float, seed: int, device="cpu"):
    """A residual as it looks after some iterations: |r| below the threshold."""
    gen = _gen(seed, device)
    return (torch.rand(n, device=device, generator=gen) * 2 - 1).mul_(scale).to(torch.float32)
