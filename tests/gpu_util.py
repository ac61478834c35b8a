"""Helpers shared by the GPU parity tests (test plumbing, no method arithmetic)."""
from __future__ import annotations

import numpy as np
import torch

DEV = "cuda"

# Aggregates of W workers: the acceptance bar for fp32 sums whose order may
# differ (relative 1e-6 plus absolute 1e-7).  The 2-bit merge adds in the same
# worker order as the oracle and is also checked bit for bit.
AGG_RTOL = 1e-6
AGG_ATOL = 1e-7


def qga():
    import quantized_gradient_aggregation_b200 as q
    return q


def u32(t: torch.Tensor) -> np.ndarray:
    """Device int32 words -> host uint32 array."""
    return t.detach().cpu().numpy().view(np.uint32)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float32, copy=False)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def same_bits_f32(a: np.ndarray, b: np.ndarray) -> bool:
    """Bitwise equality, except that any NaN equals any NaN (the GPU returns
    the canonical NaN where the CPU keeps an input NaN's payload)."""
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    if a.shape != b.shape:
        return False
    na, nb = np.isnan(a), np.isnan(b)
    if not np.array_equal(na, nb):
        return False
    return np.array_equal(a[~na].view(np.uint32), b[~nb].view(np.uint32))


def first_diff(a, b):
    a = np.asarray(a)
    b = np.asarray(b)
    idx = np.flatnonzero(a.view(np.uint32) != b.view(np.uint32)) if a.dtype == np.float32 else \
        np.flatnonzero(a != b)
    return (int(idx[0]), a.flat[idx[0]], b.flat[idx[0]]) if idx.size else None


def offset_view(n: int, dtype, offset_elems: int, fill=None):
    """A contiguous CUDA tensor of n elements starting offset_elems past a
    256-byte-aligned allocation (exercises the misaligned scalar path)."""
    base = torch.empty(n + offset_elems + 8, dtype=dtype, device=DEV)
    if fill is not None:
        base.fill_(fill)
    return base[offset_elems:offset_elems + n]


def sample_words(nwords: int, count: int, seed: int) -> np.ndarray:
    """Word indices to check at full size: the first and last few plus a
    uniform random sample."""
    rng = np.random.default_rng(seed)
    pick = set(range(min(4, nwords))) | set(range(max(0, nwords - 4), nwords))
    pick |= set(rng.integers(0, nwords, min(count, nwords)).tolist())
    return np.array(sorted(pick), np.int64)


def gather_elems(t: torch.Tensor, word_idx: np.ndarray, per_word: int, n: int):
    """Elements [per_word*k, per_word*k + per_word) for each sampled word k,
    clipped to n; returns (host values, list of (start, stop) per word)."""
    spans = [(int(k) * per_word, min(int(k) * per_word + per_word, n)) for k in word_idx]
    idx = np.concatenate([np.arange(a, b) for a, b in spans]) if spans else np.zeros(0, np.int64)
    vals = t.index_select(0, torch.from_numpy(idx).to(t.device)).cpu()
    return vals, spans
