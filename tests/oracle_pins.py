"""Pins of the CPU oracle to facts outside the oracle itself.

Each ``pin_*`` function takes a loaded oracle library (the real one, or a
deliberately broken copy in the mutation test) and raises AssertionError when
the library disagrees with:

* the worked example printed in MXNet pull request #8342 "[WIP] 2bit gradient
  compression" ("Two bit quantization", "Format of compressed gradient");
* closed forms (base-4 / base-2^b numerals for the bit layout, exact sums of
  powers of two for the merge, integer identities for QSGD);
* IEEE-754 rounding bounds checked in exact rational arithmetic, and the
  classic result that a binary32 sum or difference computed in binary64 and
  rounded once to binary32 is the correctly rounded binary32 result
  (53 >= 2*24 + 2);
* invariants of error feedback (a telescoping sum over iterations);
* published known-answer vectors of Philox4x32-10 (Salmon et al., SC'11);
* library routines (numpy's max of |x|, torch's bfloat16 widening);
* statistics of the stochastic rounding (uniformity of u, unbiasedness).
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
F32 = np.float32


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(" ")
            out[key] = val
    return out


def read_golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x, 16) for x in line.split()])
    return rows


def f32_of_bits(u):
    return np.array([u], np.uint32).view(np.float32)[0]


def bits_of_f32(x):
    return int(np.array([x], np.float32).view(np.uint32)[0])


def rn32_sum(a, b):
    """Correctly rounded binary32 a + b via one binary64 add (exact for these
    operands' sum up to one rounding, innocuous double rounding)."""
    return np.float32(np.float64(np.float32(a)) + np.float64(np.float32(b)))


def rn32_diff(a, b):
    return np.float32(np.float64(np.float32(a)) - np.float64(np.float32(b)))


def half_ulp(x):
    """Half of the binary32 unit in the last place of x, as a Fraction."""
    return Fraction(float(np.spacing(np.abs(np.float32(x))))) / 2


def base4_word(codes16):
    """A 32-bit word whose 16 two-bit digits, most significant first, are codes16."""
    w = 0
    for c in codes16:
        w = w * 4 + c
    return w


def base4_digits(word):
    """The 16 two-bit digits of a word, most significant first."""
    digits = []
    for _ in range(16):
        word, d = divmod(word, 4)
        digits.append(d)
    return digits[::-1]


def code_value(code, neg, pos):
    return {1: pos, 2: neg}.get(code, 0.0)


THRESHOLD_PAIRS = [(-2.0, 2.0), (-0.5, 0.5), (-0.01, 0.01), (-2e-3, 2e-3), (-0.75, 1.5),
                   (-3.0, 0.125)]


# ============================================================== 2-bit ====

def pin_worked_example(L):
    gold = read_golden("two_bit_worked_example.txt")
    neg, pos, n = float(gold["neg_threshold"]), float(gold["pos_threshold"]), int(gold["n"])
    codes = [int(c, 2) for c in gold["codes"].split()]
    # The page's figure with the input values is lost; these eight values
    # produce the printed codes and touch both thresholds exactly (2.0, -2.0).
    g = np.array([1.0, 2.5, -1.0, -3.0, 2.0, 0.5, 0.0, -2.0], np.float32)
    compr, res = oracle.quantize_2bit(g, np.zeros(n, np.float32), neg, pos, L)
    assert compr.size == 4, compr.size
    word = int(gold["word_bits"].replace(" ", ""), 2)
    assert int(compr[3]) == word == base4_word(codes + [0] * 8), hex(int(compr[3]))
    printed = [float(x) for x in gold["compr"].split()]
    assert f32_of_bits(compr[0]) == F32(printed[0])
    assert f32_of_bits(compr[1]) == F32(printed[1])
    assert f32_of_bits(compr[2]) == F32(printed[2])
    assert f32_of_bits(compr[3]) == F32(printed[3])
    # what each code does not carry stays behind: g - value(code), exact here
    expect = [gv - code_value(c, neg, pos) for gv, c in zip(g.tolist(), codes)]
    assert res.tolist() == expect, res.tolist()
    back = oracle.dequantize_2bit(compr, n, L)
    assert back.tolist() == [code_value(c, neg, pos) for c in codes]


def pin_all_code_patterns(L):
    """All 3^8 code sequences: inputs equal to the code values reproduce the
    codes, the base-4 numeral of the words, a zero residual and themselves
    after dequantization."""
    patterns = np.array(np.meshgrid(*[[0, 1, 2]] * 8, indexing="ij")).reshape(8, -1).T
    codes = patterns.reshape(-1)                      # 6561 * 8 = 52488 elements
    for neg, pos in [(-2.0, 2.0), (-0.75, 1.5)]:
        vals = np.where(codes == 1, pos, np.where(codes == 2, neg, 0.0)).astype(np.float32)
        compr, res = oracle.quantize_2bit(vals, np.zeros(vals.size, np.float32), neg, pos, L)
        assert not res.any(), "residual must vanish when g equals a code value"
        padded = np.concatenate([codes, np.zeros((-codes.size) % 16, codes.dtype)])
        words = [base4_word(padded[i:i + 16].tolist()) for i in range(0, padded.size, 16)]
        assert compr[3:].tolist() == words
        back = oracle.dequantize_2bit(compr, vals.size, L)
        assert np.array_equal(back, vals)


def _grid(neg, pos):
    vals = [0.0, -0.0, neg, pos, 2 * neg, 2 * pos, neg / 2, pos / 2, 1e-30, -1e-30, 3.0, -3.0]
    vals += [float(np.nextafter(F32(t), F32(d))) for t in (neg, pos) for d in (-np.inf, np.inf)]
    return np.array(vals, np.float32)


def pin_brute_force_grid(L):
    """Every (g, r) pair from a boundary grid, for six threshold pairs: the code
    follows the page's rule on the correctly rounded g + r, and the new
    residual is the correctly rounded difference."""
    for neg, pos in THRESHOLD_PAIRS:
        neg32, pos32 = F32(neg), F32(pos)
        grid = _grid(float(neg32), float(pos32))
        gg, rr = np.meshgrid(grid, grid, indexing="ij")
        g, r = gg.reshape(-1).copy(), rr.reshape(-1).copy()
        compr, res = oracle.quantize_2bit(g, r, neg32, pos32, L)
        for e in range(g.size):
            r1 = rn32_sum(g[e], r[e])
            if r1 >= pos32:
                code, dq = 1, pos32
            elif r1 <= neg32:
                code, dq = 2, neg32
            else:
                code, dq = 0, F32(0.0)
            got = (int(compr[3 + e // 16]) >> (30 - 2 * (e % 16))) & 3
            assert got == code, (neg, pos, g[e], r[e], got, code)
            want = rn32_diff(r1, dq)
            assert bits_of_f32(res[e]) == bits_of_f32(want), (g[e], r[e], res[e], want)


def pin_rounding_bounds(L):
    """Random inputs: the residual is within half an ulp of the exact
    g + r - value, where g + r is itself within half an ulp of exact."""
    rng = np.random.default_rng(11)
    n = 3000
    g = (rng.standard_normal(n) * 0.01).astype(np.float32)
    r = (rng.uniform(-0.01, 0.01, n)).astype(np.float32)
    neg, pos = F32(-0.01), F32(0.01)
    compr, res = oracle.quantize_2bit(g, r, neg, pos, L)
    for e in range(n):
        exact_r1 = Fraction(float(g[e])) + Fraction(float(r[e]))
        code = (int(compr[3 + e // 16]) >> (30 - 2 * (e % 16))) & 3
        assert code in (0, 1, 2)
        dq = Fraction(float(code_value(code, neg, pos)))
        # the code must be the one the rule assigns to SOME binary32 value
        # within half an ulp of the exact sum
        slack = half_ulp(float(exact_r1)) * 2
        if code == 1:
            assert exact_r1 >= Fraction(float(pos)) - slack
        elif code == 2:
            assert exact_r1 <= Fraction(float(neg)) + slack
        else:
            assert Fraction(float(neg)) - slack < exact_r1 < Fraction(float(pos)) + slack
        err = abs(Fraction(float(res[e])) - (exact_r1 - dq))
        assert err <= half_ulp(float(exact_r1)) + half_ulp(float(res[e])), (e, float(err))


def pin_error_feedback_telescopes(L):
    """Over T iterations nothing is lost: r_T + sum_t value_t equals
    r_0 + sum_t g_t up to the accumulated rounding of 2 roundings per step."""
    rng = np.random.default_rng(5)
    n, T = 2048, 25
    neg, pos = F32(-0.5), F32(0.5)
    r = np.zeros(n, np.float32)
    sent = [Fraction(0)] * n
    fed = [Fraction(0)] * n
    bound = [Fraction(0)] * n
    for _ in range(T):
        g = rng.standard_normal(n).astype(np.float32) * F32(0.3)
        compr, r_next = oracle.quantize_2bit(g, r, neg, pos, L)
        dq = oracle.dequantize_2bit(compr, n, L)
        for e in range(n):
            fed[e] += Fraction(float(g[e]))
            sent[e] += Fraction(float(dq[e]))
            bound[e] += 2 * half_ulp(abs(float(g[e])) + abs(float(r[e])) + float(pos))
        r = r_next
    for e in range(n):
        drift = abs(Fraction(float(r[e])) + sent[e] - fed[e])
        assert drift <= bound[e], (e, float(drift), float(bound[e]))


def pin_sizes_tail_and_header(L):
    """Word count 3 + ceil(n/16); unused tail codes are zero even when the
    output buffer held garbage; the header's third word is binary32(n)."""
    rng = np.random.default_rng(3)
    for n in list(range(0, 41)) + [255, 256, 257]:
        assert int(L.oracle_2bit_words(n)) == 3 + -(-n // 16)
        g = rng.standard_normal(n).astype(np.float32) * 3
        compr, _ = oracle.quantize_2bit(g, np.zeros(n, np.float32), -1.0, 1.0, L)
        assert compr.size == 3 + -(-n // 16)
        assert f32_of_bits(compr[2]) == F32(n)
        if n % 16:
            used = 2 * (n % 16)
            assert int(compr[-1]) & ((1 << (32 - used)) - 1) == 0
    # above 2^24 the header's n is rounded to nearest even: 2^24+1 is a tie
    # that goes down to 2^24, 2^24+3 a tie that goes up to 2^24+4
    for n, want in ((16_777_217, 16_777_216), (16_777_219, 16_777_220)):
        compr, _ = oracle.quantize_2bit(np.zeros(n, np.float32), np.zeros(n, np.float32),
                                        -1.0, 1.0, L)
        assert int(f32_of_bits(compr[2])) == want == int(F32(n))
    # garbage in the output buffer must not leak into the tail
    n = 21
    compr = np.full(int(L.oracle_2bit_words(n)), 0xFFFFFFFF, np.uint32)
    g = np.zeros(n, np.float32)
    r = np.zeros(n, np.float32)
    L.oracle_quantize_2bit(g.ctypes.data, r.ctypes.data, compr.ctypes.data, n, -1.0, 1.0)
    assert compr[3:].tolist() == [0, 0]


def pin_dequantize_random_words(L):
    """Random payload words (code 11 included) decode digit by digit."""
    rng = np.random.default_rng(7)
    for neg, pos in THRESHOLD_PAIRS:
        n = 16 * 37 + 5
        words = rng.integers(0, 1 << 32, 3 + -(-n // 16), dtype=np.uint64).astype(np.uint32)
        words[0], words[1], words[2] = bits_of_f32(neg), bits_of_f32(pos), bits_of_f32(n)
        out = oracle.dequantize_2bit(words, n, L)
        for e in range(n):
            d = base4_digits(int(words[3 + e // 16]))[e % 16]
            assert out[e] == F32(code_value(d, F32(neg), F32(pos))), (e, d, out[e])


def _random_record(rng, n, neg, pos):
    words = rng.integers(0, 1 << 32, 3 + -(-n // 16), dtype=np.uint64).astype(np.uint32)
    # clear code 11 (never produced by the quantizer): 11 -> 01
    payload = words[3:].astype(np.uint64)
    both = payload & (payload >> 1) & 0x55555555
    payload ^= (both << 1)
    words[3:] = payload.astype(np.uint32)
    words[0], words[1], words[2] = bits_of_f32(neg), bits_of_f32(pos), bits_of_f32(n)
    return words


def pin_merge_closed_form(L):
    """With power-of-two thresholds the merged value is exactly
    k+ * pos + k- * neg summed over workers (every partial sum exact)."""
    rng = np.random.default_rng(9)
    pow2 = [0.125, 0.25, 0.5, 1.0, 2.0]
    for W in (1, 2, 3, 4, 8):
        n = 16 * 20 + 3
        thr = [(-float(rng.choice(pow2)), float(rng.choice(pow2))) for _ in range(W)]
        recs = [_random_record(rng, n, a, b) for a, b in thr]
        out = oracle.dequant_accumulate_2bit(recs, n, L)
        for e in range(n):
            total = Fraction(0)
            for w in range(W):
                d = base4_digits(int(recs[w][3 + e // 16]))[e % 16]
                total += Fraction(code_value(d, *thr[w]))
            assert Fraction(float(out[e])) == total, (W, e)
        if W == 1:
            assert np.array_equal(out, oracle.dequantize_2bit(recs[0], n, L))


def pin_merge_order(L):
    """The sum starts at +0 and adds worker 0 first: 1 + 2^-24 + 2^-24 rounds
    back to 1 at each step (ties to even), whereas adding the two small
    values first would give 1 + 2^-23."""
    n = 16
    small = 2.0 ** -24
    recs = []
    for pos in (1.0, small, small):
        w = np.zeros(4, np.uint32)
        w[0], w[1], w[2] = bits_of_f32(-1.0), bits_of_f32(pos), bits_of_f32(n)
        w[3] = 0x40000000          # element 0 coded 01
        recs.append(w)
    out = oracle.dequant_accumulate_2bit(recs, n, L)
    assert out[0] == F32(1.0), out[0]
    assert not out[1:].any()
    # -0 never appears: an all-zero merge is +0
    assert bits_of_f32(out[1]) == 0


def pin_bf16_widening(L):
    """The bf16 operator equals the fp32 operator on torch's bf16 -> fp32
    conversion of the same gradient."""
    import torch
    rng = np.random.default_rng(13)
    n = 16 * 9 + 7
    g = torch.from_numpy(rng.standard_normal(n).astype(np.float32) * 0.02).to(torch.bfloat16)
    g_bits = g.view(torch.int16).numpy().view(np.uint16)
    g32 = g.to(torch.float32).numpy()
    r = rng.uniform(-0.01, 0.01, n).astype(np.float32)
    c1, r1 = oracle.quantize_2bit(g_bits, r, -0.02, 0.02, L)
    c2, r2 = oracle.quantize_2bit(g32, r, -0.02, 0.02, L)
    assert np.array_equal(c1, c2) and np.array_equal(r1.view(np.uint32), r2.view(np.uint32))


def pin_bucket_is_concatenation(L):
    """A bucket equals its tensors' standalone records one after the other;
    its merge equals the per-tensor merges."""
    rng = np.random.default_rng(17)
    sizes = [0, 1, 15, 16, 17, 33, 768, 5]
    W = 3
    thr = [(-float(a), float(a)) for a in rng.uniform(0.1, 1.0, len(sizes)).astype(np.float32)]
    buckets, res_all = [], []
    for w in range(W):
        grads = [rng.standard_normal(s).astype(np.float32) for s in sizes]
        res = [rng.uniform(-0.1, 0.1, s).astype(np.float32) for s in sizes]
        compr, new_res = oracle.quantize_2bit_bucket(grads, res, [a for a, _ in thr],
                                                     [b for _, b in thr], L)
        pieces = []
        for t, s in enumerate(sizes):
            c, rr = oracle.quantize_2bit(grads[t], res[t], thr[t][0], thr[t][1], L)
            pieces.append(c)
            assert np.array_equal(rr.view(np.uint32), new_res[t].view(np.uint32))
        assert np.array_equal(compr, np.concatenate(pieces))
        assert compr.size == sum(3 + -(-s // 16) for s in sizes)
        buckets.append((compr, pieces))
    merged = oracle.dequant_accumulate_2bit_bucket([b for b, _ in buckets], sizes, L)
    parts = [oracle.dequant_accumulate_2bit([buckets[w][1][t] for w in range(W)], s, L)
             for t, s in enumerate(sizes)]
    assert np.array_equal(merged, np.concatenate(parts))


# =============================================================== QSGD ====

def pin_philox_known_answers(L):
    for row in read_golden_rows("philox4x32_10_kat.txt"):
        ctr, key, want = row[0:4], row[4:6], row[6:10]
        got = oracle.philox4x32_10(ctr, key, L)
        assert got.tolist() == want, ([hex(x) for x in got], [hex(x) for x in want])


def pin_uniform_draws(L):
    """u is a multiple of 2^-24 in [0, 1), element e uses output word e mod 4
    of counter block e div 4, and the draws look uniform."""
    for seed in (0, 1234, (1 << 40) + 7):
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for blk in (0, 1, 5, (1 << 33) + 3):
            words = oracle.philox4x32_10([blk & 0xFFFFFFFF, blk >> 32, 0, 0], key, L)
            for lane in range(4):
                u = oracle.qsgd_uniform(seed, 4 * blk + lane, L)
                assert u == (int(words[lane]) >> 8) / 2.0 ** 24, (seed, blk, lane)
    us = np.array([oracle.qsgd_uniform(99, e, L) for e in range(40000)])
    assert us.min() >= 0.0 and us.max() < 1.0
    assert abs(us.mean() - 0.5) < 5 * (1 / 12) ** 0.5 / 200
    counts = np.histogram(us, bins=16, range=(0, 1))[0]
    chi2 = (((counts - 2500.0) ** 2) / 2500.0).sum()
    assert chi2 < 45, chi2          # 15 dof; p < 1e-4 above 45


def pin_max_is_library_max(L):
    rng = np.random.default_rng(19)
    for W in (1, 3, 8):
        gs = [np.clip(rng.standard_normal(1000 + 13) * rng.uniform(0.1, 5), -7, 7)
              .astype(np.float32) for _ in range(W)]
        gs[-1][500] = -7.25       # the largest magnitude, negative
        assert oracle.qsgd_mn_max(gs, L) == np.max(np.abs(np.stack(gs))) == F32(7.25)
    gs = [np.array([-0.0, 0.0, np.nan, 3.0], np.float32)]
    assert oracle.qsgd_mn_max(gs, L) == F32(3.0)          # NaN skipped
    assert oracle.qsgd_mn_max([np.full(5, -0.0, np.float32)], L) == 0.0


def pin_qsgd_levels_exact(L):
    """Away from integer boundaries, q = sign(g) * min(floor(|g|/M*s + u), s)
    in exact arithmetic; |q| <= s always; special cases."""
    rng = np.random.default_rng(23)
    for b in (2, 4, 8):
        s = 2 ** (b - 1) - 1
        M = F32(50.0)
        g = (rng.standard_normal(1500) * 10).astype(np.float32)
        g[:3] = [50.0, -50.0, 0.0]
        for e in range(g.size):
            seed = 1234 + (e % 8)
            q = oracle.qsgd_level(g[e], M, b, seed, e, L)
            assert abs(q) <= s
            u = Fraction(oracle.qsgd_uniform(seed, e, L))
            x = Fraction(abs(float(g[e]))) / Fraction(float(M)) * s + u
            fl = x.numerator // x.denominator
            dist = min(x - fl, fl + 1 - x)
            if dist > Fraction(1, 1 << 12):          # far above 3 roundings (< 2^-14 in all)
                want = min(fl, s)
                want = -want if g[e] < 0 else want
                assert q == want, (b, e, float(g[e]), q, want)
            assert oracle.qsgd_level(-g[e], M, b, seed, e, L) == (-q if g[e] != 0 else 0)
        assert oracle.qsgd_level(50.0, M, b, 1, 0, L) == s
        assert oracle.qsgd_level(60.0, M, b, 1, 0, L) == s         # capped at s
        assert oracle.qsgd_level(-75.0, M, b, 1, 3, L) == -s
        assert oracle.qsgd_level(-50.0, M, b, 1, 0, L) == -s
        assert oracle.qsgd_level(0.0, M, b, 1, 0, L) == 0
        assert oracle.qsgd_level(-0.0, M, b, 1, 0, L) == 0
        assert oracle.qsgd_level(0.0, 0.0, b, 1, 0, L) == 0      # M == 0
        assert oracle.qsgd_level(float("nan"), M, b, 1, 0, L) == 0


def pin_qsgd_unbiased(L):
    """E[q] * M / s = g: averaged over many independent draws the decoded
    value matches g within a few standard errors."""
    M = 4.0
    draws = 6000
    for b in (2, 4):
        s = 2 ** (b - 1) - 1
        for gval in (1.3, -2.9, 0.37, 3.99):
            q = np.array([oracle.qsgd_level(gval, M, b, 77, e, L) for e in range(draws)])
            est = q.mean() * M / s
            sd = (M / s) * 0.5 / np.sqrt(draws)
            assert abs(est - gval) < 5 * sd + 1e-6, (b, gval, est)


def _qsgd_digits(word, b):
    per = 32 // b
    out = []
    for _ in range(per):
        word, d = divmod(word, 1 << b)
        out.append(d - (1 << b) if d >= (1 << (b - 1)) else d)
    return out[::-1]


def pin_qsgd_record_layout(L):
    """Header [M, b, n]; 32/b two's-complement digits per word, most
    significant first, that equal the per-element levels; zero tail."""
    rng = np.random.default_rng(29)
    for b in (2, 4, 8):
        for n in (0, 1, 5, 16, 33, 257):
            g = (rng.standard_normal(n) * 2).astype(np.float32)
            M = F32(np.max(np.abs(g))) if n else F32(1.0)
            compr = oracle.qsgd_mn_quantize(g, b, 4321, M, L)
            assert compr.size == 3 + -(-(n * b) // 32) == int(L.oracle_qsgd_words(n, b))
            assert f32_of_bits(compr[0]) == M and f32_of_bits(compr[1]) == F32(b)
            assert f32_of_bits(compr[2]) == F32(n)
            digits = [d for w in compr[3:].tolist() for d in _qsgd_digits(int(w), b)]
            want = [oracle.qsgd_level(g[e], M, b, 4321, e, L) for e in range(n)]
            assert digits[:n] == want
            assert not any(digits[n:])


def pin_qsgd_merge_identity(L):
    """Merged value = (sum of integer levels) * binary32(M / s), the product
    correctly rounded; the step is within half an ulp of M / s."""
    rng = np.random.default_rng(31)
    for b in (2, 4, 8):
        s = 2 ** (b - 1) - 1
        W, n = 8, 16 * 11 + 9
        gs = [(rng.standard_normal(n) * 3).astype(np.float32) for _ in range(W)]
        M = oracle.qsgd_mn_max(gs, L)
        recs = [oracle.qsgd_mn_quantize(gs[w], b, 1234 + w, M, L) for w in range(W)]
        out = oracle.qsgd_mn_dequant_accumulate(recs, n, b, L)
        step = F32(np.float64(M) / np.float64(s))      # correctly rounded M / s
        assert abs(Fraction(float(step)) - Fraction(float(M)) / s) <= half_ulp(step)
        for e in range(n):
            total = sum(_qsgd_digits(int(recs[w][3 + e // (32 // b)]), b)[e % (32 // b)]
                        for w in range(W))
            want = F32(np.float64(total) * np.float64(step))    # exact product, one rounding
            assert out[e] == want, (b, e, out[e], want)


# ========================================================== QSGD-MN-TS ====

def _mnts_split(compr, n, b1):
    """The two sub-records of a two-scale record: coarse (b1 bits), fine."""
    k = 3 + -(-(n * b1) // 32)
    return compr[:k], compr[k:]


def _mnts_levels(sub, n, b):
    return [d for w in sub[3:].tolist() for d in _qsgd_digits(int(w), b)][:n]


def pin_qsgd_mnts_reduces_to_qsgd(L):
    """With b1 = 2 (s1 = 1) the fine scale equals the coarse one: the fine
    sub-record is the (pinned) QSGD-MaxNorm record of b2 bits, the coarse one
    holds only its header, and the merge is the QSGD-MaxNorm merge."""
    rng = np.random.default_rng(41)
    for b2 in (2, 4, 8):
        for n in (0, 1, 33, 257):
            W = 3
            gs = [(rng.standard_normal(n) * 2).astype(np.float32) for _ in range(W)]
            M = oracle.qsgd_mn_max(gs, L) if n else F32(1.0)
            recs, fines = [], []
            for w in range(W):
                ts = oracle.qsgd_mnts_quantize(gs[w], 2, b2, 900 + w, M, L)
                coarse, fine = _mnts_split(ts, n, 2)
                assert ts.size == oracle.qsgd_mnts_words(n, 2, b2, L) == coarse.size + fine.size
                assert np.array_equal(fine, oracle.qsgd_mn_quantize(gs[w], b2, 900 + w, M, L))
                assert coarse[:3].tolist() == [bits_of_f32(M), bits_of_f32(2.0), bits_of_f32(n)]
                assert not coarse[3:].any()
                recs.append(ts)
                fines.append(fine)
            got = oracle.qsgd_mnts_dequant_accumulate(recs, n, 2, b2, L)
            want = oracle.qsgd_mn_dequant_accumulate(fines, n, b2, L)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def pin_qsgd_mnts_scale_assignment(L):
    """Fine scale = binary32(M / s1) (correctly rounded); an element with
    |g| <= fine scale has its (pinned) QSGD-MaxNorm level on the fine scale
    with b2 bits and 0 on the coarse one, any other element the reverse;
    headers [M, b1, n] and [M2, b2, n]; |levels| <= s per scale."""
    rng = np.random.default_rng(43)
    for b1 in (4, 8):
        s1 = 2 ** (b1 - 1) - 1
        for b2 in (2, 4, 8):
            s2 = 2 ** (b2 - 1) - 1
            n = 301
            g = (rng.standard_normal(n) * 3).astype(np.float32)
            g[::37] = 50.0
            M = F32(np.max(np.abs(g)))
            M2 = oracle.qsgd_mnts_fine_scale(M, b1, L)
            assert abs(Fraction(float(M2)) - Fraction(float(M)) / s1) <= half_ulp(M2)
            g[5], g[6] = M2, -M2                                     # on the boundary: fine
            g[7] = np.nextafter(M2, F32(np.inf))                     # just above: coarse
            g[8] = -np.nextafter(M2, F32(0))                         # just below: fine
            seed = 77 + b1 + b2
            ts = oracle.qsgd_mnts_quantize(g, b1, b2, seed, M, L)
            coarse, fine = _mnts_split(ts, n, b1)
            assert coarse[:3].tolist() == [bits_of_f32(M), bits_of_f32(b1), bits_of_f32(n)]
            assert fine[:3].tolist() == [bits_of_f32(M2), bits_of_f32(b2), bits_of_f32(n)]
            q1, q2 = _mnts_levels(coarse, n, b1), _mnts_levels(fine, n, b2)
            for e in range(n):
                assert abs(q1[e]) <= s1 and abs(q2[e]) <= s2
                if abs(g[e]) <= M2:
                    assert q1[e] == 0 and q2[e] == oracle.qsgd_level(g[e], M2, b2, seed, e, L), (b1, b2, e)
                else:
                    assert q2[e] == 0 and q1[e] == oracle.qsgd_level(g[e], M, b1, seed, e, L), (b1, b2, e)
            assert q2[5] == s2 and q2[6] == -s2 and q1[5] == q1[6] == 0
            assert q2[7] == 0 and q1[7] >= 1 and q1[8] == 0


def pin_qsgd_mnts_unbiased(L):
    """E[value] = g on both scales: value = q1 M / s1 + q2 M2 / s2 averaged
    over many independent draws matches g within a few standard errors."""
    draws = 6000
    b1, b2 = 4, 4
    s1, s2 = 7, 7
    M = F32(7.0)                                   # fine scale M2 = 1
    for gval in (0.37, -0.9, 1.0, 2.6, -6.1):
        g = np.full(draws, gval, np.float32)
        ts = oracle.qsgd_mnts_quantize(g, b1, b2, 55, M, L)
        coarse, fine = _mnts_split(ts, draws, b1)
        q1 = np.array(_mnts_levels(coarse, draws, b1))
        q2 = np.array(_mnts_levels(fine, draws, b2))
        est = (q1 * (7.0 / s1) + q2 * (1.0 / s2)).mean()
        step = 1.0 / s2 if abs(gval) <= 1.0 else 7.0 / s1
        sd = step * 0.5 / np.sqrt(draws)
        assert abs(est - gval) < 5 * sd + 1e-6, (gval, est)


def pin_qsgd_mnts_merge_exact(L):
    """With power-of-two steps (M = 7/8, b1 = 4: coarse step 1/8, fine
    scale 1/8, b2 = 2: fine step 1/8) every product and the final add are
    exact: the merge equals (sum of coarse + fine levels) / 8."""
    rng = np.random.default_rng(47)
    n, W = 16 * 9 + 5, 8
    M = F32(0.875)
    gs = []
    for _ in range(W):
        g = (rng.uniform(-0.875, 0.875, n)).astype(np.float32)
        g[::5] *= F32(0.1)                         # plenty of fine elements
        gs.append(g)
    recs = [oracle.qsgd_mnts_quantize(gs[w], 4, 2, 600 + w, M, L) for w in range(W)]
    out = oracle.qsgd_mnts_dequant_accumulate(recs, n, 4, 2, L)
    total = np.zeros(n, np.int64)
    coarse_seen = fine_seen = False
    for r in recs:
        coarse, fine = _mnts_split(r, n, 4)
        q1, q2 = np.array(_mnts_levels(coarse, n, 4)), np.array(_mnts_levels(fine, n, 2))
        coarse_seen |= bool(q1.any())
        fine_seen |= bool(q2.any())
        total += q1 + q2
    assert coarse_seen and fine_seen
    assert np.array_equal(out, (total / 8.0).astype(np.float32))


# ======================================================= dense ternary ====

def _ternary_bytes(compr, nbytes):
    return [int(b) for b in compr[3:].view(np.uint8)[:nbytes]]


def _base3_digits(byte):
    digits = []
    for _ in range(5):
        byte, d = divmod(byte, 3)
        digits.append(d)
    return digits[::-1]


def pin_ternary_matches_2bit(L):
    """The dense record carries exactly the 2-bit operator's codes (a pinned
    routine) and leaves exactly its residual."""
    rng = np.random.default_rng(37)
    for n in (0, 1, 4, 5, 6, 19, 20, 21, 99, 1000):
        g = (rng.standard_normal(n) * 0.6).astype(np.float32)
        r = rng.uniform(-0.5, 0.5, n).astype(np.float32)
        c2, r2 = oracle.quantize_2bit(g, r, -0.5, 0.5, L)
        c3, r3 = oracle.quantize_ternary(g, r, -0.5, 0.5, L)
        assert np.array_equal(r2.view(np.uint32), r3.view(np.uint32)), n
        assert c3.size == 3 + -(-n // 20) == int(L.oracle_ternary_words(n))
        assert c3[:3].tolist() == c2[:3].tolist()
        trits = [d for b in _ternary_bytes(c3, -(-n // 5)) for d in _base3_digits(b)]
        codes = [(int(c2[3 + e // 16]) >> (30 - 2 * (e % 16))) & 3 for e in range(n)]
        assert trits[:n] == codes, n
        assert not any(trits[n:])
        # padding bytes past the last element's byte are zero
        assert not any(int(b) for b in c3[3:].view(np.uint8)[-(-n // 5):])


def pin_ternary_numeral(L):
    """All 3^5 trit patterns: a byte is the base-3 numeral of its five codes,
    first element most significant; the worked example's codes give bytes
    34 and 18 (word 0x00001222)."""
    gold = read_golden("two_bit_worked_example.txt")
    codes = [int(c, 2) for c in gold["codes"].split()]
    g = np.array([1.0, 2.5, -1.0, -3.0, 2.0, 0.5, 0.0, -2.0], np.float32)
    c, _ = oracle.quantize_ternary(g, np.zeros(8, np.float32), -2.0, 2.0, L)
    want = [0, 0]
    for i, t in enumerate(codes + [0, 0]):
        want[i // 5] = want[i // 5] * 3 + t
    assert _ternary_bytes(c, 2) == want == [34, 18]
    assert int(c[3]) == 0x1222
    patterns = np.array(np.meshgrid(*[[0, 1, 2]] * 5, indexing="ij")).reshape(5, -1).T
    codes = patterns.reshape(-1)                     # 243 * 5 elements
    vals = np.where(codes == 1, 1.5, np.where(codes == 2, -0.75, 0.0)).astype(np.float32)
    c, r = oracle.quantize_ternary(vals, np.zeros(vals.size, np.float32), -0.75, 1.5, L)
    assert not r.any()
    assert _ternary_bytes(c, 243) == list(range(243))
    assert np.array_equal(oracle.dequantize_ternary(c, vals.size, L), vals)


def pin_ternary_dequantize_and_merge(L):
    """Random bytes decode digit by digit; the merge of power-of-two
    thresholds is the exact sum; W = 1 equals dequantize."""
    rng = np.random.default_rng(41)
    n = 5 * 61 + 3
    pow2 = [0.25, 0.5, 1.0, 2.0]
    recs, thr = [], []
    for w in range(5):
        a, b = -float(rng.choice(pow2)), float(rng.choice(pow2))
        words = np.zeros(3 + -(-n // 20), np.uint32)
        words[:3] = np.array([a, b, n], np.float32).view(np.uint32)
        nbytes = -(-n // 5)
        bytes_ = rng.integers(0, 243, nbytes).astype(np.uint8)
        # trits past n stay zero
        last = _base3_digits(int(bytes_[-1]))
        keep = n - 5 * (nbytes - 1)
        v = 0
        for i, d in enumerate(last):
            v = v * 3 + (d if i < keep else 0)
        bytes_[-1] = v
        words[3:].view(np.uint8)[:nbytes] = bytes_
        recs.append(words)
        thr.append((a, b))
    out = oracle.dequantize_ternary(recs[0], n, L)
    trits = [d for b in _ternary_bytes(recs[0], -(-n // 5)) for d in _base3_digits(b)]
    assert out.tolist() == [code_value(t, *thr[0]) for t in trits[:n]]
    assert np.array_equal(oracle.dequant_accumulate_ternary(recs[:1], n, L), out)
    merged = oracle.dequant_accumulate_ternary(recs, n, L)
    all_trits = [[d for b in _ternary_bytes(r, -(-n // 5)) for d in _base3_digits(b)] for r in recs]
    for e in range(n):
        total = sum(Fraction(code_value(all_trits[w][e], *thr[w])) for w in range(len(recs)))
        assert Fraction(float(merged[e])) == total, e


# ====================================================== GRandK-MN ====

def _grandk_case(rng, n, K, W, sorted_index=False):
    gs = [(rng.standard_normal(n) * 2).astype(np.float32) for _ in range(W)]
    index = rng.choice(n, size=K, replace=False).astype(np.int64)
    if sorted_index:
        index.sort()
    if K:
        gs[W - 1][index[K // 2]] = -9.5          # the largest kept magnitude
    return gs, index


def pin_grandk_is_qsgd_of_kept_values(L):
    """The kept coordinates' record is the (pinned) QSGD-MaxNorm record of the
    K-vector g[index]: M is the library max over kept values of all workers,
    draws follow the position in the index list, the header holds K; the
    merge puts the QSGD merge of those records at the kept coordinates and
    +0 everywhere else.  With index = 0..n-1 everything is plain QSGD-MN."""
    rng = np.random.default_rng(41)
    for b in (2, 4, 8):
        for n, K, W in ((3001, 777, 3), (4099, 1, 2), (257, 257, 4), (1000, 33, 8)):
            gs, index = _grandk_case(rng, n, K, W)
            M = oracle.grandk_mn_max(gs, index, L)
            kept = [g[index] for g in gs]
            assert M == np.max(np.abs(np.stack(kept))) == oracle.qsgd_mn_max(kept, L)
            recs = []
            for w in range(W):
                rec = oracle.grandk_mn_quantize(gs[w], index, b, 1234 + w, M, L)
                assert np.array_equal(rec, oracle.qsgd_mn_quantize(kept[w], b, 1234 + w, M, L))
                recs.append(rec)
            out = oracle.grandk_mn_dequant_accumulate(recs, index, n, b, L)
            want = np.zeros(n, np.float32)
            want[index] = oracle.qsgd_mn_dequant_accumulate(recs, K, b, L)
            assert np.array_equal(out.view(np.uint32), want.view(np.uint32)), (b, n, K)
        # the identity selection is QSGD-MN itself
        gs = [(rng.standard_normal(500) * 3).astype(np.float32) for _ in range(2)]
        ident = np.arange(500, dtype=np.int64)
        M = oracle.grandk_mn_max(gs, ident, L)
        assert M == oracle.qsgd_mn_max(gs, L)
        recs = [oracle.grandk_mn_quantize(g, ident, b, 9 + w, M, L) for w, g in enumerate(gs)]
        assert all(np.array_equal(r, oracle.qsgd_mn_quantize(g, b, 9 + w, M, L))
                   for w, (r, g) in enumerate(zip(recs, gs)))
        assert np.array_equal(oracle.grandk_mn_dequant_accumulate(recs, ident, 500, b, L),
                              oracle.qsgd_mn_dequant_accumulate(recs, 500, b, L))


def pin_grandk_skips_outside_coordinates_and_empty(L):
    """Coordinates outside [0, n) do not enter M, get level 0 and are not
    stored; K = 0 gives a header-only record and an all +0 merge."""
    rng = np.random.default_rng(43)
    n = 600
    for b in (2, 8):
        gs, index = _grandk_case(rng, n, 40, 2)
        index[[3, 17, 29]] = [-1, n, 1 << 40]
        valid = (index >= 0) & (index < n)
        M = oracle.grandk_mn_max(gs, index, L)
        assert M == np.max(np.abs(np.stack([g[index[valid]] for g in gs])))
        recs = []
        for w, g in enumerate(gs):
            x = np.zeros(index.size, np.float32)
            x[valid] = g[index[valid]]
            rec = oracle.grandk_mn_quantize(g, index, b, 70 + w, M, L)
            assert np.array_equal(rec, oracle.qsgd_mn_quantize(x, b, 70 + w, M, L))
            recs.append(rec)
        out = oracle.grandk_mn_dequant_accumulate(recs, index, n, b, L)
        want = np.zeros(n, np.float32)
        want[index[valid]] = oracle.qsgd_mn_dequant_accumulate(recs, index.size, b, L)[valid]
        assert np.array_equal(out.view(np.uint32), want.view(np.uint32))
        empty = np.zeros(0, np.int64)
        assert oracle.grandk_mn_max(gs, empty, L) == 0.0
        rec0 = oracle.grandk_mn_quantize(gs[0], empty, b, 1, F32(2.0), L)
        assert rec0.tolist() == [bits_of_f32(2.0), bits_of_f32(b), 0]
        assert not oracle.grandk_mn_dequant_accumulate([rec0], empty, n, b, L).view(np.uint32).any()


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
