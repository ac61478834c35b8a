"""Plausible mistakes planted in a copy of the oracle must fail a pin.

Each mutant is one small edit of ``oracle/qga_oracle.c`` -- a flipped
comparison, a dropped term, a wrong sign, index or shift, a typo in a
constant.  The copy is compiled into a temporary library and every pin is run
against it; at least one pin has to reject it.  This shows the pins would
catch such a mistake in the oracle itself.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "qga_oracle.c")

MUTANTS = [
    ("pos threshold strict", "if (value >= pos_thr)", "if (value > pos_thr)"),
    ("neg threshold strict", "if (value <= neg_thr)", "if (value < neg_thr)"),
    ("codes swapped", "        return 1u;\n    if (value <= neg_thr)\n        return 2u;",
     "        return 2u;\n    if (value <= neg_thr)\n        return 1u;"),
    ("residual not added", "float with_residual = grad + *residual;",
     "float with_residual = grad;"),
    ("residual sign", "*residual = with_residual - two_bit_value",
     "*residual = with_residual + two_bit_value"),
    ("residual not updated", "*residual = with_residual - two_bit_value(code, neg_thr, pos_thr);",
     "*residual = with_residual;"),
    ("lsb-first packing", "return 30 - 2 * (int)(e % 16);", "return 2 * (int)(e % 16);"),
    ("header n as integer", "compr[2] = bits_of((float)n); /* the example",
     "compr[2] = (uint32_t)n; /* the example"),
    ("qsgd header n as integer", "compr[2] = bits_of((float)n);\n    for (int64_t w = 0; w < (n * b",
     "compr[2] = (uint32_t)n;\n    for (int64_t w = 0; w < (n * b"),
    ("header thresholds swapped", "compr[0] = bits_of(neg_thr);\n    compr[1] = bits_of(pos_thr);",
     "compr[0] = bits_of(pos_thr);\n    compr[1] = bits_of(neg_thr);"),
    ("decode values swapped", "    if (code == 1u)\n        return pos_thr;",
     "    if (code == 1u)\n        return neg_thr;"),
    ("merge in reverse worker order",
     "for (int w = 0; w < W; ++w) {\n            float neg_thr = float_of(compr[w][0]);\n"
     "            float pos_thr = float_of(compr[w][1]);\n            sum = sum + two_bit_value(two_bit_code_at",
     "for (int w = W - 1; w >= 0; --w) {\n            float neg_thr = float_of(compr[w][0]);\n"
     "            float pos_thr = float_of(compr[w][1]);\n            sum = sum + two_bit_value(two_bit_code_at"),
    ("merge uses worker 0 thresholds",
     "            float pos_thr = float_of(compr[w][1]);\n            sum = sum + two_bit_value(two_bit_code_at",
     "            float pos_thr = float_of(compr[0][1]);\n            sum = sum + two_bit_value(two_bit_code_at"),
    ("ternary merge uses worker 0 thresholds",
     "            float pos_thr = float_of(compr[w][1]);\n            sum = sum + two_bit_value(ternary_code_at",
     "            float pos_thr = float_of(compr[0][1]);\n            sum = sum + two_bit_value(ternary_code_at"),
    ("bf16 widening shift", "return float_of((uint32_t)h << 16);",
     "return float_of((uint32_t)h << 15);"),
    ("bucket offset without header", "        offset += oracle_2bit_words(n[t]);",
     "        offset += (n[t] + 15) / 16;"),
    ("philox key dropped", "next[0] = (uint32_t)(p1 >> 32) ^ ctr[1] ^ key[0];",
     "next[0] = (uint32_t)(p1 >> 32) ^ ctr[1];"),
    ("philox weyl typo", "key[1] += 0xBB67AE85u;", "key[1] += 0xBB67AE86u;"),
    ("philox nine rounds", "for (int round = 0; round < 10; ++round)",
     "for (int round = 0; round < 9; ++round)"),
    ("counter in high words", "uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), 0u, 0u};",
     "uint32_t ctr[4] = {0u, 0u, (uint32_t)block, (uint32_t)(block >> 32)};"),
    ("wrong output lane", "return (float)(out[e % 4] >> 8) * 0x1p-24f;",
     "return (float)(out[0] >> 8) * 0x1p-24f;"),
    ("max of signed values", "float a = fabsf(grad[w][e]);", "float a = grad[w][e];"),
    ("scale multiplies", "float scaled = fabsf(grad) / M;", "float scaled = fabsf(grad) * M;"),
    ("no stochastic draw", "float t = stretched + u;", "float t = stretched;"),
    ("no cap at s", "    if (level > (float)s)\n        level = (float)s;\n", ""),
    ("sign dropped", "return grad < 0.0f ? -q : q;", "return q;"),
    ("qsgd lsb-first", "int shift = 32 - b * (int)(e % per_word + 1);\n        compr[3 + e / per_word] |=",
     "int shift = b * (int)(e % per_word);\n        compr[3 + e / per_word] |="),
    ("no sign extension", "        q -= (int32_t)(1u << b);", "        q += 0;"),
    ("merge step 2^(b-1)", "float step = M / (float)qsgd_levels(b);\n    for (int64_t e = 0; e < n; ++e) {",
     "float step = M / (float)(1 << (b - 1));\n    for (int64_t e = 0; e < n; ++e) {"),
    ("grandk merge step 2^(b-1)",
     "float step = M / (float)qsgd_levels(b);\n    for (int64_t e = 0; e < n; ++e)\n",
     "float step = M / (float)(1 << (b - 1));\n    for (int64_t e = 0; e < n; ++e)\n"),
    ("ternary base 4", "            value = value * 3 + trit;", "            value = value * 4 + trit;"),
    ("ternary least significant first", "    for (int64_t k = e % 5; k < 4; ++k)\n        value /= 3;",
     "    for (int64_t k = 0; k < e % 5; ++k)\n        value /= 3;"),
    ("ternary words per 16", "    return 3 + (n + 19) / 20;", "    return 3 + (n + 15) / 16;"),
    ("ts boundary strict", "int is_fine = fabsf(grad) <= M2;", "int is_fine = fabsf(grad) < M2;"),
    ("ts fine scale is M", "return M / (float)qsgd_levels(b1);", "return M;"),
    ("ts fine level with coarse bits", "oracle_qsgd_level(grad, M2, b2, seed, e)",
     "oracle_qsgd_level(grad, M2, b1, seed, e)"),
    ("ts fine draw of the next element", "oracle_qsgd_level(grad, M2, b2, seed, e)",
     "oracle_qsgd_level(grad, M2, b2, seed, e + 1)"),
    ("ts merge fine step from coarse header", "float step2 = float_of(compr[0][fine_off])",
     "float step2 = float_of(compr[0][0])"),
    ("ts merge drops coarse part", "out[e] = coarse_part + fine_part;", "out[e] = fine_part;"),
    ("ts fields swapped", "q[0] = is_fine ? 0 : oracle_qsgd_level",
     "q[0] = !is_fine ? 0 : oracle_qsgd_level"),
    ("grandk draw keyed on coordinate", "q = oracle_qsgd_level(grad[index[k]], M, b, seed, k);",
     "q = oracle_qsgd_level(grad[index[k]], M, b, seed, index[k]);"),
    ("grandk level of position k", "q = oracle_qsgd_level(grad[index[k]], M, b, seed, k);",
     "q = oracle_qsgd_level(grad[k], M, b, seed, k);"),
    ("grandk header holds n", "compr[2] = bits_of((float)K);", "compr[2] = bits_of((float)n);"),
    ("grandk max over leading values", "float a = fabsf(grad[w][index[k]]);",
     "float a = fabsf(grad[w][k]);"),
    ("grandk merge not cleared", "    for (int64_t e = 0; e < n; ++e)\n        out[e] = 0.0f;\n", ""),
    ("grandk scatter to position", "out[index[k]] = (float)sum * step;", "out[k] = (float)sum * step;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique/not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                    "-shared", "-o", str(so), str(path), "-lm"], check=True)
    L = oracle.lib(str(so))
    failures = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(L)
        except AssertionError:
            failures.append(pin.__name__)
            break
    assert failures, f"mutant '{name}' passed every pin"
