"""Plant plausible mistakes in copies of the oracle (CPU only) and check that the pins catch each.

Every mutant is a textual edit of ``oracle/rra_oracle.c`` compiled to a temporary library; the
real oracle source is never modified.
"""
import os
import subprocess
import sys

import pytest

import oracle_pins
from oracle import oracle as O

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "rra_oracle.c")

L2_LOOP = """    score_zero(s);
    for (int c = 0; c < C; ++c)
        score_add_square(s, load_elem(x, dtype, row * C + c));"""

MUTANTS = {
    "drop_scale": ("s[j] = acc * scale;", "s[j] = acc;"),
    "max_sign": ("s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);"),
    "no_max_shift": ("s[j] = exp(s[j] - m);", "s[j] = exp(s[j]);"),
    "no_denominator": ("out[c] = acc / denom;", "out[c] = acc;"),
    "key_wrong_head": ("load_elem(k, dtype, ((seq_start + j) * H + h) * (int64_t)d + c)",
                       "load_elem(k, dtype, ((seq_start + j) * H + 0) * (int64_t)d + c)"),
    "qk_transposed": ("load_elem(q, dtype, (t * H + h) * (int64_t)d + c) *",
                      "load_elem(q, dtype, ((seq_start + j) * H + h) * (int64_t)d + c) *"),
    "value_from_query_row": ("acc += s[j] * load_elem(v, dtype, ((seq_start + j) * H + h) * (int64_t)d + c);",
                             "acc += s[j] * load_elem(v, dtype, (t * H + h) * (int64_t)d + c);"),
    "causal": ("for (int64_t j = 0; j < L; ++j) {\n        double acc = 0.0;",
               "for (int64_t j = 0; j < L; ++j) {\n        if (seq_start + j > t) { s[j] = -INFINITY; continue; }\n        double acc = 0.0;"),
    "last_key_dropped": ("for (int64_t j = 0; j < L; ++j) {\n        s[j] = exp(s[j] - m);",
                         "for (int64_t j = 0; j < L; ++j) {\n        s[j] = (j == L - 1) ? 0.0 : exp(s[j] - m);"),
    "rank_off_by_one": ("rank[(int64_t)b * N + n] = r++;", "rank[(int64_t)b * N + n] = ++r;"),
    "cu_not_cumulative": ("cu[b + 1] = (int32_t)run;", "cu[b + 1] = (int32_t)run; run = 0;"),
    "pack_reverse_order": ("int64_t out_row = (int64_t)cu[b] + r;",
                           "int64_t out_row = (int64_t)cu[b + 1] - 1 - r;"),
    "pack_ignores_capacity": ("if (out_row >= capacity)\n                continue;", ""),
    "unpack_no_fill": ("memset(out, 0, (size_t)row_bytes);", ";"),
    "unpack_wrong_row": ("int64_t src_row = (int64_t)cu[b] + r;", "int64_t src_row = (int64_t)b * N + n;"),
    "f16_bias": ("v = ldexp((double)(1024 + m), e - 25);", "v = ldexp((double)(1024 + m), e - 24);"),
    "f16_subnormal": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "bf16_truncated": ("uint32_t u = ((uint32_t)b) << 16;", "uint32_t u = ((uint32_t)(b & 0xFFF0)) << 16;"),
    "l2_tie_takes_higher_index": ("if (cand[n] && (best < 0 || score_cmp(&score[n], &score[best]) > 0))",
                                  "if (cand[n] && (best < 0 || score_cmp(&score[n], &score[best]) >= 0))"),
    "l2_cls_not_forced": ("        mask[(int64_t)b * N] = 1;\n        if (k_keep != NULL) {",
                          "        if (k_keep != NULL) {"),
    "l2_ignores_previous_stage": ("cand[n] = (char)(n >= 1 && (prev == NULL || prev[(int64_t)b * N + n] != 0));",
                                  "cand[n] = (char)(n >= 1);"),
    "l2_threshold_strict": ("score_cmp(&score[n], &thr) >= 0)", "score_cmp(&score[n], &thr) > 0)"),
    "l2_is_l1": ("words_add(s->w, m * m, 2 * e - SCORE_EMIN);", "words_add(s->w, m, e - SCORE_EMIN);"),
    # the exact score replaced by rounded accumulations: single precision in index order,
    # double precision in index order, double precision in reverse order
    "l2_fp32_chain": (L2_LOOP, "    float f = 0.0f;\n    for (int c = 0; c < C; ++c) { float v = (float)load_elem(x, dtype, row * C + c); "
                      "f = fmaf(v, v, f); }\n    if (isnan(f)) { score_zero(s); s->cls = SCORE_NAN; } else score_ceil(s, f);"),
    "l2_fp64_chain": (L2_LOOP, "    double f = 0.0;\n    for (int c = 0; c < C; ++c) { double v = load_elem(x, dtype, row * C + c); "
                      "f = fma(v, v, f); }\n    if (isnan(f)) { score_zero(s); s->cls = SCORE_NAN; } else score_ceil(s, f);"),
    "l2_fp64_reversed": (L2_LOOP, "    double f = 0.0;\n    for (int c = C - 1; c >= 0; --c) { double v = load_elem(x, dtype, row * C + c); "
                         "f = fma(v, v, f); }\n    if (isnan(f)) { score_zero(s); s->cls = SCORE_NAN; } else score_ceil(s, f);"),
    "l2_carry_dropped": ("        carry = t >> 32;", "        carry = 0;"),
    "l2_square_bit_off_by_one": ("words_add(s->w, m * m, 2 * e - SCORE_EMIN);", "words_add(s->w, m * m, 2 * e - SCORE_EMIN + 1);"),
    "l2_inf_not_above_finite": ("        if (s->cls != SCORE_NAN)\n            s->cls = SCORE_INF;", "        ;"),
    "mask_byte_is_bool": ("if (mask[(int64_t)b * N + n] != 0)\n                run += 1;",
                          "if (mask[(int64_t)b * N + n] == 1)\n                run += 1;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib_path = str(tmp_path / "libmutant.so")
    O.build(src=str(src), out=lib_path, extra_flags=("-w",))
    # Run the pins in a child process: a mutant that writes out of bounds may crash, which
    # also counts as caught.
    tests_dir = os.path.dirname(os.path.abspath(__file__))
    code = (
        "import sys; sys.path[:0] = [%r, %r]\n"
        "import oracle_pins\n"
        "from oracle import oracle as O\n"
        "lib = O.load(%r)\n"
        "bad = []\n"
        "for pin in oracle_pins.ALL_PINS:\n"
        "    try:\n"
        "        pin(lib)\n"
        "    except Exception:\n"
        "        bad.append(pin.__name__)\n"
        "print('FAILED_PINS', bad)\n"
        "sys.exit(3 if bad else 0)\n"
    ) % (tests_dir, os.path.dirname(tests_dir), lib_path)
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert proc.returncode != 0, f"mutant {name} passed every pin: {proc.stdout[-500:]}"
