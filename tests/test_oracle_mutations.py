"""Planted-mistake check of the oracle pins (CPU only).

Each case copies oracle/oracle.c into a temporary directory, plants one plausible
mistake (a dropped term, a wrong sign, index or comparison, a transposed operand, a
wrong order), compiles it, and runs the pin tests against the mutant.  Every mutant must
make at least one pin fail; a mutant that passes every pin would mean the pins cannot
tell that mistake from the definition.  Mistakes are planted only in the copy; the
real oracle is untouched.
"""
import os
import subprocess
import sys

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")
TESTS = os.path.dirname(os.path.abspath(__file__))

# Pin groups, run in a child process by name (a mutant may also crash the process, which
# counts as rejected).
FORMAT_PINS = "format"
SELECT_PINS = "select"
PRODUCT_PINS = "products"
HALF_PINS = "half"
FFN_PINS = "ffn"
TOKEN_PINS = "tokens"
SPLIT_PINS = "split24"

CHILD = {
    "half": "import test_oracle_half as H; H.test_all_half_patterns_match_numpy()",
    "format": ("import test_oracle_format as F\n"
               "for c in F.GOLDEN: F.test_golden_encode(c); F.test_golden_decode(c)\n"
               "F.test_random_masks(257, 511, 0.5)\n"
               "F.test_kept_signed_zero_and_specials_preserved()"),
    "select": ("import test_oracle_select as S\n"
               "[S.test_threshold_brute_force(s) for s in range(40)]\n"
               "S.test_threshold_special_cases()\n"
               "[S.test_topk_brute_force(s) for s in range(30)]\n"
               "S.test_topk_ties_prefer_lower_index()"),
    "products": ("import test_oracle_products as P\n"
                 "[P.test_spmv_exact_rational(s) for s in range(25)]\n"
                 "P.test_spmv_matches_numpy(65, 130, 3, 0.0)\n"
                 "P.test_spmv_act_bits_restrict_columns(); P.test_identity_is_exact()\n"
                 "P.test_diagonal_is_exact(); P.test_spmm_matches_numpy_and_rows()\n"
                 "P.test_spmm_transposed_operand_would_fail()"),
    "ffn": ("import test_oracle_ffn as Q\n"
            "Q.test_round_to_half_matches_numpy(); Q.test_round_to_half_round_trip_and_ties()\n"
            "Q.test_silu_mul_worked_value(); Q.test_silu_odd_part_identity()\n"
            "Q.test_silu_limits_and_zeros()"),
    "tokens": ("import test_oracle_tokens as G\n"
               "[G.test_spmm_tokens_exact_rational(s) for s in range(20)]\n"
               "[G.test_each_row_is_that_tokens_decode(t) for t in (0.0, 0.4, 1.2)]\n"
               "G.test_threshold_zero_is_the_plain_product(); G.test_rule_boundary_and_rows()\n"
               "G.test_groups_reverse_order_closed_form()\n"
               "G.test_groups_equal_signatures_keep_index_order()\n"
               "G.test_groups_word_zero_decides_first_and_threshold_counts()\n"
               "[G.test_groups_match_vectorised_restatement(s) for s in range(12)]"),
    "split24": ("import test_oracle_split24 as S\n"
                "S.test_hand_example(); S.test_structured_mask_has_empty_residual()\n"
                "S.test_partition_and_counts(33, 130, 0.5); S.test_partition_and_counts(64, 257, 0.7)\n"
                "S.test_parts_sum_to_the_product()"),
}

MUTANTS = [
    ("subnormal_exponent", "ldexp((double)fraction, -24)", "ldexp((double)fraction, -25)",
     [HALF_PINS]),
    ("normal_bias", "exponent - 25);", "exponent - 24);", [HALF_PINS]),
    ("row_major_tile_order",
     "for (int k = (int)kt * TCB_COLS; k < ((int)kt + 1) * TCB_COLS; k++)\n                for (int r = 0; r < TCB_ROWS; r++) {\n                    int n = (int)s * TCB_ROWS + r;\n                    if (!kept(",
     "for (int r = 0; r < TCB_ROWS; r++)\n                for (int k = (int)kt * TCB_COLS; k < ((int)kt + 1) * TCB_COLS; k++) {\n                    int n = (int)s * TCB_ROWS + r;\n                    if (!kept(",
     [FORMAT_PINS]),
    ("no_tile_padding", "uint64_t tile_units = (j + 7) / 8;", "uint64_t tile_units = (j + 8) / 8;",
     [FORMAT_PINS]),
    ("bit_reversed", "word |= 1ull << r;", "word |= 1ull << (63 - r);", [FORMAT_PINS]),
    ("section_not_aligned", "g.off_values = round_up(g.off_tileptr + 4 * (n_tiles + 1), 256);",
     "g.off_values = round_up(g.off_tileptr + 4 * (n_tiles + 1), 16);", [FORMAT_PINS]),
    ("threshold_le", "!(fabs(v) < t)", "!(fabs(v) <= t)", [SELECT_PINS, PRODUCT_PINS]),
    ("zeros_kept", "return v != 0.0 && !(fabs(v) < t);", "return !(fabs(v) < t);", [SELECT_PINS]),
    ("topk_ties_high_first", "return (p->index > q->index) - (p->index < q->index);",
     "return (p->index < q->index) - (p->index > q->index);", [SELECT_PINS]),
    ("topk_signed_score", "s += fabs(v);", "s += v;", [SELECT_PINS]),
    ("spmv_act_ignored", "if (act_bits && !((act_bits[k / 32] >> (k % 32)) & 1)) continue;",
     "", [PRODUCT_PINS]),
    ("spmv_transposed_mask", "if (!mask[(size_t)n * ld_mask + k]) continue;",
     "if (!mask[((size_t)n * ld_mask + k) % ((size_t)N * K)]) continue; if (k == 1) continue;",
     [PRODUCT_PINS]),
    ("spmm_transposed", "orc_half_to_double(X[(size_t)m * ldx + k]) *",
     "orc_half_to_double(X[(size_t)m * ldx + (K - 1 - k)]) *", [PRODUCT_PINS]),
    ("spmv_dropped_term", "acc += orc_half_to_double(W[(size_t)n * ldw + k]) * v;",
     "if (k + 1 < K) acc += orc_half_to_double(W[(size_t)n * ldw + k]) * v;", [PRODUCT_PINS]),
    ("silu_exponent_sign", "double silu = gv / (1.0 + exp(-gv));",
     "double silu = gv / (1.0 + exp(gv));", [FFN_PINS]),
    ("silu_mul_dropped_factor", "h[(size_t)b * ld + r] = orc_double_to_half(silu * uv);",
     "h[(size_t)b * ld + r] = orc_double_to_half(silu);", [FFN_PINS]),
    ("half_ties_away", "if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;",
     "if (frac >= 0.5) r += 1.0;", [FFN_PINS]),
    ("half_no_carry", "    if (r == 2048.0) {", "    if (r == 4096.0) {", [FFN_PINS]),
    ("tokens_rule_ignored",
     "if (!passes_threshold(xv, (double)t)) continue; /* k is not in token m's set */", "",
     [TOKEN_PINS]),
    ("tokens_other_token", "double xv = orc_half_to_double(X[(size_t)m * ldx + k]);",
     "double xv = orc_half_to_double(X[(size_t)(M - 1 - m) * ldx + k]);", [TOKEN_PINS]),
    ("token_order_reversed",
     "if (x->sig[w] != y->sig[w]) return x->sig[w] < y->sig[w] ? -1 : 1;",
     "if (x->sig[w] != y->sig[w]) return x->sig[w] < y->sig[w] ? 1 : -1;", [TOKEN_PINS]),
    ("token_ties_high_first", "return (x->token > y->token) - (x->token < y->token);",
     "return (x->token < y->token) - (x->token > y->token);", [TOKEN_PINS]),
    ("token_ktile_width", "int kt = k / 64;", "int kt = k / 32;", [TOKEN_PINS]),
    ("token_tile_shifted", "tile_sig[(size_t)(r / T) * words + w] |= keys[r].sig[w];",
     "tile_sig[(size_t)(((r + 1) % M) / T) * words + w] |= keys[r].sig[w];", [TOKEN_PINS]),
    ("split_three_structured", "if (taken < 2) {", "if (taken < 3) {", [SPLIT_PINS]),
    ("split_groups_of_two", "for (int k = g; k < g + 4 && k < K; k++) {",
     "for (int k = g; k < g + 4 && k < K; k++) { if (k == g + 2) taken = 0;", [SPLIT_PINS]),
    ("topk_keeps_one_more", "for (int i = 0; i < k; i++) act_bits",
     "for (int i = 0; i < k + (k < K); i++) act_bits", [SELECT_PINS]),
    ("topk_nonfinite_lowest", "cols[c].score = finite ? s : INFINITY;",
     "cols[c].score = finite ? s : -1.0;", [SELECT_PINS]),
    ("tileptr_shifted", "put_u32(buf + g.off_tileptr + 4 * t, (uint32_t)unit);",
     "put_u32(buf + g.off_tileptr + 4 * t, (uint32_t)(unit + (t > 0)));", [FORMAT_PINS]),
    ("spmm_rows_ignored",
     "int m = rows ? rows[i] : i;\n        if (m < 0 || m >= M) return ORC_ERR_ARG;\n"
     "        for (int n = 0; n < N; n++) {\n            double acc = 0.0;\n"
     "            for (int k = 0; k < K; k++)\n",
     "int m = i;\n        if (m < 0 || m >= M) return ORC_ERR_ARG;\n"
     "        for (int n = 0; n < N; n++) {\n            double acc = 0.0;\n"
     "            for (int k = 0; k < K; k++)\n", [PRODUCT_PINS]),
    ("tokens_rows_ignored",
     "int m = rows ? rows[i] : i;\n        if (m < 0 || m >= M) return ORC_ERR_ARG;\n"
     "        for (int n = 0; n < N; n++) {\n            double acc = 0.0;\n"
     "            for (int k = 0; k < K; k++) {\n",
     "int m = i;\n        if (m < 0 || m >= M) return ORC_ERR_ARG;\n"
     "        for (int n = 0; n < N; n++) {\n            double acc = 0.0;\n"
     "            for (int k = 0; k < K; k++) {\n", [TOKEN_PINS]),
    ("split_last_two_structured", "if (taken < 2) {",
     "if (taken < 2 && !(k == g && mask[(size_t)n * ld_mask + k + (k + 1 < K)])) {", [SPLIT_PINS]),
]


def pins_pass(lib: str, group: str) -> bool:
    root = os.path.dirname(TESTS)
    path = os.pathsep.join([root, TESTS, os.environ.get("PYTHONPATH", "")])
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=lib, PYTHONPATH=path)
    proc = subprocess.run([sys.executable, "-c", CHILD[group]], cwd=TESTS, env=env,
                          capture_output=True, timeout=600)
    return proc.returncode == 0


@pytest.mark.parametrize("name,old,new,groups", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_planted_mistake(tmp_path, name, old, new, groups):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                    "-o", str(lib), str(path), "-lm"], check=True)
    assert not all(pins_pass(str(lib), g) for g in groups), \
        f"no pin rejects the planted mistake {name!r}"


def test_unmutated_oracle_passes_the_same_pins():
    lib = oracle.build()
    for group in CHILD:
        assert pins_pass(lib, group), group
