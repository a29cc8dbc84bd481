"""Plant plausible mistakes in copies of the oracle and check the pins catch each.

Each mutant is the oracle's C source with one edit (a dropped scale, a wrong
sign, a transposed or reversed operand, a dropped term, a wrong bit layout,
in the forward, the transpose product and the BQQ weight),
compiled into a temporary library on the CPU.  The pins of
test_oracle_pins.py are then run against the mutant; at least one must fail.
This shows the pins are strong enough to trust the unmutated oracle.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_bqq as bqq
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "dbf_oracle.c")

MUTANTS = {
    "drop_b": ("ubuf[j] = xt[j] * b[j];", "ubuf[j] = xt[j];"),
    "drop_mid": ("vbuf[l] = mid[l] * acc;", "vbuf[l] = acc;"),
    "drop_a": ("y[tok * n + i] = a[i] * acc;", "y[tok * n + i] = acc;"),
    "wrong_sign_B": ("acc += (double)Bl[j] * ubuf[j];", "acc -= (double)Bl[j] * ubuf[j];"),
    "transposed_A": ("acc += (double)Ai[l] * vbuf[l];", "acc += (double)A[l * n + i] * vbuf[l];"),
    "reversed_B": ("acc += (double)Bl[j] * ubuf[j];", "acc += (double)Bl[m_in - 1 - j] * ubuf[j];"),
    "dropped_last_term": ("for (int64_t l = 0; l < k; ++l) acc += (double)Ai[l]",
                          "for (int64_t l = 0; l + 1 < k; ++l) acc += (double)Ai[l]"),
    "mid_indexed_by_row": ("vbuf[l] = mid[l] * acc;", "vbuf[l] = mid[l % (k > 1 ? k - 1 : 1)] * acc;"),
    "natural_bit_layout": ("static int bit_of_column(int64_t c) { return (int)((c % 256) / 16) + 16 * (int)(c % 2); }",
                           "static int bit_of_column(int64_t c) { return (int)(c % 32); }"),
    "words_per_32_columns": ("static int64_t word_of_column(int64_t c) { return (c / 256) * 8 + (c % 16) / 2; }",
                             "static int64_t word_of_column(int64_t c) { return c / 32; }"),
    "dense_drops_b": ("Wi[j] += left * ((double)Bl[j] * b[j]);", "Wi[j] += left * ((double)Bl[j]);"),
    "dense_transposed_B": ("Wi[j] += left * ((double)Bl[j] * b[j]);",
                           "Wi[j] += left * ((double)B[(j % k) * m_in + (l % m_in)] * b[j]);"),
    "transposed_drops_b": ("dx[tok * m_in + j] = b[j] * acc;", "dx[tok * m_in + j] = acc;"),
    "transposed_scales_swapped": ("for (int64_t i = 0; i < n; ++i) gbuf[i] = a[i] * dyt[i];",
                                  "for (int64_t i = 0; i < n; ++i) gbuf[i] = a[(i + 1) % n] * dyt[i];"),
    "transposed_reads_A_as_k_by_n": ("acc += (double)A[i * k + l] * gbuf[i];",
                                     "acc += (double)A[l * n + i] * gbuf[i];"),
    "transposed_B_not_transposed": ("acc += (double)B[l * m_in + j] * vbuf[l];",
                                    "acc += (double)B[(j % k) * m_in + (l % m_in)] * vbuf[l];"),
    "scale_bits_drop_mid": ("return 16.0 * (double)(n + k + m_in) / ((double)n * (double)m_in);",
                            "return 16.0 * (double)(n + m_in) / ((double)n * (double)m_in);"),
    "bqq_drops_s_term": ("        w += s[i] * y_row;\n", "        w += 0.0 * y_row;\n"),
    "bqq_t_on_rows_of_Y": ("        w += t[i] * z_col;\n", "        w += t[i] * y_row;\n"),
    "bqq_Z_transposed": ("          yz += (double)Yi[a * k + l] * (double)Zi[l * m + c];",
                         "          yz += (double)Yi[a * k + l] * (double)Zi[(c % k) * m + (l % m)];"),
    "bqq_u_dropped": ("      double w = u;", "      double w = 0.0;"),
    "bqq_last_term_dropped": ("      for (int64_t i = 0; i < p; ++i) {\n        const int8_t* Yi",
                              "      for (int64_t i = 0; i + 1 < p; ++i) {\n        const int8_t* Yi"),
    "bpw_off": ("return (double)k * (double)(n + m_in) / ((double)n * (double)m_in);",
                "return (double)k * (double)(n + m_in) / ((double)n * (double)(m_in + 1));"),
}

PIN_CHECKS = [
    lambda o: pins.test_hand_worked_example(o),
    lambda o: pins.test_exhaustive_2x2x2(o),
    lambda o: pins.test_brute_force_fractions(o, 3, 2, 5),
    lambda o: pins.test_staged_equals_dense(o, 96, 64, 320, 2),
    lambda o: pins.test_integer_mode_is_exact(o),
    lambda o: pins.test_hadamard_closed_form(o, 3),
    lambda o: pins.test_k1_outer_product(o),
    lambda o: pins.test_orientation_is_not_transposed(o),
    lambda o: pins.test_bits_per_weight_closed_form(o, 4096, 2048, 4096, 1.0),
    lambda o: pins.test_scale_bits_per_weight_counts_stored_vectors(o, 1024, 832, 4096),
    lambda o: pins.test_layout_table(o),
    lambda o: pins.test_layout_round_trip_and_padding(o, 3, 128),
    lambda o: pins.test_layout_hand_words(o),
    lambda o: pins.test_transposed_adjoint_identity(o, 48, 64, 80, 3),
    lambda o: pins.test_transposed_equals_dense(o, 33, 64, 65, 3),
    lambda o: pins.test_transposed_hadamard_closed_form(o, 3),
    lambda o: pins.test_transposed_integer_exact(o),
    lambda o: pins.test_transposed_uses_each_scale_once(o),
    lambda o: bqq.test_bqq_hand_worked_example(o),
    lambda o: bqq.test_bqq_product_term_is_integer_matmul(o, 16, 8, 33),
    lambda o: bqq.test_bqq_all_ones_closed_form(o),
    lambda o: bqq.test_bqq_reduces_to_dbf_weight(o, 3, 33, 24, 17),
    lambda o: bqq.test_bqq_without_product_terms_has_rank_two(o),
]


def _build_mutant(name, tmpdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found; update the mutant table"
    path_c = os.path.join(tmpdir, f"{name}.c")
    path_so = os.path.join(tmpdir, f"{name}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new, 1))
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", path_so, path_c, "-lm"],
                   check=True)
    return path_so


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    with tempfile.TemporaryDirectory() as tmpdir:
        so = _build_mutant(name, tmpdir)
        prev = oracle.use_library(so)
        caught = []
        try:
            for i, check in enumerate(PIN_CHECKS):
                try:
                    check(oracle)
                except AssertionError:
                    caught.append(i)
        finally:
            oracle.restore_library(prev)
    assert caught, f"no pin caught mutant {name}"


def test_unmutated_oracle_passes_all_checks():
    for check in PIN_CHECKS:
        check(oracle)
