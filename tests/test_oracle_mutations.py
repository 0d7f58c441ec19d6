"""The pins must reject plausible mistakes in the oracle.

Each case copies oracle.c, plants one mistake (a transposed operand, the wrong
slice, a reversed tie rule, a dropped term ...), builds the copy on the CPU and
runs the pins against it: at least one pin must fail. The real oracle is left
untouched."""
import os
import subprocess

import pytest

import oracle
from oracle import build as oracle_build
from tests import test_oracle_pins as pins

MUTATIONS = {
    "rotation transposed": ("acc += x[i * d + a] * P[(int64_t)a * d + c];",
                            "acc += x[i * d + a] * P[(int64_t)c * d + a];"),
    "trailing dims scored": ("for (int c = 0; c < r; ++c)\n                sj += qhat[j * d + c] * kt[c];",
                             "for (int c = d - r; c < d; ++c)\n                sj += qhat[j * d + c] * kt[c];"),
    "ties to the higher index": ("return (a->t > b->t) - (a->t < b->t);",
                                 "return (a->t < b->t) - (a->t > b->t);"),
    "scale dropped": ("z[i] = s * scale;", "z[i] = s;"),
    "softmax sign": ("z[i] = exp(z[i] - zmax);", "z[i] = exp(zmax - z[i]);"),
    "recent window shifted": ("T[keff + i] = ncand + i;", "T[keff + i] = ncand + i - 1;"),
    "group: last head only": ("* kt[c];\n            if (group_max)\n                s = sj > s ? sj : s;\n"
                              "            else\n                s += sj;",
                              "* kt[c];\n            if (group_max)\n                s = sj > s ? sj : s;\n"
                              "            else\n                s = sj;"),
    "bf16 truncates": ("nearbyint(ldexp(v, -spacing_exp))", "trunc(ldexp(v, -spacing_exp))"),
    "dense unnormalised": ("acc += z[t] / denom * V[(int64_t)t * d + c];",
                           "acc += z[t] * V[(int64_t)t * d + c];"),
    "window not excluded": ("int ncand = L - w_eff;\n\n    /* Step 3: approximate scores from the leading",
                            "int ncand = L - w_eff + (w_eff > 0);\n\n    /* Step 3: approximate scores from the leading"),
    "k off by one": ("int keff = k < ncand ? k : ncand;", "int keff = k < ncand ? k - (k > 1) : ncand;"),
    "slab energy not squared": ("e[s] += u * u;", "e[s] += fabs(u);"),
    "slab energy of the first head only": ("for (int j = 0; j < g; ++j)\n                    e[s] +=",
                                           "for (int j = 0; j < 1; ++j)\n                    e[s] +="),
    "slabs: lightest kept": ("if (e[o] > e[s] || (e[o] == e[s] && o < s))",
                             "if (e[o] < e[s] || (e[o] == e[s] && o < s))"),
    "slab ties to the higher index": ("if (e[o] > e[s] || (e[o] == e[s] && o < s))",
                                      "if (e[o] > e[s] || (e[o] == e[s] && o > s))"),
    "slab off by one dim": ("for (int c = 16 * s; c < 16 * s + 16; ++c) {",
                            "for (int c = 16 * s + 1; c < 16 * s + 16; ++c) {"),
    "dims: lightest kept": ("if (w[o] > w[c] || (w[o] == w[c] && o < c))",
                            "if (w[o] < w[c] || (w[o] == w[c] && o < c))"),
    "dim ties to the higher index": ("if (w[o] > w[c] || (w[o] == w[c] && o < c))",
                                     "if (w[o] > w[c] || (w[o] == w[c] && o > c))"),
    "dim magnitude signed": ("w[c] = fabs(acc);", "w[c] = acc;"),
    "dim magnitude of the first head only": ("for (int j = 0; j < g; ++j)\n                acc += qhat[j * d + c];",
                                             "for (int j = 0; j < 1; ++j)\n                acc += qhat[j * d + c];"),
    "dims decode scores the leading dims": ("sj += qhat[j * d + dims[i]] * kt[dims[i]];",
                                            "sj += qhat[j * d + i] * kt[i];"),
    "dims decode drops the last chosen dim": ("for (int i = 0; i < r; ++i)\n                sj += qhat",
                                              "for (int i = 0; i < r - 1; ++i)\n                sj += qhat"),
    "asym query factor is P": ("acc += q[j * d + a] * Aq[(int64_t)a * ri + c];",
                               "acc += q[j * d + a] * P[(int64_t)a * d + c];"),
    "asym index not rounded": ("out[i * ri + c] = dtype == 1 ? oracle_round_bf16(acc) : (double)(float)acc;",
                               "out[i * ri + c] = acc;"),
    "asym group: last head only": ("* x[c];\n            if (group_max)\n                s = sj > s ? sj : s;\n"
                                   "            else\n                s += sj;",
                                   "* x[c];\n            if (group_max)\n                s = sj > s ? sj : s;\n"
                                   "            else\n                s = sj;"),
}

PIN_FUNCS = [
    pins.test_round_bf16_matches_torch_on_binary32_values,
    pins.test_round_bf16_hand_cases,
    pins.test_append_with_identity_and_signed_permutation,
    pins.test_rotation_invariance_of_full_rank_scores,
    pins.test_rotation_transposed_would_fail,
    pins.test_dense_is_rotation_invariant,
    pins.test_dense_matches_textbook_softmax,
    pins.test_leading_dims_are_the_first_r_columns,
    pins.test_group_sum_and_max_readings,
    pins.test_k1_returns_the_argmax_row_exactly,
    pins.test_equal_scores_keep_the_lowest_indices,
    pins.test_zero_keys_average_the_kept_values,
    pins.test_one_hot_values_expose_the_softmax_weights,
    pins.test_recent_window_only,
    pins.test_head_permutation_within_group,
    pins.test_magnitude_slabs_known_answer,
    pins.test_magnitude_slabs_follow_the_basis,
    pins.test_magnitude_slabs_energy_is_conserved,
    pins.test_magnitude_slabs_maximise_the_kept_energy,
    pins.test_magnitude_slabs_reduce_and_ties,
    pins.test_magnitude_dims_known_answer,
    pins.test_magnitude_dims_follow_the_basis,
    pins.test_magnitude_dims_energy_is_conserved,
    pins.test_magnitude_dims_maximise_the_kept_energy,
    pins.test_magnitude_dims_reduce_and_ties,
    pins.test_dims_decode_scores_are_exact_on_the_query_support,
    pins.test_dims_decode_reduces_to_leading_and_to_slabs,
    pins.test_index_keys_with_pca_factor_is_the_appended_slice,
    pins.test_asym_decode_with_symmetric_factors_is_the_leading_decode,
    pins.test_asym_decode_brute_force,
] + [lambda t=t: pins.test_topk_brute_force(t) for t in range(20)] + [
    lambda n=n: pins.test_golden_fixture(n)
    for n in sorted(x for x in os.listdir(pins.GOLDEN) if x.endswith(".json"))
]


def build_mutant(tmp_path, old, new):
    src = open(oracle_build.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique or missing: {old!r}"
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                    str(path), "-o", str(lib), "-lm"], check=True)
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_mutant(name, tmp_path):
    old, new = MUTATIONS[name]
    lib = build_mutant(tmp_path, old, new)
    failures = 0
    oracle.use_library(lib)
    try:
        for fn in PIN_FUNCS:
            try:
                fn()
            except (AssertionError, ValueError):
                failures += 1
    finally:
        oracle.use_library(None)
    assert failures > 0, f"no pin caught the planted mistake: {name}"
