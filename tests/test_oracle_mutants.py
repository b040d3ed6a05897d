"""Plant plausible mistakes in copies of the oracle (CPU only) and check that
each one fails at least one pin. This is what shows the pins are tight enough
to trust the oracle: a dropped term, a wrong sign or index, a transposed
operand or a misplaced update must not slip through."""
import pytest

import oracle
from tests import oracle_pins

# (name, exact source fragment, replacement)
MUTANTS = [
    ("no_sqrt_d_scale", "score[j] = acc * inv_sqrt_d;", "score[j] = acc;"),
    ("diagonal_masked", "for (int64_t j = 0; j <= i; ++j) {\n          double acc",
     "for (int64_t j = 0; j < i + (i == 0); ++j) {\n          double acc"),
    ("elu_without_plus_one", "return x > 0.0 ? x + 1.0 : std::exp(x);", "return x > 0.0 ? x : std::exp(x);"),
    ("retrieval_uses_M_transposed", "num[j] += sq[c] * M[c * d + j];", "num[j] += sq[c] * M[j * d + c];"),
    ("z_counts_tokens", "z[c] += sk;", "z[c] += 1.0;"),
    ("gate_swapped", "out_seg[i * d + j] = g * amem + (1.0 - g) * adot[j];",
     "out_seg[i * d + j] = (1.0 - g) * amem + g * adot[j];"),
    ("denominator_without_sigma", "den += sq[c] * z[c];", "den += qrow[c] * z[c];"),
    ("zero_denominator_falls_back_to_local", "(den == 0.0) ? 0.0 : num[j] / den",
     "(den == 0.0) ? adot[j] : num[j] / den"),
    ("update_uses_wrong_value_index",
     "M[c * d + j] += sk * vseg[i * d + j];",
     "M[c * d + j] += sk * vseg[i * d + c];"),
    ("incoming_state_ignored", "if (P.M_in) {", "if (false) {"),
    ("softmax_not_normalised", "adot[c] /= den_soft;", "adot[c] /= 1.0;"),
    ("gate_sign_flipped", "return 1.0 / (1.0 + std::exp(-b));", "return 1.0 / (1.0 + std::exp(b));"),
    ("sigma_on_value_in_update",
     "M[c * d + j] += sk * vseg[i * d + j];",
     "M[c * d + j] += sk * sigma(vseg[i * d + j]);"),
    ("current_segment_visible_to_retrieval",
     "    if (slot[s] >= 0) {\n      double* out_seg",
     "    for (int64_t i = 0; i < N && s > 0; ++i) {\n"
     "      for (int64_t c = 0; c < d; ++c) {\n"
     "        const double sk = sigma(kseg[i * d + c]);\n"
     "        z[c] += sk;\n"
     "        for (int64_t j = 0; j < d; ++j) M[c * d + j] += sk * vseg[i * d + j];\n"
     "      }\n    }\n"
     "    if (slot[s] >= 0) {\n      double* out_seg"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) >= 1, "mutation anchor not found: " + name
    fwd = oracle.compile_variant(src.replace(old, new, 1), str(tmp_path))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(fwd)
        except Exception:  # an assertion, or a NaN/shape error the mutant causes
            failed.append(pin.__name__)
    assert failed, "no pin caught the planted mistake " + name
