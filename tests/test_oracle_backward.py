"""The oracle's backward against finite differences of its forward, and
planted mistakes in copies of the backward code that the pins must catch (CPU
only)."""
import pytest

import oracle
from tests import oracle_backward_pins as bp


@pytest.mark.parametrize("pin", bp.ALL_BACKWARD_PINS, ids=[p.__name__ for p in bp.ALL_BACKWARD_PINS])
def test_backward_pin(pin):
    fwd = lambda *a, **kw: oracle.forward(*a, **kw)  # noqa: E731
    fwd.backward = oracle.backward
    pin(fwd)


# (name, exact source fragment inside the backward, replacement)
BACKWARD_MUTANTS = [
    ("dq_without_sigma_derivative", "P.dq[(row0 + t) * d + c] += dsq * dsigma(qrow[c]);",
     "P.dq[(row0 + t) * d + c] += dsq;"),
    ("denominator_gradient_sign", "for (int64_t j = 0; j < d; ++j) dden -= dAm[j] * amem[j];",
     "for (int64_t j = 0; j < d; ++j) dden += dAm[j] * amem[j];"),
    ("keys_see_own_segment_queries",
     "  for (int64_t s = S - 1; s >= 0; --s) {\n    // Keys and values of segment s enter M_s.",
     "  for (int64_t s = S - 1; s >= 0; --s) {\n"
     "    for (int64_t e = 0; e < d * d; ++e) G[e] += dMprev[s * d * d + e];\n"
     "    // Keys and values of segment s enter M_s."),
    ("output_state_gradient_dropped", "  if (P.dM_out) {\n    for (int64_t i = 0; i < d * d; ++i) G[i]",
     "  if (false) {\n    for (int64_t i = 0; i < d * d; ++i) G[i]"),
    ("local_branch_not_gated", "dA[c] = (1.0 - g) * go[c];", "dA[c] = go[c];"),
    ("softmax_backward_without_row_term", "const double ds = p[j] * (dp[j] - pdp);",
     "const double ds = p[j] * dp[j];"),
    ("beta_gradient_without_sigmoid_derivative", "dbeta += g * (1.0 - g) * go[c] * (amem[c] - adot[c]);",
     "dbeta += g * go[c] * (amem[c] - adot[c]);"),
    ("key_gradient_misses_z", "        double dsk = Gz[c];", "        double dsk = 0.0;"),
]


@pytest.mark.parametrize("name,old,new", BACKWARD_MUTANTS, ids=[m[0] for m in BACKWARD_MUTANTS])
def test_planted_backward_mistake_is_caught(name, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) == 1, "mutation anchor not unique: " + name
    fwd = oracle.compile_variant(src.replace(old, new), str(tmp_path))
    failed = []
    for pin in bp.ALL_BACKWARD_PINS:
        try:
            pin(fwd)
        except Exception:
            failed.append(pin.__name__)
    assert failed, "no backward pin caught the planted mistake " + name
