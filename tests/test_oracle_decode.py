"""The oracle's decode step against its pins, and planted mistakes in copies of
the decode code that the pins must catch (CPU only)."""
import pytest

import oracle
from tests import oracle_decode_pins as dp


@pytest.mark.parametrize("pin", dp.ALL_DECODE_PINS, ids=[p.__name__ for p in dp.ALL_DECODE_PINS])
def test_decode_pin(pin):
    fwd = lambda *a, **kw: oracle.forward(*a, **kw)  # noqa: E731
    fwd.decode = oracle.decode_step
    pin(fwd)


# (name, exact source fragment inside the decode step, replacement)
DECODE_MUTANTS = [
    ("fold_skips_last_token", "    for (int64_t i = 0; i < N; ++i)\n      for (int64_t c = 0; c < d; ++c) {\n        const double sk = sigma(kseg[i * d + c]);\n        zh[c] += sk;",
     "    for (int64_t i = 0; i < N - 1; ++i)\n      for (int64_t c = 0; c < d; ++c) {\n        const double sk = sigma(kseg[i * d + c]);\n        zh[c] += sk;"),
    ("current_key_invisible", "  for (int64_t j = 0; j <= pos; ++j) {\n    double acc",
     "  for (int64_t j = 0; j < pos + (pos == 0); ++j) {\n    double acc"),
    ("cache_row_off_by_one", "kseg[j * d + c] = widen(kc, dtype, (bh * N + j) * d + c);",
     "kseg[j * d + c] = widen(kc, dtype, (bh * N + j + 1) * d + c);"),
    ("fold_every_step", "  if (pos == N - 1) {", "  if (true) {"),
    ("fold_before_output", "  // Retrieval from the memory of earlier segments [HF Memory Retrieval].",
     "  if (pos == N - 1) { for (int64_t c = 0; c < d; ++c) zh[c] += 1.0; }\n"
     "  // Retrieval from the memory of earlier segments [HF Memory Retrieval]."),
    ("decode_gate_swapped", "    out[bh * d + j] = g * amem + (1.0 - g) * adot[j];",
     "    out[bh * d + j] = (1.0 - g) * amem + g * adot[j];"),
]


@pytest.mark.parametrize("name,old,new", DECODE_MUTANTS, ids=[m[0] for m in DECODE_MUTANTS])
def test_planted_decode_mistake_is_caught(name, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) == 1, "mutation anchor not unique: " + name
    fwd = oracle.compile_variant(src.replace(old, new), str(tmp_path))
    failed = []
    for pin in dp.ALL_DECODE_PINS:
        try:
            pin(fwd)
        except Exception:
            failed.append(pin.__name__)
    assert failed, "no decode pin caught the planted mistake " + name
