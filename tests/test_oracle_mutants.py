"""Plant plausible mistakes in a copy of the oracle and check that the pins catch
each one (the pins have teeth).  Everything here runs on the CPU; the real
oracle source is read, never modified."""
import os

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "fa_oracle.c")

# (name, text in fa_oracle.c, replacement)
MUTANTS = [
    ("dropped_scale", "srow[j] = scale * dot;", "srow[j] = dot;"),
    ("diagonal_masked", "if (causal && j > i) {", "if (causal && j >= i) {"),
    ("mask_off", "if (causal && j > i) {", "if (0 && causal && j > i) {"),
    ("lse_without_max", "lse_out[r] = m + log(l);", "lse_out[r] = log(l);"),
    ("lse_log2", "lse_out[r] = m + log(l);", "lse_out[r] = m + log2(l);"),
    ("exp_sign_flipped", "srow[j] = exp(srow[j] - m);", "srow[j] = exp(m - srow[j]);"),
    ("not_normalised", "for (int64_t j = 0; j < n; ++j) srow[j] /= l;", ""),
    ("v_row_from_query", "const float* vj = v + j * d;", "const float* vj = v + q_rows[r] * d;"),
    ("k_row_from_query", "const float* kj = k + j * d;", "const float* kj = k + i * d;"),
    ("diagonal_term_dropped", "const int64_t j_end = causal ? q_rows[r] + 1 : n;",
     "const int64_t j_end = causal ? q_rows[r] : n;"),
    ("q_transposed", "dot += (double)qi[t] * (double)kj[t];",
     "dot += (double)q[t * n + i % n] * (double)kj[t];"),
    ("fp32_dot", "double dot = 0.0;", "float dot = 0.0f;"),
    ("max_from_first_key_only", "if (srow[j] > m) m = srow[j];", "if (j == 0) m = srow[j];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_src = tmp_path / "fa_oracle_mutant.c"
    mutant_src.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(str(mutant_src), out=str(tmp_path / "libmutant.so")))
    failures = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, FloatingPointError):
            failures.append(pin.__name__)
    assert failures, f"mutant {name} passed every pin"
