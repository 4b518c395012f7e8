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
    # the decode function
    ("decode_top_left_mask", "const int64_t last = causal ? nk - nq + qi : nk - 1;",
     "const int64_t last = causal ? qi : nk - 1;"),
    ("decode_own_key_masked", "const int64_t last = causal ? nk - nq + qi : nk - 1;",
     "const int64_t last = causal ? nk - nq + qi - 1 : nk - 1;"),
    ("decode_last_key_dropped", "const int64_t last = causal ? nk - nq + qi : nk - 1;",
     "const int64_t last = causal ? nk - nq + qi : nk - 2;"),
    ("decode_scale_dropped", "w[kj] = acc * scale;", "w[kj] = acc;"),
    ("decode_lse_without_max", "lse[h * nq + qi] = mx + log(sum);", "lse[h * nq + qi] = log(sum);"),
    ("decode_not_normalised", "orow[t] = acc / sum;", "orow[t] = acc;"),
    ("decode_v_of_key_0", "acc += w[kj] * (double)vh[kj * d + t];", "acc += w[kj] * (double)vh[t];"),
    ("decode_query_of_head_0", "const float* qrow = q + (h * nq + qi) * d;", "const float* qrow = q + qi * d;"),
    # the backward pass
    ("bwd_dk_scale_dropped", "dkh[c * d + t] = scale * ak;", "dkh[c * d + t] = ak;"),
    ("bwd_dq_scale_dropped", "dqh[r * d + t] = scale * aq;", "dqh[r * d + t] = aq;"),
    ("bwd_no_softmax_jacobian", "gm[r * n + c] = pm[r * n + c] * (gm[r * n + c] - drow);",
     "gm[r * n + c] = pm[r * n + c] * gm[r * n + c];"),
    ("bwd_ds_without_p", "gm[r * n + c] = pm[r * n + c] * (gm[r * n + c] - drow);",
     "gm[r * n + c] = gm[r * n + c] - drow;"),
    ("bwd_dv_from_p_not_transposed", "av += pm[r * n + c] * (double)gh[r * d + t];",
     "av += pm[c * n + r] * (double)gh[r * d + t];"),
    ("bwd_mask_off", "if (causal && c > r) {", "if (0 && causal && c > r) {"),
    ("merge_without_max", "const double w = exp((double)lse_parts[i * rows + r] - big);",
     "const double w = exp((double)lse_parts[i * rows + r]);"),
    ("merge_lse_without_max", "lse[r] = big + log(tot);", "lse[r] = log(tot);"),
    ("merge_not_normalised", "for (int64_t t = 0; t < d; ++t) o[r * d + t] /= tot;", ""),
    # the row-sampled backward
    ("bwd_rows_dq_scale_dropped", "for (int64_t t = 0; t < d; ++t) out[t] *= scale;", ""),
    ("bwd_rows_dk_scale_dropped", "for (int64_t t = 0; t < d; ++t) okk[t] *= scale;", ""),
    ("bwd_rows_max_from_first_key_only", "m = srow[j] > m ? srow[j] : m;", "m = j == 0 ? srow[j] : m;"),
    ("bwd_rows_lse_without_max", "lse[i] = m + log(l);", "lse[i] = log(l);"),
    ("bwd_rows_no_softmax_jacobian", "const double dsij = pij * (dp - dsum[i]);\n                        for (int64_t t = 0; t < d; ++t) out[t]",
     "const double dsij = pij * dp;\n                        for (int64_t t = 0; t < d; ++t) out[t]"),
    ("bwd_rows_key_mask_off", "const int64_t ibeg = causal ? j : 0;", "const int64_t ibeg = 0;"),
    ("bwd_rows_key_diagonal_dropped", "const int64_t ibeg = causal ? j : 0;", "const int64_t ibeg = causal ? j + 1 : 0;"),
    ("bwd_rows_dv_with_q", "okv[t] += pij * (double)gh[i * d + t];", "okv[t] += pij * (double)qh[i * d + t];"),
    ("bwd_rows_d_from_v", "acc += (double)gh[i * d + t] * orow[t];", "acc += (double)gh[i * d + t] * (double)vh[i * d + t];"),
    ("bwd_dp_with_k", "for (int64_t t = 0; t < d; ++t) acc += (double)gh[r * d + t] * (double)vh[c * d + t];",
     "for (int64_t t = 0; t < d; ++t) acc += (double)gh[r * d + t] * (double)kh[c * d + t];"),
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
