"""Each plausible mistake planted in a copy of the oracle source must fail a pin.

The mutants are built in a temporary directory from textual edits of
oracle/lightning_oracle.c; the real oracle is untouched.
"""
import os

import pytest

import oracle
from tests import oracle_pins as P

# (name, original text, mutated text): each edit hits the first occurrence only.
MUTANTS = [
    ("forward_exponent_off_by_one",
     "double w = pw[i - j] * dot(q + i * d, k + j * d, d);",
     "double w = pw[i - j > 0 ? i - j - 1 : 0] * dot(q + i * d, k + j * d, d);"),
    ("forward_drops_diagonal",
     "for (long j = 0; j <= i; ++j) {\n            double w = pw[i - j]",
     "for (long j = 0; j < i; ++j) {\n            double w = pw[i - j]"),
    ("forward_swaps_query_key_rows",
     "double w = pw[i - j] * dot(q + i * d, k + j * d, d);",
     "double w = pw[i - j] * dot(q + j * d, k + i * d, d);"),
    ("state_transposed",
     "state[a * d + b] += ka * v[j * d + b];",
     "state[b * d + a] += ka * v[j * d + b];"),
    ("state_exponent_off_by_one",
     "double w = pw[N - 1 - j];",
     "double w = pw[N - 1 - j > 0 ? N - 2 - j : 0];"),
    ("recurrence_outer_product_transposed",
     "S[a * d + b] = lam * S[a * d + b] + kt[a] * vt[b];",
     "S[a * d + b] = lam * S[a * d + b] + kt[b] * vt[a];"),
    ("recurrence_drops_decay",
     "S[a * d + b] = lam * S[a * d + b] + kt[a] * vt[b];",
     "S[a * d + b] = S[a * d + b] + kt[a] * vt[b];"),
    ("decode_drops_decay",
     "S[a * d + b] = lam[p] * S[a * d + b] + kp[a] * vp[b];",
     "S[a * d + b] = S[a * d + b] + kp[a] * vp[b];"),
    ("decode_reads_out_with_old_state",
     "        for (long b = 0; b < d; ++b) {\n            double s = 0.0;\n"
     "            for (long a = 0; a < d; ++a) s += qp[a] * S[a * d + b];",
     "        for (long b = 0; b < d; ++b) {\n            double s = 0.0;\n"
     "            for (long a = 0; a < d; ++a) s += qp[a] * (S[a * d + b] - kp[a] * vp[b]);"),
    ("rows_exponent_off_by_one",
     "double w = pow(lam, (double)(i - j)) * dot",
     "double w = pow(lam, (double)(i - j + 1)) * dot"),
    ("backward_dq_wrong_operand",
     "dq[i * d + c] += w * k[j * d + c];",
     "dq[i * d + c] += w * v[j * d + c];"),
    ("backward_dk_wrong_operand",
     "dk[j * d + c] += wk * q[i * d + c];",
     "dk[j * d + c] += wk * k[i * d + c];"),
    ("backward_dv_swapped_rows",
     "double wv = pw[i - j] * dot(q + i * d, k + j * d, d);",
     "double wv = pw[i - j] * dot(q + j * d, k + i * d, d);"),
    ("from_state_exponent_off_by_one",
     "double w = pow(lam, (double)(i + 1));",
     "double w = pow(lam, (double)i);"),
    ("from_state_transposed",
     "s += q[i * d + a] * state_in[a * d + b];",
     "s += q[i * d + a] * state_in[b * d + a];"),
    ("from_state_state_decay_off_by_one",
     "double w = pow(lam, (double)N);",
     "double w = pow(lam, (double)(N > 0 ? N - 1 : 0));"),
    ("from_state_drops_state_term",
     "state[a] += w * state_in[a];",
     "state[a] += 0.0 * state_in[a];"),
    ("recurrence_ignores_state_in",
     "if (state_in) memcpy(S, state_in",
     "if (0) memcpy(S, state_in"),
    ("norm_sum_of_values_not_squares",
     "ss += x * x;",
     "ss += x;"),
    ("norm_mean_over_one_head",
     "double r = 1.0 / sqrt(ss / (double)(H * d) + eps);",
     "double r = 1.0 / sqrt(ss / (double)d + eps);"),
    ("norm_drops_eps",
     "double r = 1.0 / sqrt(ss / (double)(H * d) + eps);",
     "double r = 1.0 / sqrt(ss / (double)(H * d));"),
    ("gate_sign_flipped",
     "double gate = 1.0 / (1.0 + exp(-g[t * H * d + f]));",
     "double gate = 1.0 / (1.0 + exp(g[t * H * d + f]));"),
    ("norm_gate_output_transposed",
     "y[t * H * d + f] = w[f] * x * r * gate;",
     "y[t * H * d + c * H + h] = w[f] * x * r * gate;"),
    ("norm_gate_reads_o_token_major",
     "double x = o[((b * H + h) * N + n) * d + c];\n                double gate",
     "double x = o[t * H * d + f];\n                double gate"),
    ("state_prefix_includes_own_chunk_decay",
     "for (long q = p + 1; q < r; ++q) between += lens[q];",
     "for (long q = p; q < r; ++q) between += lens[q];"),
    ("state_prefix_includes_chunk_r",
     "for (long p = 0; p < r; ++p) {\n            long between",
     "for (long p = 0; p <= r && p < R; ++p) {\n            long between"),
    ("state_prefix_decay_from_the_front",
     "for (long q = p + 1; q < r; ++q) between += lens[q];",
     "for (long q = 0; q < p; ++q) between += lens[q];"),
    ("varlen_zero_length_state_not_cleared",
     "if (st) for (long a = 0; a < d * d; ++a) st[a] = 0.0;\n            continue;",
     "continue;"),
]


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_fails_a_pin(tmp_path, name, orig, mut):
    src = open(oracle.SOURCE).read()
    assert orig in src, f"mutation anchor for {name} not found"
    mutated = src.replace(orig, mut, 1)
    path_c = os.path.join(tmp_path, "mutant.c")
    path_so = os.path.join(tmp_path, "mutant.so")
    with open(path_c, "w") as f:
        f.write(mutated)
    oracle.build(force=True, src=path_c, out=path_so)
    orc = oracle.Oracle(path_so)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
