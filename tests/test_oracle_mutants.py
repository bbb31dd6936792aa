"""Planted mistakes in a copy of the oracle must each fail at least one pin.

Each mutant is a single textual edit of oracle/trimul_oracle.c (a dropped term, a
wrong sign, a transposed index, a swapped operand). The edited copy is compiled
into a temporary library and the whole pin battery of oracle_pins.py runs
against it. The real oracle source is never modified.
"""
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "unbiased_variance": ("    var /= (double)C;", "    var /= (double)(C - 1);"),
    "eps_outside_sqrt": ("double rstd = 1.0 / sqrt(var + eps);", "double rstd = 1.0 / (sqrt(var) + eps);"),
    "gamma_beta_swapped": ("yr[c] = (xr[c] - mean) * rstd * g + bb;", "yr[c] = (xr[c] - mean) * rstd * bb + g;"),
    "bias_dropped": ("y[r * c_out + o] = s + (bias ? bias[o] : 0.0);", "y[r * c_out + o] = s;"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(v));"),
    "gate_and_projection_swapped": ("y[t] = m * logistic(g[t]) * y[t];", "y[t] = m * logistic(y[t]) * g[t];"),
    "ab_mask_dropped": ("        double m = mask ? mask[r] : 1.0;\n        for (int64_t o = 0; o < c_out; ++o) {",
                        "        double m = 1.0;\n        for (int64_t o = 0; o < c_out; ++o) {"),
    "output_mask_dropped": ("out[t] = m * logistic(g[t]) * out[t];", "out[t] = logistic(g[t]) * out[t];"),
    "outgoing_b_transposed": ("xij[c] += ai[k * C + c] * bj[k * C + c];",
                              "xij[c] += ai[k * C + c] * bm[bb * plane + k * row + j * C + c];"),
    "incoming_a_transposed": ("const double *aki = a + bb * plane + k * row + i * C;",
                              "const double *aki = a + bb * plane + i * row + k * C;"),
    "outgoing_last_k_skipped": ("for (int64_t k = 0; k < N; ++k)\n                        for (int64_t c = 0; c < C; ++c) xij[c]",
                                "for (int64_t k = 0; k < N - 1; ++k)\n                        for (int64_t c = 0; c < C; ++c) xij[c]"),
    "output_layernorm_skipped": ("oracle_linear(rows, c_h, c_z, xn, Wo, bo, out);",
                                 "oracle_linear(rows, c_h, c_z, x, Wo, bo, out);"),
    "gate_reads_raw_z": ("rc = oracle_output_gate(P, c_z, c_h, zhat, x, mask,",
                         "rc = oracle_output_gate(P, c_z, c_h, z, x, mask,"),
    "a_uses_b_weights": ("oracle_gated_projection(P, c_z, c_h, zhat, mask, w->w_ag, w->b_ag, w->w_ap, w->b_ap, a);",
                         "oracle_gated_projection(P, c_z, c_h, zhat, mask, w->w_bg, w->b_bg, w->w_bp, w->b_bp, a);"),
    "sampled_gather_transposed": ("int64_t pr = direction == ORACLE_OUTGOING ? S[p] * N + k : k * N + S[p];",
                                  "int64_t pr = direction == ORACLE_OUTGOING ? k * N + S[p] : S[p] * N + k;"),
    "sampled_output_pair_transposed": ("int64_t pr = I[p] * N + J[q];", "int64_t pr = J[q] * N + I[p];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site for {name} must match exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load_library(oracle.compile_library(str(path), str(tmp_path / "libmutant.so"), force=True))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
