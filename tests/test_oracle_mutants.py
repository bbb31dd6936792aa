"""Planted mistakes in a copy of the oracle must each fail at least one pin.

Each mutant is a single textual edit of oracle/trimul_oracle.c (a dropped term, a
wrong sign, a transposed index, a swapped operand). The edited copy is compiled
into a temporary library and the whole pin battery of oracle_pins.py runs
against it. The steps written in Python (the pair update and the pair transition)
are mutated the same way: the edited function is compiled from its source text and
stands in for the real one while the pins run. The real oracle source is never
modified.
"""
import inspect
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


PY_MUTANTS = {
    "pair_update_second_step_reads_z": ("pair_update", [
        ('out = z_mid + trimul(z_mid, mask, weights_in, "incoming", eps, lib=lib)',
         'out = z_mid + trimul(z, mask, weights_in, "incoming", eps, lib=lib)')]),
    "pair_update_first_residual_dropped": ("pair_update", [
        ('z_mid = z + trimul(z, mask, weights_out, "outgoing", eps, lib=lib)',
         'z_mid = trimul(z, mask, weights_out, "outgoing", eps, lib=lib)')]),
    "pair_update_second_residual_from_z": ("pair_update", [
        ('out = z_mid + trimul(z_mid,', 'out = z + trimul(z_mid,')]),
    "pair_update_directions_swapped": ("pair_update", [
        ('weights_out, "outgoing", eps', 'weights_out, "incoming", eps'),
        ('weights_in, "incoming", eps', 'weights_in, "outgoing", eps')]),
    "pair_update_weights_swapped": ("pair_update", [
        ('mask, weights_out, "outgoing"', 'mask, weights_in, "outgoing"'),
        ('mask, weights_in, "incoming"', 'mask, weights_out, "incoming"')]),
    "transition_relu_dropped": ("pair_transition", [("hid = np.maximum(hid, 0.0)", "hid = hid")]),
    "transition_relu_as_abs": ("pair_transition", [("hid = np.maximum(hid, 0.0)", "hid = np.abs(hid)")]),
    "transition_b1_dropped": ("pair_transition", [("hid = hid + _f64(b1)", "hid = hid")]),
    "transition_b2_dropped": ("pair_transition", [("upd = upd + _f64(b2)", "upd = upd")]),
    "transition_mask_dropped": ("pair_transition", [("upd = upd * _f64(mask)[..., None]", "upd = upd")]),
    "transition_residual_dropped": ("pair_transition", [("return z + upd", "return upd")]),
    "transition_b2_outside_mask": ("pair_transition", [
        ("upd = upd + _f64(b2)", "pass"),
        ("return z + upd", "return z + upd + (_f64(b2) if b2 is not None else 0.0)")]),
}


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_python_mutant_is_caught(name, monkeypatch):
    func, edits = PY_MUTANTS[name]
    src = inspect.getsource(getattr(oracle, func))
    for old, new in edits:
        assert src.count(old) == 1, f"mutation site for {name} must match exactly once: {old}"
        src = src.replace(old, new)
    namespace = dict(vars(oracle))
    exec(compile(src, f"<mutant {name}>", "exec"), namespace)
    monkeypatch.setattr(oracle, func, namespace[func])
    lib = oracle.load_library()
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
