"""The pins must be strong enough to catch plausible mistakes in the oracle.

Each mutant below is a copy of the oracle source with one slip planted in it (on the CPU,
compiled with gcc into a temporary library).  The test swaps the mutant in and runs the pin
suite; at least one pin must fail for every mutant.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = {
    # output read from the state before the token's update
    "o_uses_previous_state": (
        "        e[j] = v[j] - p;\n        for (int i = 0; i < K; ++i) row[i] = row[i] * a[i] + w * e[j] * k[i];\n        double s = 0.0;\n        for (int i = 0; i < K; ++i) s += row[i] * q[i];\n        o[j] = s;",
        "        e[j] = v[j] - p;\n        double s = 0.0;\n        for (int i = 0; i < K; ++i) s += row[i] * q[i];\n        o[j] = s;\n        for (int i = 0; i < K; ++i) row[i] = row[i] * a[i] + w * e[j] * k[i];"),
    # prediction made from the undecayed state
    "prediction_without_retention": ("p += row[i] * a[i] * k[i];", "p += row[i] * k[i];"),
    # wrong sign of the delta correction
    "correction_sign": ("row[i] = row[i] * a[i] + w * e[j] * k[i];", "row[i] = row[i] * a[i] - w * e[j] * k[i];"),
    # decay gate with the wrong sign of its logit
    "decay_logit_sign": ("g[i] = exp(-amp * softplus(gl[ix] + decay_bias(d, tau, h, i)));",
                         "g[i] = exp(-amp * softplus(-(gl[ix] + decay_bias(d, tau, h, i))));"),
    # decay amplitude e^{-A_dec} instead of e^{A_dec}
    "decay_amp_sign": ("return A_dec ? exp(A_dec[h]) : 1.0;", "return A_dec ? exp(-A_dec[h]) : 1.0;"),
    # decay bias added outside the softplus
    "decay_bias_outside_softplus": ("g[i] = exp(-amp * softplus(gl[ix] + decay_bias(d, tau, h, i)));",
                                    "g[i] = exp(-amp * softplus(gl[ix]) - decay_bias(d, tau, h, i));"),
    # decay bias of head 0 used for every head
    "decay_bias_wrong_head": ("return tau ? tau[(size_t)h * d->K + i] : 0.0;", "return tau ? tau[i] : 0.0;"),
    # erase gate ignoring the content signal
    "erase_without_content": ("sigm(bx[ix] + delta[i]);", "sigm(bx[ix]);"),
    # chunk mean over L instead of the chunk's actual length
    "mean_over_L": ("for (int i = 0; i < K; ++i) qbar[i] /= n;\n                    for (int j = 0; j < V; ++j) {",
                    "for (int i = 0; i < K; ++i) qbar[i] /= L;\n                    for (int j = 0; j < V; ++j) {"),
    # low-rank factor read transposed
    "A_transposed": ("s += A[((size_t)h * K + i) * R + j] * z[j];", "s += A[((size_t)j * K + i) % ((size_t)d->H * K * R)] * z[j];"),
    # alternative readout: running sum of the previous chunk's outputs instead of their mean
    "alt_sum_not_mean": ("mprev[j] = osum[j] / n;", "mprev[j] = osum[j];"),
    # harness guard: a change that does not alter any result
    "noop_guard": ("static double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }",
                   "static double sigm(double x) { return 1.0 / (exp(-x) + 1.0); }"),
    # backward: decay-gate gradient with the wrong sign
    "bwd_dgl_sign": ("dglt[i] = -da * a[i] * amp * sigm(x);", "dglt[i] = da * a[i] * amp * sigm(x);"),
    # backward: decay-logit gradient without the amplitude
    "bwd_dgl_missing_amp": ("dglt[i] = -da * a[i] * amp * sigm(x);", "dglt[i] = -da * a[i] * sigm(x);"),
    # backward: amplitude gradient without the amplitude factor of log g
    "bwd_dA_dec_missing_amp": ("if (A_dec) dAdec_u[u] += da * a[i] * (-amp * softplus(x));",
                               "if (A_dec) dAdec_u[u] += da * a[i] * (-softplus(x));"),
    # backward: readout path into dq dropped
    "bwd_no_readout_dq": ("for (int i = 0; i < K; ++i) dq[IX_TK(d, bb, toff + t, h, i, K)] += tmp[i];", "(void)tmp;"),
    # backward: write-gate gradient without the sigmoid derivative
    "bwd_dwl_no_sigmoid_prime": ("= dw * w * (1.0 - w);", "= dw;"),
    # backward: prediction term of dk dropped
    "bwd_dk_missing_prediction": ("dkt[i] -= p * de[j];", "(void)p;"),
    # write gate's content term ignored in the forward
    "write_bias_ignored": ("return sigm(wl[((size_t)b * d->T + t) * d->H + h] + dwc);",
                           "return sigm(wl[((size_t)b * d->T + t) * d->H + h]);"),
    # write gate's content term built from the wrong component of z
    "write_bias_wrong_z": ("s += Aw[(size_t)h * d->R + j] * z[j];", "s += Aw[(size_t)h * d->R + j] * z[0];"),
    # packed sequences: a sequence's gate logits read from the first rows of the packed tensor
    "varlen_gate_rows": ("double w = gates(d, bb, toff + t, h, gl, bx, wl, A_dec, tau, delta, dwc, a, g, bg);",
                         "double w = gates(d, bb, t, h, gl, bx, wl, A_dec, tau, delta, dwc, a, g, bg);"),
    # packed sequences: the chunk-mean of q read from the first rows of the packed tensor
    "varlen_qbar_rows": ("qbar[i] += q[IX_TK(d, bb, toff + t, h, i, K)];", "qbar[i] += q[IX_TK(d, bb, t, h, i, K)];"),
    # backward: the write bias's gradient not fed back into dz
    "bwd_write_bias_not_in_dz": ("if (Aw) s += Aw[(size_t)h * R + j] * ddw;", "(void)ddw;"),
}

# the mutant that changes nothing observable must survive: it guards the harness itself
NOOP = {"noop_guard"}

PIN_TESTS = [
    lambda: pins.test_transition_matrix_form(0),
    lambda: pins.test_transition_matrix_form(1),
    pins.test_retention_one_is_plain_delta_rule,
    pins.test_write_zero_is_pure_decay,
    pins.test_exact_write_with_unit_keys,
    pins.test_decay_amplitude_and_bias_closed_form,
    pins.test_orthogonal_keys_give_linear_attention,
    lambda: pins.test_content_signal_closed_form(0, False),
    lambda: pins.test_content_signal_closed_form(1, False),
    lambda: pins.test_content_signal_closed_form(0, True),
    lambda: pins.test_content_signal_closed_form(1, True),
    pins.test_state_norm_bound_every_token,
    lambda: pins.test_packed_sequences_equal_separate_calls(0),
    lambda: pins.test_gradients_central_differences(0),
    lambda: pins.test_gradients_central_differences(1),
]


def _compile(src: str, out: str):
    with open(out + ".c", "w") as f:
        f.write(src)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC", "-o", out,
                    out + ".c", "-lm"], check=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "carve_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "mut.so")
        _compile(src.replace(old, new), path)
        saved = oracle._load()
        oracle._lib = oracle.bind(path)
        failures = 0
        try:
            for t in PIN_TESTS:
                try:
                    t()
                except AssertionError:
                    failures += 1
        finally:
            oracle._lib = saved
    if name in NOOP:
        assert failures == 0, "a no-op change must not fail any pin"
    else:
        assert failures > 0, f"mutant {name} survived every pin"
