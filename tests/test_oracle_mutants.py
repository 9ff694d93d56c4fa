"""Each plausible mistake planted in a copy of the oracle's C source must fail a pin.

The copy is compiled into a temporary directory; the oracle as built is untouched.
This shows that the pins constrain every term of the oracle: a dropped term, a
wrong sign, a swapped or shifted index, a transposed operand.
"""
import subprocess

import pytest

import oracle
from oracle import build as oracle_build
from tests import oracle_pins

MUTANTS = {
    "drop_D_skip": ("y += dskip * xv;", "y += 0.0 * dskip * xv;"),
    "wrong_sign_of_A": ("const double abar = exp(delta * a);", "const double abar = exp(-delta * a);"),
    "drop_x_in_input": ("h[n] = abar * h[n] + bbar * xv;", "h[n] = abar * h[n] + bbar;"),
    "readout_uses_B": ("y += widen(J->Cm, J->dtype, bc + n) * h[n];",
                       "y += widen(J->Bm, J->dtype, bc + n) * h[n];"),
    "gate_is_sigmoid": ("y *= zv * sigmoid(zv);", "y *= sigmoid(zv);"),
    "softplus_negative_branch": ("return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v));",
                                 "return v > 0.0 ? v + log1p(exp(-v)) : log(exp(v));"),
    "A_transposed": ("const double a = (double)J->A[d * N + n];",
                     "const double a = (double)J->A[n * Dm + d];"),
    "B_C_lagged_one_token": ("const int64_t bc = (b * L + t) * N;",
                             "const int64_t bc = (b * L + (t > 0 ? t - 1 : 0)) * N;"),
    "dt_bias_ignored": ("const double bias = J->dt_bias ? (double)J->dt_bias[d] : 0.0;",
                        "const double bias = 0.0;"),
    "h0_ignored": ("h[n] = J->h0_f64 ? J->h0_f64[hi] : (J->h0 ? (double)J->h0[hi] : 0.0);",
                   "h[n] = J->h0_f64 ? J->h0_f64[hi] : 0.0;"),
    "readout_before_update": ("h[n] = abar * h[n] + bbar * xv;\n            y += widen(J->Cm, J->dtype, bc + n) * h[n];",
                              "y += widen(J->Cm, J->dtype, bc + n) * h[n];\n            h[n] = abar * h[n] + bbar * xv;"),
    "bf16_widening_shift": ("uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;",
                            "uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 15;"),
    "exact_zoh_sign": ("expm1(delta * a) / a", "expm1(delta * a) / (-a)"),
    "final_state_not_written": ("    if (J->h_last)\n", "    if (0)\n"),
    "batch_time_transposed": ("const int64_t i = (b * L + t) * Dm + d;",
                              "const int64_t i = (t * J->Bsz + b) * Dm + d;"),
    "sigmoid_sign": ("static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }",
                     "static double sigmoid(double v) { return 1.0 / (1.0 + exp(v)); }"),
    "delta_times_A_squared": ("const double abar = exp(delta * a);", "const double abar = exp(delta * a * a);"),
    "conv_taps_reversed": ("J->conv_w[d * ORACLE_CONV_K + k]", "J->conv_w[d * ORACLE_CONV_K + (ORACLE_CONV_K - 1 - k)]"),
    "conv_bias_dropped": ("double v = J->conv_b ? (double)J->conv_b[d] : 0.0;", "double v = 0.0;"),
    "conv_without_silu": ("return v * sigmoid(v);", "return v;"),
    "conv_x0_ignored": ("if (J->conv_x0) return", "if (0) return"),
    "conv_x0_rows_reversed": ("(tau + ORACLE_CONV_K - 1)", "(-1 - tau)"),
    # (the shifted window stays inside x: it moves one token ahead except at the last step)
    "conv_reads_next_token": ("raw_token(J, b, t - (ORACLE_CONV_K - 1) + k, d)",
                              "raw_token(J, b, t - (ORACLE_CONV_K - 1) + k + (t + 1 < J->L), d)"),
    "conv_skip_uses_raw_x": ("y += dskip * xv;", "y += dskip * widen(J->x, J->dtype, i);"),
    "conv_update_uses_raw_x": ("h[n] = abar * h[n] + bbar * xv;", "h[n] = abar * h[n] + bbar * widen(J->x, J->dtype, i);"),
    "bwd_gate_derivative": ("dz[i] = dq * q * sg * (1.0 + zv * (1.0 - sg));", "dz[i] = dq * q * sg;"),
    "bwd_adjoint_decay_first": ("                    g[n] += dq * widen(Cm, dtype, bc + n);\n",
                                "                    g[n] = g[n] * exp(delta[t] * a) + dq * widen(Cm, dtype, bc + n);\n"),
    "bwd_dA_without_abar": ("g[n] * (delta[t] * abar * hp + w_da", "g[n] * (delta[t] * hp + w_da"),
    "bwd_dC_previous_state": ("dC[bc + n] += dq * hs[(t + 1) * N + n];", "dC[bc + n] += dq * hs[t * N + n];"),
    "bwd_ddt_without_sigmoid": ("ddt[i] = softplus_on ? ddel * sigmoid(v) : ddel;", "ddt[i] = ddel;"),
    "bwd_dD_ungated": ("dD[d] += dq * xv;", "dD[d] += widen(dy, dtype, i) * xv;"),
    "bwd_dh_last_ignored": ("g[n] = dh_last ? dh_last[(b * Dm + d) * N + n] : 0.0;", "g[n] = 0.0;"),
    "bwd_ddelta_drops_input_term": ("ddel += g[n] * (a * abar * hp + w_dd * bn * xv);", "ddel += g[n] * (a * abar * hp);"),
    "bwd_zoh_series_coefficient": ("double term = 0.5, sum = 0.0;", "double term = 1.0 / 3.0, sum = 0.0;"),
    "bwd_zoh_closed_form_sign": ("f = (s * exp(s) - expm1(s)) / (s * s);", "f = (s * exp(s) + expm1(s)) / (s * s);"),
    "bwd_zoh_dw_ddelta_one": ("*dw_ddelta = exp(s);", "*dw_ddelta = 1.0;"),
    "bwd_zoh_dB_uses_delta": ("dB[bc + n] += g[n] * w * xv;", "dB[bc + n] += g[n] * delta[t] * xv;"),
    "bwd_zoh_dx_uses_delta": ("dxv += g[n] * w * bn;", "dxv += g[n] * delta[t] * bn;"),
    "bwd_conv_without_silu_derivative": ("dp = dxv * sp * (1.0 + p * (1.0 - sp));", "dp = dxv * sp;"),
    "bwd_conv_taps_reversed": ("const double dtok = dp * (double)conv_w[d * ORACLE_CONV_K + k];",
                               "const double dtok = dp * (double)conv_w[d * ORACLE_CONV_K + (ORACLE_CONV_K - 1 - k)];"),
    "bwd_conv_x0_gradient_dropped": ("(tau + ORACLE_CONV_K - 1)) * Dm + d] += dtok;", "(tau + ORACLE_CONV_K - 1)) * Dm + d] += 0.0 * dtok;"),
    "bwd_conv_bias_gradient_ungated": ("dconv_b[d] += dp;", "dconv_b[d] += dxv;"),
    "bwd_conv_tap_gradient_shifted": ("dconv_w[d * ORACLE_CONV_K + k] += dp * raw_token(&cj, b, tau, d);",
                                      "dconv_w[d * ORACLE_CONV_K + k] += dp * raw_token(&cj, b, tau + (t + 1 < L), d);"),
    "conv_step_ignores_window": ("y, h, h, 0, Bsz * Dm, conv_w, conv_b, conv_state};",
                                 "y, h, h, 0, Bsz * Dm, conv_w, conv_b, NULL};"),
}


def _build_variant(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                           "-o", str(so), str(c), "-lm", "-lpthread"])
    return oracle.Oracle(str(so))


def _failed_pins(orc):
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


def test_unmodified_copy_passes(tmp_path):
    src = open(oracle_build.SRC).read()
    assert _failed_pins(_build_variant(tmp_path, "same", src)) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    src = open(oracle_build.SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation pattern for {name} not found in the oracle source"
    failed = _failed_pins(_build_variant(tmp_path, name, src.replace(old, new)))
    assert failed, f"mutant {name} passed every pin"
