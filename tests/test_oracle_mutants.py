"""Plants plausible mistakes in copies of the oracle (on the CPU) and checks
that each one makes at least one pin fail, so the pins really constrain every
step of the oracle: conv, SiLU, softplus, discretisation, recurrence, readout,
skip, gate, carried state, the decode step, the RMSNorm of B and C, the projection product
the Mamba-2 form (scalar decay per head, grouped B/C) and the Mamba-3 form
(trapezoidal rule, rotating complex state, several inputs and outputs)."""

import os

import pytest

import oracle
from pins import ALL_PINS

# (name, exact text in the oracle source, replacement)
MUTANTS = [
    ("drop_skip", "const double yv = acc + (Dskip ? Dskip[d] : 0.0) * u;", "const double yv = acc;"),
    ("gate_by_z", "y[row * D + d] = yv * or_silu(z);", "y[row * D + d] = yv * z;"),
    ("gate_by_x", "y[row * D + d] = yv * or_silu(z);", "y[row * D + d] = yv * or_silu(x);"),
    ("conv_current_tap", "pre += conv_w[d * W + (W - 1)] * x;", "pre += conv_w[d * W + 0] * x;"),
    ("conv_window_tap", "pre += conv_w[d * W + k] * win[k];", "pre += conv_w[d * W + k + 1] * win[k];"),
    ("conv_bias_dropped", "double pre = conv_b ? conv_b[d] : 0.0;\n                for", "double pre = 0.0;\n                for"),
    ("silu_sign", "return v / (1.0 + exp(-v));", "return v / (1.0 + exp(v));"),
    ("softplus_no_log", "log1p(exp(-fabs(v)))", "exp(-fabs(v))"),
    ("dt_bias_dropped", "dt[row * D + d] + (dt_bias ? dt_bias[d] : 0.0)", "dt[row * D + d]"),
    ("A_sign", "const double dA = exp(delta * A[d * N + n]);", "const double dA = exp(-delta * A[d * N + n]);"),
    ("A_transposed", "const double dA = exp(delta * A[d * N + n]);", "const double dA = exp(delta * A[n * D + d]);"),
    ("dA_not_exp", "const double dA = exp(delta * A[d * N + n]);", "const double dA = 1.0 + delta * A[d * N + n];"),
    ("dBx_no_delta", "const double dBx = delta * Bm[row * N + n] * u;", "const double dBx = Bm[row * N + n] * u;"),
    ("dBx_raw_x", "const double dBx = delta * Bm[row * N + n] * u;", "const double dBx = delta * Bm[row * N + n] * x;"),
    ("B_previous_token", "const double dBx = delta * Bm[row * N + n] * u;",
     "const double dBx = delta * Bm[(t > 0 ? row - 1 : row) * N + n] * u;"),
    ("C_as_B", "acc += Cm[row * N + n] * h[n];", "acc += Bm[row * N + n] * h[n];"),
    ("readout_before_update",
     "h[n] = dA * h[n] + dBx;\n                    acc += Cm[row * N + n] * h[n];",
     "acc += Cm[row * N + n] * h[n];\n                    h[n] = dA * h[n] + dBx;"),
    ("h0_ignored", "h[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;", "h[n] = 0.0;"),
    ("conv_state_ignored", "win[j] = conv_state_in ? conv_state_in[(b * D + d) * (W - 1) + j] : 0.0;", "win[j] = 0.0;"),
    ("window_not_appended", "if (W > 1) win[W - 2] = x;", "if (W > 1) win[W - 2] = 0.0;"),
    ("window_order", "for (int64_t j = 0; j + 1 < W - 1; ++j) win[j] = win[j + 1];",
     "for (int64_t j = W - 3; j >= 0; --j) win[j + 1] = win[j];"),
    ("h_last_not_written", "for (int64_t n = 0; n < N; ++n) h_last[(b * D + d) * N + n] = h[n];",
     "for (int64_t n = 0; n < N; ++n) h_last[(b * D + d) * N + n] = 0.0;"),
    ("decode_A_sign", "const double dA = exp(delta * A[ld * N + n]);", "const double dA = exp(-delta * A[ld * N + n]);"),
    ("decode_readout_before_update",
     "h[n] = dA * h[n] + delta * Bm[lb * N + n] * u;\n            acc += Cm[lb * N + n] * h[n];",
     "acc += Cm[lb * N + n] * h[n];\n            h[n] = dA * h[n] + delta * Bm[lb * N + n] * u;"),
    ("decode_window_not_shifted", "for (int64_t k = 0; k + 1 < W - 1; ++k) cs[k] = cs[k + 1];", ""),
    ("decode_params_of_layer0", "const int64_t ld = l * D + d;", "const int64_t ld = d;"),
    ("decode_no_skip", "y[r] = (acc + (Dskip ? Dskip[ld] : 0.0) * u) * or_silu(z[r]);", "y[r] = acc * or_silu(z[r]);"),
    ("rms_no_sqrt", "const double inv = 1.0 / sqrt(ss / (double)n + eps);",
     "const double inv = 1.0 / (ss / (double)n + eps);"),
    ("rms_sum_not_mean", "const double inv = 1.0 / sqrt(ss / (double)n + eps);",
     "const double inv = 1.0 / sqrt(ss + eps);"),
    ("rms_eps_outside", "const double inv = 1.0 / sqrt(ss / (double)n + eps);",
     "const double inv = 1.0 / (sqrt(ss / (double)n) + eps);"),
    ("rms_weight_dropped", "out[r * n + i] = x[r * n + i] * inv * w[i];", "out[r * n + i] = x[r * n + i] * inv;"),
    ("rms_weight_reversed", "out[r * n + i] = x[r * n + i] * inv * w[i];",
     "out[r * n + i] = x[r * n + i] * inv * w[n - 1 - i];"),
    ("rms_abs_not_square", "ss += x[r * n + i] * x[r * n + i];", "ss += fabs(x[r * n + i]);"),
    ("matmul_weight_transposed", "acc += A[m * K + k] * Bw[n * K + k];", "acc += A[m * K + k] * Bw[k * N + n];"),
    ("matmul_last_term_dropped", "for (int64_t k = 0; k < K; ++k) acc += A[m * K + k] * Bw[n * K + k];",
     "for (int64_t k = 0; k + 1 < K; ++k) acc += A[m * K + k] * Bw[n * K + k];"),
    ("matmul_no_accumulate", "acc += A[m * K + k] * Bw[n * K + k];", "acc = A[m * K + k] * Bw[n * K + k];"),
    ("matmul_row_of_A", "acc += A[m * K + k] * Bw[n * K + k];", "acc += A[n * K + k] * Bw[n * K + k];"),
    ("ssd_A_sign", "const double decay = exp(delta * A[h]);", "const double decay = exp(-delta * A[h]);"),
    ("ssd_decay_not_exp", "const double decay = exp(delta * A[h]);", "const double decay = 1.0 + delta * A[h];"),
    ("ssd_no_delta_on_B", "s[n] = decay * s[n] + delta * Bt[n] * xv;", "s[n] = decay * s[n] + Bt[n] * xv;"),
    ("ssd_readout_before_update", "s[n] = decay * s[n] + delta * Bt[n] * xv;\n                    acc += Ct[n] * s[n];",
     "acc += Ct[n] * s[n];\n                    s[n] = decay * s[n] + delta * Bt[n] * xv;"),
    ("ssd_C_as_B", "acc += Ct[n] * s[n];", "acc += Bt[n] * s[n];"),
    ("ssd_group_interleaved", "const int64_t g = h / heads_per_group;", "const int64_t g = h % G;"),
    ("ssd_skip_dropped", "const double yv = acc + (Dskip ? Dskip[h] : 0.0) * xv;\n                y[row * C + c]",
     "const double yv = acc;\n                y[row * C + c]"),
    ("ssd_gate_by_z", "y[row * C + c] = z ? yv * or_silu(z[row * C + c]) : yv;",
     "y[row * C + c] = z ? yv * z[row * C + c] : yv;"),
    ("ssd_dt_bias_of_head0", "or_softplus(dt[row * H + h] + (dt_bias ? dt_bias[h] : 0.0));\n                const double decay",
     "or_softplus(dt[row * H + h] + (dt_bias ? dt_bias[0] : 0.0));\n                const double decay"),
    ("ssd_dt_of_channel", "or_softplus(dt[row * H + h] + (dt_bias ? dt_bias[h] : 0.0));\n                const double decay",
     "or_softplus(dt[row * H + c % H] + (dt_bias ? dt_bias[h] : 0.0));\n                const double decay"),
    ("ssd_h0_ignored", "s[n] = h0 ? h0[(b * C + c) * N + n] : 0.0;", "s[n] = 0.0;"),
    ("ssd_head_of_channel", "const int64_t h = c / P;\n            const int64_t g = h / heads_per_group;",
     "const int64_t h = c % H;\n            const int64_t g = h / heads_per_group;"),
    ("ssd_h_last_not_written", "for (int64_t n = 0; n < N; ++n) h_last[(b * C + c) * N + n] = s[n];",
     "for (int64_t n = 0; n < N; ++n) h_last[(b * C + c) * N + n] = 0.0;"),
    ("m3_lambda_swapped", "const double pr = sr[k] + (1.0 - lam) * delta * ur[k];",
     "const double pr = sr[k] + lam * delta * ur[k];"),
    ("m3_trapezoid_tap_undecayed",
     "sr[k] = ar * pr - ai * pi + lam * delta * vr;",
     "sr[k] = ar * sr[k] - ai * si[k] + (1.0 - lam) * delta * ur[k] + lam * delta * vr;"),
    ("m3_rotation_sign", "const double ar = mag * cos(ang), ai = mag * sin(ang);",
     "const double ar = mag * cos(ang), ai = -mag * sin(ang);"),
    ("m3_rotation_dropped", "const double ar = mag * cos(ang), ai = mag * sin(ang);",
     "const double ar = mag, ai = 0.0 * ang;"),
    ("m3_readout_imag_dropped", "acc += Ct[2 * k] * sr[k] + Ct[2 * k + 1] * si[k];", "acc += Ct[2 * k] * sr[k];"),
    ("m3_pairs_as_halves", "vr += Bt[2 * k] * xv;\n                        vi += Bt[2 * k + 1] * xv;",
     "vr += Bt[k] * xv;\n                        vi += Bt[k + K] * xv;"),
    ("m3_prev_input_not_kept", "                    ur[k] = vr;\n                    ui[k] = vi;\n", ""),
    ("m3_x_prev_ignored", "if (x_prev && B_prev) {", "if (0) {"),
    ("m3_mimo_first_input_only", "for (int64_t r = 0; r < R; ++r) {\n                        const double xv = x[(row * R + r) * C + c];\n                        const double* Bt",
     "for (int64_t r = 0; r < 1; ++r) {\n                        const double xv = x[(row * R + r) * C + c];\n                        const double* Bt"),
    ("m3_readout_with_first_C", "const double* Ct = Cm + ((row * R + r) * G + g) * N;",
     "const double* Ct = Cm + ((row * R + 0) * G + g) * N;"),
    ("m3_trap_default", "const double lam = trap ? trap[row * H + h] : 0.5;", "const double lam = trap ? trap[row * H + h] : 1.0;"),
    ("m3_theta_of_head0", "const double ang = delta * theta[h * K + k];", "const double ang = delta * theta[k];"),
    ("m3_h_last_imag_part", "h_last[(b * C + c) * N + 2 * k + 1] = si[k];", "h_last[(b * C + c) * N + 2 * k + 1] = sr[k];"),
    ("m3_group_interleaved", "const int64_t g = h * G / H;",
     "const int64_t g = h % G;"),
    ("m3_skip_dropped", "const double yv = acc + (Dskip ? Dskip[h] : 0.0) * xv;\n                    const int64_t o",
     "const double yv = acc;\n                    const int64_t o"),
]


def _run_pins(lib):
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = tmp_path / f"mut_{name}.c"
    mutated.write_text(src.replace(old, new))
    so = oracle.compile_source(str(mutated), str(tmp_path / f"libmut_{name}.so"))
    lib = oracle.load_library(so)
    failed = _run_pins(lib)
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_passes_all_pins():
    assert _run_pins(oracle.lib()) == []
