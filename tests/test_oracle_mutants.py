"""Plant plausible mistakes in a copy of the oracle source and check that the
pins catch every one of them (CPU only; the planted copies live in a
temporary directory and are never used by anything else)."""
import os

import pytest

import oracle
from tests import oracle_pins

# (name, text in one of the oracle sources, replacement)
MUTANTS = [
    ("drop_skip_term", "acc += (double)D[d] * x;\n        if (z)\n            acc *= silu(load_value(z, dtype, i));\n        y[t] = acc;",
     "acc += 0.0 * x;\n        if (z)\n            acc *= silu(load_value(z, dtype, i));\n        y[t] = acc;"),
    ("sign_of_exponent", "exp(dt * a) * h[n]", "exp(-dt * a) * h[n]"),
    ("zoh_input_matrix", "const double Bbar = dt * load_value(B, dtype, j);",
     "const double Bbar = (exp(dt * a) - 1.0) / a * load_value(B, dtype, j);"),
    ("readout_before_update",
     "h[n] = exp(dt * a) * h[n] + Bbar * x;\n            acc += load_value(C, dtype, j) * h[n];",
     "acc += load_value(C, dtype, j) * h[n];\n            h[n] = exp(dt * a) * h[n] + Bbar * x;"),
    ("bias_after_softplus",
     "if (delta_bias)\n            dt += (double)delta_bias[d];\n        if (delta_softplus)\n            dt = softplus(dt);",
     "if (delta_softplus)\n            dt = softplus(dt);\n        if (delta_bias)\n            dt += (double)delta_bias[d];"),
    ("no_gate", "acc *= silu(load_value(z, dtype, i));\n        y[t] = acc;", "(void)0;\n        y[t] = acc;"),
    ("sigmoid_not_silu", "return v / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(-v));"),
    ("transition_index_transposed", "const double a = (double)A[d * dstate + n];",
     "const double a = (double)A[n * dim + d];"),
    ("input_index_uses_state_row", "const double Bbar = dt * load_value(B, dtype, j);",
     "const double Bbar = dt * load_value(B, dtype, (b * dstate + n) * seqlen + (seqlen - 1 - t));"),
    ("softplus_is_exp", "return v > 20.0 ? v : log1p(exp(v));", "return v > 20.0 ? v : exp(v);"),
    ("bf16_shift", "<< 16;", "<< 15;"),
    ("token_not_scaled", "h[n] = exp(dt * a) * h[n] + Bbar * x;", "h[n] = exp(dt * a) * h[n] + Bbar;"),
    ("state_not_reset_per_row",
     "h[n] = h0 ? h0[r * dstate + n] : 0.0;\n        scan_row(b, d, dim, dstate, seqlen, dtype, u, NULL,",
     "h[n] = h0 ? h0[r * dstate + n] : (r > 0 ? 0.5 : 0.0);\n        scan_row(b, d, dim, dstate, seqlen, dtype, u, NULL,"),
    ("conv_taps_not_reversed", "acc += (double)w[k] * load_value(x, dtype, row * seqlen + s);",
     "acc += (double)w[width - 1 - k] * load_value(x, dtype, row * seqlen + s);"),
    ("conv_window_off_by_one", "const int64_t s = t - (width - 1) + k;", "const int64_t s = t - width + k;"),
    ("conv_no_silu", "u_row[t] = conv_silu ? silu(acc) : acc;", "u_row[t] = acc;"),
    ("conv_bias_dropped", "double acc = bias;", "double acc = 0.0 * bias;"),
    ("conv_state_not_shifted", "cs[k] = cs[k + 1];", "cs[k] = cs[k];"),
    ("trap_beta_without_decay", "const double beta = (1.0 - lam) * dt * alpha;",
     "const double beta = (1.0 - lam) * dt;"),
    ("trap_gate_weights_swapped", "const double gamma = lam * dt;", "const double gamma = (1.0 - lam) * dt;"),
    ("trap_previous_input_frozen", "v_prev[n] = v;", "v_prev[n] = 0.0 * v;"),
    ("trap_no_sigmoid", "const double lam = sigmoid(load_value(lambda_raw, dtype, i));",
     "const double lam = load_value(lambda_raw, dtype, i);"),
    ("bwd_decay_term_dropped", "ddt += gn * (Bb[n * L + t] * ur[t] + hprev * a * Ar[n]);",
     "ddt += gn * (Bb[n * L + t] * ur[t]);"),
    ("bwd_transition_uses_new_state", "dA[d * N + n] += gn * hprev * a * dt;",
     "dA[d * N + n] += gn * H[t * N + n] * a * dt;"),
    ("bwd_final_state_gradient_ignored", "g[n] = dhT ? dhT[row * N + n] : 0.0;", "g[n] = 0.0;"),
    ("bwd_softplus_derivative_missing", "ddt *= 1.0 / (1.0 + exp(-(dr[t] + bias)));", "ddt *= 1.0;"),
    ("bwd_gate_derivative_is_silu", "dz[row * L + t] = ds * sp[t] * sg * (1.0 + zz * (1.0 - sg));",
     "dz[row * L + t] = ds * sp[t] * zz * sg;"),
    ("bwd_input_matrix_gradient_misses_token", "dB[(b * N + n) * L + t] += gn * dt * ur[t];",
     "dB[(b * N + n) * L + t] += gn * dt;"),
    ("bwd_carry_not_decayed", "g[n] = a * gn;", "g[n] = gn;"),
    ("conv_decode_taps_reversed", "acc += (double)conv_w[d * width + k] * cs[k];",
     "acc += (double)conv_w[d * width + width - 1 - k] * cs[k];"),
    ("ssd_group_index_modulo", "g = h / heads_per_group;", "g = h % ngroups;"),
    ("ssd_skip_dropped", "acc += (double)D[h] * xv;", "acc += 0.0 * xv;"),
    ("ssd_decay_sign", "const double a = exp(delta * (double)A[h]);", "const double a = exp(-delta * (double)A[h]);"),
    ("ssd_input_not_discretised", "const double xbar = delta * xv;", "const double xbar = xv;"),
    ("ssd_readout_reads_C_as_B", "acc += *hpn * ssd_load(C, dtype, brow + n);",
     "acc += *hpn * ssd_load(B, dtype, brow + n);"),
    ("ssd_bias_after_softplus",
     "if (dt_bias)\n                delta += (double)dt_bias[h];\n            if (dt_softplus)\n"
     "                delta = delta > 20.0 ? delta : log1p(exp(delta));",
     "if (dt_softplus)\n                delta = delta > 20.0 ? delta : log1p(exp(delta));\n"
     "            if (dt_bias)\n                delta += (double)dt_bias[h];"),
    ("ssd_gate_dropped", "acc *= zv / (1.0 + exp(-zv));", "acc *= 1.0 + 0.0 * zv;"),
    ("ssd_state_not_reset_per_pair", "H[i] = h0 ? h0[r * P * N + i] : 0.0;",
     "H[i] = h0 ? h0[r * P * N + i] : (r > 0 ? 0.25 : 0.0);"),
    ("ssd_bf16_shift", "<< 16u;", "<< 15u;"),
    ("ssd_rec_decay_applied_to_input", "*hpn = a[t] * *hpn + X[t * P + p] * B[t * N + n];",
     "*hpn = a[t] * (*hpn + X[t * P + p] * B[t * N + n]);"),
    ("ssd_rec_readout_before_update",
     "*hpn = a[t] * *hpn + X[t * P + p] * B[t * N + n];\n                acc += *hpn * C[t * N + n];",
     "acc += *hpn * C[t * N + n];\n                *hpn = a[t] * *hpn + X[t * P + p] * B[t * N + n];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    texts = {src: open(src).read() for src in oracle.SOURCES}
    assert sum(t.count(old) for t in texts.values()) == 1, f"mutation site for {name} not found exactly once"
    paths = []
    for src, text in texts.items():
        path = os.path.join(tmp_path, os.path.basename(src))
        with open(path, "w") as f:
            f.write(text.replace(old, new))
        paths.append(path)
    orc = oracle.Variant(oracle.compile_source(paths, os.path.join(tmp_path, f"{name}.so")))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
