"""The oracle's pins must be able to fail.  Each case plants one plausible
mistake (a transposed operand, a wrong sign or index, a dropped term) in a
copy of ``oracle.c``, compiles it on the CPU, swaps it in, and checks that at
least one pin from ``test_oracle_pins`` now fails.  CPU only."""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, original text, mutated text)
MUTATIONS = [
    ("B_for_C_in_update", "h[n] = a * h[n] + delta * Brow[n * L + t] * u[t];",
     "h[n] = a * h[n] + delta * Crow[n * L + t] * u[t];"),
    ("decay_sign", "double a = exp(delta * A[d * N + n]);", "double a = exp(-delta * A[d * N + n]);"),
    ("drop_skip_term", "y += (Dv ? Dv[d] : 0.0) * u[t];", "(void)Dv;"),
    ("history_index", "xin[k] = hist_w ? hist_w[k + 1] : 0.0;", "xin[k] = hist_w ? hist_w[k] : 0.0;"),
    ("flipped_taps", "acc += w[k] * xin[t + k];", "acc += w[W - 1 - k] * xin[t + k];"),
    ("softplus_formula", "return log1p(exp(v));", "return exp(v);"),
    ("gate_added", "if (z) y *= o_silu(z[row * L + t]);", "if (z) y += o_silu(z[row * L + t]);"),
    ("dt_bias_dropped_scan", "double v = dt[row * L + t] + (dt_bias ? dt_bias[d] : 0.0);",
     "double v = dt[row * L + t];"),
    ("h0_ignored", "for (n = 0; n < N; ++n) h[n] = h0 ? h0[row * N + n] : 0.0;",
     "for (n = 0; n < N; ++n) h[n] = 0.0;"),
    ("group_index_scan", "const int64_t g = d / (D / G);", "const int64_t g = d % G;"),
    ("ssu_roll_direction", "for (k = 0; k < W - 1; ++k) cs[k] = cs[k + 1];",
     "for (k = W - 2; k >= 0; --k) cs[k + 1] = cs[k];"),
    ("ssu_decay_sign", "double a = exp(delta * A[hp * N + n]);", "double a = exp(delta * A[hp * N + n] * 0.5);"),
    ("ssu_skip_dropped", "y += (Dv ? Dv[hp] : 0.0) * u;", "(void)Dv;"),
    ("ssu_state_written_late", "s[n] = a * s[n] + delta * Bv[n] * u;\n                    y += Cv[n] * s[n];",
     "y += Cv[n] * s[n];\n                    s[n] = a * s[n] + delta * Bv[n] * u;"),
    ("mamba2_group_index", "const double* Bv = Bm + (b * G + hh / heads_per_group) * N;",
     "const double* Bv = Bm + (b * G + hh % G) * N;"),
    ("mamba2_skip_uses_state", "if (D_head) y += D_head[hh] * xv;", "if (D_head) y += D_head[hh] * s[0];"),
    ("conv_state_out_shift", "for (k = 0; k < W; ++k) hist_out[k] = all[L + k];",
     "for (k = 0; k < W; ++k) hist_out[k] = all[L + k - (k > 0)];"),
    ("m2_prefill_group_index", "const int64_t grp = hh / per_group;", "const int64_t grp = hh % G;"),
    ("m2_prefill_readout_before_update",
     "S[p * N + n] = decay * S[p * N + n] + delta * Bg[n * L + t] * xv;\n                        acc += Cg[n * L + t] * S[p * N + n];",
     "acc += Cg[n * L + t] * S[p * N + n];\n                        S[p * N + n] = decay * S[p * N + n] + delta * Bg[n * L + t] * xv;"),
    ("m2_prefill_bias_dropped", "double v = dt[(b * H + hh) * L + t] + (dt_bias_head ? dt_bias_head[hh] : 0.0);",
     "double v = dt[(b * H + hh) * L + t];"),
    ("m2_prefill_skip_dropped", "if (D_head) acc += D_head[hh] * xv;", "(void)D_head;"),
    ("m2_prefill_decay_sign", "double decay = exp(delta * A_head[hh]);", "double decay = exp(-delta * A_head[hh]);"),
    ("m2_prefill_C_for_B_in_update", "delta * Bg[n * L + t] * xv", "delta * Cg[n * L + t] * xv"),
    ("m2_prefill_h0_ignored", "S[p * N + n] = h0 ? h0[((b * H + hh) * P + p) * N + n] : 0.0;",
     "S[p * N + n] = 0.0;"),
    ("m2_prefill_gate_on_x", "if (z) acc *= o_silu(z[at]);", "if (z) acc *= o_silu(x[at]);"),
    ("m2_prefill_softplus_ignored",
     "double v = dt[(b * H + hh) * L + t] + (dt_bias_head ? dt_bias_head[hh] : 0.0);\n"
     "                double delta = dt_softplus ? o_softplus(v) : v;",
     "double v = dt[(b * H + hh) * L + t] + (dt_bias_head ? dt_bias_head[hh] : 0.0);\n"
     "                double delta = v;"),
    ("m2_prefill_time_reversed", "const int64_t at = ((b * H + hh) * P + p) * L + t;",
     "const int64_t at = ((b * H + hh) * P + p) * L + (L - 1 - t);"),
    ("conv_bias_dropped", "double acc = bias;", "double acc = 0.0; (void)bias;"),
    ("conv_silu_skipped", "out[t] = silu ? o_silu(acc) : acc;", "out[t] = acc; (void)silu;"),
    ("scan_A_transposed", "double a = exp(delta * A[d * N + n]);", "double a = exp(delta * A[n * D + d]);"),
    ("ssu_conv_silu_skipped", "u = o_silu(acc);", "u = acc;"),
    ("ssu_dt_bias_dropped", "double v = dt[row] + (dt_bias ? dt_bias[hp] : 0.0);", "double v = dt[row];"),
    ("ssu_gate_dropped", "y += (Dv ? Dv[hp] : 0.0) * u;\n                if (z) y *= o_silu(z[row]);",
     "y += (Dv ? Dv[hp] : 0.0) * u;\n                (void)z;"),
    ("mamba2_decay_of_head_zero", "double dA = exp(delta * A_head[hh]);", "double dA = exp(delta * A_head[0]);"),
    ("round_ties_away_from_zero", "const double r = nearbyint(v / q) * q;", "const double r = round(v / q) * q;"),
    ("round_f16_one_bit_short", "v[i] = o_round_bits(v[i], 11, -14, 65504.0, 16.0);",
     "v[i] = o_round_bits(v[i], 10, -14, 65504.0, 16.0);"),
    ("round_bf16_one_bit_long", "v[i] = o_round_bits(v[i], 8, -126,", "v[i] = o_round_bits(v[i], 9, -126,"),
    ("round_f16_subnormal_quantum", "v[i] = o_round_bits(v[i], 11, -14, 65504.0, 16.0);",
     "v[i] = o_round_bits(v[i], 11, -15, 65504.0, 16.0);"),
    ("delta_sum_bias_dropped", "const double v = dt[(b * D + d) * L + t] + (dt_bias ? dt_bias[d] : 0.0);",
     "const double v = dt[(b * D + d) * L + t];"),
    ("delta_sum_softplus_skipped", "sum += dt_softplus ? o_softplus(v) : v;", "sum += v;"),
    ("carry_fold_decay_sign", "state[i] = exp(A[d * N + n] * S[b * D + d]) * state[i] + h_end[i];",
     "state[i] = exp(-A[d * N + n] * S[b * D + d]) * state[i] + h_end[i];"),
    ("carry_fold_end_state_dropped", "state[i] = exp(A[d * N + n] * S[b * D + d]) * state[i] + h_end[i];",
     "state[i] = exp(A[d * N + n] * S[b * D + d]) * state[i];"),
    ("carry_fold_A_transposed", "state[i] = exp(A[d * N + n] * S[b * D + d]) * state[i] + h_end[i];",
     "state[i] = exp(A[n * D + d] * S[b * D + d]) * state[i] + h_end[i];"),
    ("gated_conv_gates_swapped", "for (t = 0; t < L; ++t) v[t] = Bg[row * L + t] * x[row * L + t];",
     "for (t = 0; t < L; ++t) v[t] = Cg[row * L + t] * x[row * L + t];"),
    ("gated_conv_output_gate_dropped", "for (t = 0; t < L; ++t) out[row * L + t] = Cg[row * L + t] * c[t];",
     "for (t = 0; t < L; ++t) out[row * L + t] = c[t];"),
    ("gated_conv_input_gate_after_conv", "for (t = 0; t < L; ++t) v[t] = Bg[row * L + t] * x[row * L + t];",
     "for (t = 0; t < L; ++t) v[t] = x[row * L + t];"),
    ("gated_conv_bias_dropped", "bias ? bias[d] : 0.0, 0, c,", "0.0, 0, c,"),
    ("gated_conv_output_gate_one_step_late", "out[row * L + t] = Cg[row * L + t] * c[t];",
     "out[row * L + t] = Cg[row * L + (t > 0 ? t - 1 : 0)] * c[t];"),
    ("gated_conv_state_ignored", "o_conv_channel(L, W, conv_state_in ? conv_state_in + row * W : NULL, v,",
     "o_conv_channel(L, W, NULL, v,"),
]

# pins exercised against each mutant (all cheap)
PIN_CALLS = [
    lambda: pins.test_scan_matches_brute_force(2, 2, 3, 8, 4, 1, 4),
    lambda: pins.test_scan_matches_brute_force(3, 1, 3, 7, 2, 3, 3),
    lambda: pins.test_scan_matches_brute_force(4, 2, 2, 3, 4, 2, 4),
    lambda: pins.test_scan_matches_brute_force(6, 1, 4, 5, 2, 2, 4),
    lambda: pins.test_scan_closed_form_constant_inputs(-0.7),
    lambda: pins.test_prefill_then_decode_equals_full_prefill(3),
    lambda: pins.test_ssu_single_step_matches_scan_brute_force_with_groups(),
    lambda: pins.test_mamba2_notation_matches_general_form(2),
    lambda: pins.test_mamba2_groups_map_consecutive_heads(),
    lambda: pins.test_conv_matches_numpy_convolve_and_state(7),
    lambda: pins.test_conv_matches_numpy_convolve_and_state(2),
    lambda: pins.test_conv_impulse_response(4),
    lambda: pins.test_activation_special_values(),
    lambda: pins.test_mamba2_prefill_matches_mamba1_scan_with_heads_expanded(2),
    lambda: pins.test_mamba2_prefill_equals_repeated_decode(),
    lambda: pins.test_mamba2_prefill_two_steps_by_hand(),
    lambda: pins.test_round_cache_matches_library_conversions(),
    lambda: pins.test_round_cache_ties_go_to_even(),
    lambda: pins.test_delta_sum_is_the_decay_exponent_of_the_scan(True),
    lambda: pins.test_carry_fold_composes_sequence_pieces((3, 8)),
    lambda: pins.test_gated_conv_matches_numpy_convolve_and_state(5, 3),
    lambda: pins.test_gated_conv_impulse_response(3),
]


@pytest.mark.parametrize("name,orig,mut", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, orig, mut, tmp_path):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(orig, mut))
    lib_path = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", str(path), "-o",
                           str(lib_path), "-lm"])
    saved = oracle._load()
    oracle._lib = oracle.configure(ctypes.CDLL(str(lib_path)))
    failures = 0
    try:
        for call in PIN_CALLS:
            try:
                call()
            except AssertionError:
                failures += 1
    finally:
        oracle._lib = saved
    assert failures > 0, f"no pin caught the planted mistake {name}"
