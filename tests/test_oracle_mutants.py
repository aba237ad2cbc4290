"""Plant a mistake in a copy of the oracle and check that some pin catches it.

Each mutant is oracle.c with one plausible slip (a dropped term, a wrong sign, a
wrong index, a transposed operand), compiled into a temporary directory.  The test
passes when every mutant fails at least one pin, which shows that the pins do not
merely re-run the oracle's own formula.  CPU only; nothing here touches a GPU.
"""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "drop_D_skip": ("yt += D[d] * x;", "yt += 0.0 * x;"),
    "decay_sign": ("exp(dt * A[d * N + n])", "exp(-dt * A[d * N + n])"),
    "bbar_without_delta": ("if (!zoh || An == 0.0) return dt * Bn;", "if (!zoh || An == 0.0) return Bn;"),
    "readout_uses_B": ("yt += Ct[n] * h[n];", "yt += Bt[n] * h[n];"),
    "A_transposed": ("exp(dt * A[d * N + n])", "exp(dt * A[n * Di + d])"),
    "readout_before_update": (
        "h[n] = Abar * h[n] + Bbar * x;                    /* h_t = Abar h + Bbar x */\n"
        "                yt += Ct[n] * h[n];",
        "yt += Ct[n] * h[n];\n                h[n] = Abar * h[n] + Bbar * x;"),
    "backward_not_reversed": ("order[t] = L - 1 - t;", "order[t] = t;"),
    "backward_uses_forward_bias": ("D + Di, bias + Di, order", "D + Di, bias, order"),
    "backward_uses_forward_bc": ("B + bc_dir_stride, C + bc_dir_stride", "B, C"),
    "softplus_wrong": ("log1p(exp(x))", "log(exp(x) + 0.5)"),
    "gate_is_sigmoid": ("return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    "column_scan_is_row_scan": ("int64_t h = s % H, w = s / H;", "int64_t h = s / W, w = s % W;"),
    "column_scan_transposed": ("p = h * W + w;", "p = w * H + h;"),
    "cross_bc_not_per_direction": ("B + k * bc, C + k * bc", "B, C"),
    "merge_ignores_order": ("int64_t p = order[t];\n                for (int64_t c = 0",
                            "int64_t p = t;\n                for (int64_t c = 0"),
    "delta_bias_ignored": ("softplus(delta[ix] + bias[d])", "softplus(delta[ix])"),
    "conv_backward_taps_forward": ("int64_t s = reversed ? t + 1 - k : t + k - 1;",
                                   "int64_t s = t + k - 1;"),
    "conv_bias_dropped": ("double acc = cb[d];", "double acc = 0.0;"),
    "conv_padding_crosses_sequences": ("if (s >= 0 && s < L) acc += w[d * 3 + k] * x[(b * L + s) * Di + d];",
                                       "if (b * L + s >= 0 && b * L + s < batch * L)\n"
                                       "                        acc += w[d * 3 + k] * x[(b * L + s) * Di + d];"),
    "conv_no_silu": ("u[(b * L + t) * Di + d] = silu(acc);", "u[(b * L + t) * Di + d] = acc;"),
    "conv_backward_uses_forward_weights": ("oracle_conv_silu(x, conv_w + (int64_t)Di * 3, conv_b + Di, ub",
                                           "oracle_conv_silu(x, conv_w, conv_b, ub"),
    "zoh_ignored": ("return expm1(dt * An) / An * Bn;", "return dt * Bn;"),
    "zoh_no_division_by_A": ("return expm1(dt * An) / An * Bn;", "return expm1(dt * An) * Bn;"),
    "zoh_exp_for_expm1": ("return expm1(dt * An) / An * Bn;", "return exp(dt * An) / An * Bn;"),
    "zoh_delta_twice": ("return expm1(dt * An) / An * Bn;", "return dt * expm1(dt * An) / An * Bn;"),
    "zoh_dropped_in_bidir": ("delta_is_raw, 0, zoh);", "delta_is_raw, 0, 0);"),
    "zoh_dropped_in_cross": ("delta_is_raw, k > 0, zoh);", "delta_is_raw, k > 0, 0);"),
    "bwd_adjoint_not_decayed": ("g[n] *= Abar;", "g[n] *= 1.0;"),
    "bwd_hprev_is_h": ("double hprev = t > 0 ? hs[(t - 1) * N + n] : 0.0;", "double hprev = hs[t * N + n];"),
    "bwd_dA_without_delta": ("dA_loc[d * N + n] += dAbar * Abar * dt;", "dA_loc[d * N + n] += dAbar * Abar;"),
    "bwd_dB_without_u": ("dBt[n] += g[n] * gain * x;", "dBt[n] += g[n] * gain;"),
    "bwd_softplus_grad_sign": ("return x > 20.0 ? 1.0 : 1.0 / (1.0 + exp(-x));",
                               "return x > 20.0 ? 1.0 : 1.0 / (1.0 + exp(x));"),
    "bwd_gate_grad_is_sigmoid": ("return s * (1.0 + z * (1.0 - s));", "return s;"),
    "bwd_D_skip_dropped": ("double dDelta = 0.0, dx = D[d] * e;", "double dDelta = 0.0, dx = 0.0;"),
    "bwd_backward_dir_forward_params": ("A + (int64_t)Di * N, D + Di, bias + Di, order, dy,",
                                        "A, D, bias, order, dy,"),
    "bwd_dy_ungated": ("dy[i] = dout[i] * silu(z[i]);", "dy[i] = dout[i];"),
    "xproj_weight_transposed": ("acc += u[m * Di + d] * Wx[(int64_t)d * NO + j];",
                                "acc += u[m * Di + d] * Wx[(int64_t)j * Di + d];"),
    "cross_bwd_same_order": ("rc |= oracle_cross_order(k, H, W, order);\n        rc |= oracle_s6_direction_bwd",
                             "rc |= oracle_cross_order(0, H, W, order);\n        rc |= oracle_s6_direction_bwd"),
    "zoh_sign": ("return expm1(dt * An) / An * Bn;", "return expm1(-dt * An) / An * Bn;"),
    # the exact hold's derivative
    "zoh_bwd_ddelta_first_order": ("g[n] * Bt[n] * x * hold_gain_ddt(dt, Ad[n], zoh)", "g[n] * Bt[n] * x * 1.0"),
    "zoh_bwd_dA_hold_term_dropped": (
        "if (zoh) dA_loc[d * N + n] += g[n] * Bt[n] * x * hold_gain_dA(dt, Ad[n], zoh);", ""),
    "zoh_bwd_series_coefficient": ("c[k] = (double)k / f;", "c[k] = 1.0 / f;"),
    "zoh_bwd_closed_form_sign": ("(zz * exp(zz) - expm1(zz))", "(zz * exp(zz) + expm1(zz))"),
    # the convolution front's derivative
    "conv_bwd_no_silu_grad": ("double dpre = du[k][(b * L + t) * Di + d] * silu_grad(pre);",
                              "double dpre = du[k][(b * L + t) * Di + d];"),
    "conv_bwd_taps_not_reversed": ("int64_t s = k ? t + 1 - j : t + j - 1;", "int64_t s = t + j - 1;"),
    "conv_bwd_dw_without_x": ("dw[d * 3 + j] += dpre * x[(b * L + s) * Di + d];", "dw[d * 3 + j] += dpre;"),
    "conv_bwd_dx_tap_flipped": ("dx[(b * L + s) * Di + d] += w[d * 3 + j] * dpre;",
                                "dx[(b * L + s) * Di + d] += w[d * 3 + 2 - j] * dpre;"),
    # the projections' derivative
    "block_bwd_ds_without_wdt": ("ds += ddr[k][m * Di + d] * wdt[d];", "ds += ddr[k][m * Di + d];"),
    "block_bwd_dwx_transposed": ("dW[d * NO + j] += u[k][m * Di + d] * dP[j];",
                                 "dW[d * NO + j] += u[k][m * Di + d] * dP[NO - 1 - j];"),
    "block_bwd_du_misses_projection": ("                du[k][m * Di + d] += acc;", "                du[k][m * Di + d] += 0.0 * acc;"),
    "block_bwd_dwdt_without_s": ("dwdt[d] += ddr[k][m * Di + d] * s;", "dwdt[d] += ddr[k][m * Di + d];"),
    "conv_bwd_shared_du": ("rc |= oracle_s6_direction_bwd(u[1], delta, B + bc_dir_stride, C + bc_dir_stride,\n"
                           "                                      A + (int64_t)Di * N, D + Di, bias + Di, order, dy, du[1],",
                           "rc |= oracle_s6_direction_bwd(u[1], delta, B + bc_dir_stride, C + bc_dir_stride,\n"
                           "                                      A + (int64_t)Di * N, D + Di, bias + Di, order, dy, du[0],"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path_c = tmp_path / "oracle_mut.c"
    path_c.write_text(src.replace(old, new))
    path_so = tmp_path / "liboracle_mut.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(path_so), str(path_c), "-lm"],
                   check=True)
    mutant = oracle.Oracle(str(path_so))
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
