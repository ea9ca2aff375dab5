"""Plant plausible mistakes in copies of the oracle and check the pins catch each.

Every mutant is a one-line edit of oracle/ssd_oracle.c (a dropped term, a
wrong sign or index, a swapped operand), compiled to a temporary library on
the CPU.  The test passes only if at least one pin rejects every mutant.
"""
import os
import subprocess

import pytest

import oracle
from oracle_pins import PINS

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "ssd_oracle.c")

MUTANTS = {
    "drop_D_skip": ("yt[p] = acc + Dh * xp;", "yt[p] = acc;"),
    "decay_sign": ("const double a = exp(dtv * Ah);", "const double a = exp(-dtv * Ah);"),
    "decay_missing_dt": ("const double a = exp(dtv * Ah);", "const double a = exp(Ah);"),
    "input_missing_dt": ("const double u = dtv * xp;", "const double u = xp;"),
    "output_uses_B": ("acc += (double)Ct[n] * Sp[n];", "acc += (double)Bt[n] * Sp[n];"),
    "output_before_update": (
        "Sp[n] = a * Sp[n] + u * (double)Bt[n];\n                    acc += (double)Ct[n] * Sp[n];",
        "acc += (double)Ct[n] * Sp[n];\n                    Sp[n] = a * Sp[n] + u * (double)Bt[n];"),
    "h0_ignored": ("S[i] = h0 ? h0[(((int64_t)bi * H + h) * P) * N + i] : 0.0;", "S[i] = 0.0;"),
    "group_index": ("const int g = (int)((int64_t)h * G / H);", "const int g = h % G;"),
    "ckpt_off_by_one": ("if (h_ckpt && s > 0 && (t + 1) % s == 0) {\n                const int64_t k = (t + 1) / s - 1;",
                        "if (h_ckpt && s > 0 && t % s == 0 && t > 0) {\n                const int64_t k = t / s - 1;"),
    "conv_shift": ("int64_t tt = t - (ORACLE_CONV_K - 1) + k;",
                   "int64_t tt = t - (ORACLE_CONV_K - 1) + k - 1;"),
    "conv_weight_flip": ("z += (double)w[c * ORACLE_CONV_K + k] * val;",
                         "z += (double)w[c * ORACLE_CONV_K + (ORACLE_CONV_K - 1 - k)] * val;"),
    "conv_tail_order": ("else val = tb ? (double)tb[(3 + tt) * Cch + c] : 0.0;",
                        "else val = tb ? (double)tb[(-1 - tt) * Cch + c] : 0.0;"),
    "silu_sign": ("double silu = z / (1.0 + exp(-z));", "double silu = z / (1.0 + exp(z));"),
    "tail_out_shift": ("int64_t pos = L - 3 + r;", "int64_t pos = L - 4 + r;"),
    "bf16_ties_away": ("double r = nearbyint(ldexp(fabs(d), -q));", "double r = round(ldexp(fabs(d), -q));"),
    "bias_dropped": ("double z = bias ? (double)bias[c] : 0.0;", "double z = 0.0;"),
    # reverse mode
    "bwd_decay_grad_dropped": ("ddt[((int64_t)bi * L + t) * H + h] = ddt_acc + Ah * dA_t;",
                               "ddt[((int64_t)bi * L + t) * H + h] = ddt_acc;"),
    "bwd_adjoint_not_decayed": ("for (int64_t i = 0; i < PN; ++i) Gs[i] *= a_t;",
                                "for (int64_t i = 0; i < PN; ++i) Gs[i] *= 1.0;"),
    "bwd_dC_previous_state": ("c_acc += dyt[p] * hcur[(int64_t)p * N + n];",
                              "c_acc += dyt[p] * hprev[(int64_t)p * N + n];"),
    "bwd_dB_missing_dt": ("dBt[n] = dtv * b_acc;", "dBt[n] = b_acc;"),
    "bwd_dx_skip_dropped": ("dxt[p] = Dh * dyt[p] + dtv * acc;", "dxt[p] = dtv * acc;"),
    "bwd_seed_ignored": ("Gs[i] = dh_final ? dh_final[((int64_t)bi * H + h) * PN + i] : 0.0;", "Gs[i] = 0.0;"),
    "bwd_dA_missing_dt": ("dA_acc += dtv * dA_t;", "dA_acc += dA_t;"),
    "bwd_wrong_checkpoint": ("else v = h_ckpt[(((int64_t)bi * n_ckpt + (k - 1)) * H + h) * PN + i];",
                             "else v = h_ckpt[(((int64_t)bi * n_ckpt + (k > 1 ? k - 2 : 0)) * H + h) * PN + i];"),
    # gated RMS norm
    "norm_gate_dropped": ("v[c] = (double)y[r * y_rs + c] * (zc / (1.0 + exp(-zc)));",
                          "v[c] = (double)y[r * y_rs + c];"),
    "norm_eps_outside_sqrt": ("const double scale = 1.0 / sqrt(ss / group + eps);",
                              "const double scale = 1.0 / (sqrt(ss / group) + eps);"),
    "norm_mean_over_all_channels": ("const double scale = 1.0 / sqrt(ss / group + eps);",
                                    "const double scale = 1.0 / sqrt(ss / d + eps);"),
    "norm_weight_dropped": ("out[r * out_rs + c] = (float)round_io(v[c] * scale * (double)w[c], io_round);",
                            "out[r * out_rs + c] = (float)round_io(v[c] * scale, io_round);"),
    # reverse mode of the whole layer (conv + SiLU, then the recurrence)
    "layer_bwd_silu_grad_dropped": ("const double dz = dv[j * Cch + c] * (sg * (1.0 + zz * (1.0 - sg)));",
                                    "const double dz = dv[j * Cch + c];"),
    "layer_bwd_sigmoid_grad_instead": ("const double dz = dv[j * Cch + c] * (sg * (1.0 + zz * (1.0 - sg)));",
                                       "const double dz = dv[j * Cch + c] * (sg * (1.0 - sg));"),
    "layer_bwd_cell_buffer_zero": ("else val = conv_ckpt[(((int64_t)bi * n_ckpt + (k - 1)) * 3 + r) * Cch + c];",
                                   "else val = 0.0;"),
    "layer_bwd_tail_grad_dropped": ("else dtb[(3 + tt) * Cch + c] += wv * dz;",
                                    "else dtb[(3 + tt) * Cch + c] += 0.0 * wv * dz;"),
    "layer_bwd_dw_taps_flipped": ("dwb[c * ORACLE_CONV_K + kk] += dz * val;",
                                  "dwb[c * ORACLE_CONV_K + (ORACLE_CONV_K - 1 - kk)] += dz * val;"),
    "layer_bwd_dB_heads_not_summed": ("dvt[HP + grp * N + n] += dtv * b_acc;",
                                      "dvt[HP + grp * N + n] = dtv * b_acc;"),
    "layer_bwd_tail_out_grad_ignored": ("if (at >= 0) dub[at * Cch + c] += g;",
                                        "if (at >= 0) dub[at * Cch + c] += 0.0 * g;"),
    "layer_bwd_du_misplaced": ("if (tt >= 0) dub[tt * Cch + c] += wv * dz;",
                               "if (tt >= 0) dub[t * Cch + c] += wv * dz;"),
    "bwd_adjoint_after_output": ("Gs[(int64_t)p * N + n] += dyt[p] * (double)Ct[n];",
                                 "Gs[(int64_t)p * N + n] += 0.0 * dyt[p] * (double)Ct[n];"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
                           "-fPIC", "-shared", "-std=c11", str(path), "-o", str(lib), "-lm"])
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    lib = _build_mutant(tmp_path, name, old, new)
    prev = oracle.use_library(lib)
    caught = []
    try:
        for pin in PINS:            # one rejecting pin is enough
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
                break
    finally:
        oracle.use_library(prev)
    assert caught, f"no pin rejects mutant {name}"
