"""The oracle's pins are strong enough to catch plausible slips.

Each mutant below is a copy of oracle/r2l_oracle.c with one plausible mistake
planted in it (on the CPU only).  The pin suite is run against the mutant in a
subprocess and must fail.  A mutant that survives would mean the pins do not
constrain that part of the oracle.
"""

import os
import shutil
import subprocess
import sys
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "r2l_oracle.c")

MUTANTS = {
    "dropped_D_skip": ("double yv = acc_y + Dskip[d] * u;", "double yv = acc_y;"),
    "A_sign": ("const double abar = exp(delta * A[d * d_state + n]);",
               "const double abar = exp(-delta * A[d * d_state + n]);"),
    "bwd_forward_A_sign": ("const double a = exp(delta * A[d * d_state + n]);",
                           "const double a = exp(-delta * A[d * d_state + n]);"),
    "zoh_instead_of_euler_B": ("h[n] = abar * h[n] + delta * Bm[row * d_state + n] * u;",
                               "h[n] = abar * h[n] + (abar - 1.0) / A[d * d_state + n] * Bm[row * d_state + n] * u;"),
    "exclusive_state": ("h[n] = abar * h[n] + delta * Bm[row * d_state + n] * u;\n                        acc_y += Cm[row * d_state + n] * h[n];",
                        "acc_y += Cm[row * d_state + n] * h[n];\n                        h[n] = abar * h[n] + delta * Bm[row * d_state + n] * u;"),
    "conv_taps_flipped": ("const long back = conv_width - 1 - k;", "const long back = k;"),
    "no_block_reset": ("for (long n = 0; n < d_state; ++n)\n                    h[n] = (!reverse && h0)",
                       "if (blk == 0) for (long n = 0; n < d_state; ++n)\n                    h[n] = (!reverse && h0)"),
    "softplus_is_exp": ("v > 20.0 ? v : log1p(exp(v))", "v > 20.0 ? v : exp(v)"),
    "gate_is_sigmoid": ("static double silu(double v) { return v / (1.0 + exp(-v)); }",
                        "static double silu(double v) { return 1.0 / (1.0 + exp(-v)); }"),
    "W_out_transposed": ("W_out[j * d_inner + k]", "W_out[k * d_model + j]"),
    "s_ignored": ("hidden[m * d_model + j] + s * acc", "hidden[m * d_model + j] + acc"),
    "conv_pad_outside_block": ("(tt >= s0 && tt < s1)", "(tt >= 0 && tt < seqlen)"),
    "D_on_raw_x": ("double yv = acc_y + Dskip[d] * u;", "double yv = acc_y + Dskip[d] * x[row * d_inner + d];"),
    "conv_state_oldest_first": ("xv = conv_state[(b * d_inner + d) * (conv_width - 1) + (s0 - 1 - tt)];",
                                "xv = conv_state[(b * d_inner + d) * (conv_width - 1) + (conv_width - 2 - (s0 - 1 - tt))];"),
    "conv_state_out_oldest_first": ("const long tt = s1 - 1 - j;", "const long tt = s1 - conv_width + 1 + j;"),
    "linear_transposed": ("acc += X[m * K + k] * W[n * K + k];", "acc += X[m * K + k] * W[k * N + n];"),
    "conv_silu_wrong_direction": ("const long tsrc = reverse ? t + lag : t - lag;",
                                  "const long tsrc = reverse ? t - lag : t + lag;"),
    "bwd_dA_without_a": ("dA[d * d_state + n] += da * a * delta;", "dA[d * d_state + n] += da * delta;"),
    "bwd_adjoint_without_carry": ("exp(delta_prev * An) * G[n]", "G[n]"),
    "bwd_dz_without_p": ("dz[row * d_inner + d] = dy[row * d_inner + d] * p * dg;",
                         "dz[row * d_inner + d] = dy[row * d_inner + d] * dg;"),
    "bwd_no_softplus_slope": ("const double ddt_t = ddelta / (1.0 + exp(-v));", "const double ddt_t = ddelta;"),
    "bwd_dB_without_delta": ("dB[row * d_state + n] += G[n] * delta * u;", "dB[row * d_state + n] += G[n] * u;"),
    "bwd_conv_without_silu_slope": ("const double dc = dub[t - s0] * sg * (1.0 + c * (1.0 - sg));",
                                    "const double dc = dub[t - s0] * sg;"),
    "bwd_conv_taps_flipped": ("dx[(b * seqlen + tt) * d_inner + d] += conv_w[d * W + k] * dc;",
                              "dx[(b * seqlen + tt) * d_inner + d] += conv_w[d * W + (W - 1 - k)] * dc;"),
    "conv_state_out_drops_cache": ("cs_new[j] = conv_state ? conv_state[(b * d_inner + d) * (conv_width - 1) + (s0 - 1 - tt)] : 0.0;",
                                   "cs_new[j] = 0.0;"),
}


# Mistakes planted in the Python side of the oracle (the sidecar's wiring).
PY_MUTANTS = {
    "xz_halves_swapped": ("x, z = xz[:, :d_inner], keep(xz[:, d_inner:])",
                          "z, x = keep(xz[:, :d_inner]), xz[:, d_inner:]"),
    "B_C_swapped": ("dt_low, Bm, Cm = dbl[:, :dt_rank]", "dt_low, Cm, Bm = dbl[:, :dt_rank]"),
    "sidecar_conv_forward": ("u = conv_silu(x.reshape(batch, seqlen, d_inner), w[\"conv_w\"], w[\"conv_b\"], reverse=True,",
                             "u = conv_silu(x.reshape(batch, seqlen, d_inner), w[\"conv_w\"], w[\"conv_b\"], reverse=False,"),
    "round_bf16_truncates": ("((bits + 0x7FFF + kept_lsb) & 0xFFFF0000)", "(bits & 0xFFFF0000)"),
    "round_bf16_ties_away": ("((bits + 0x7FFF + kept_lsb) & 0xFFFF0000)", "((bits + 0x8000) & 0xFFFF0000)"),
    "sidecar_dt_not_stored_bf16": ("dt = keep(linear(dt_low, w[\"W_dt\"]))", "dt = linear(dt_low, w[\"W_dt\"])"),
    "sidecar_x_rounded_before_conv": ("x, z = xz[:, :d_inner], keep(xz[:, d_inner:])",
                                      "x, z = keep(xz[:, :d_inner]), keep(xz[:, d_inner:])"),
    "sidecar_scan_forward": ("w[\"D\"], w[\"dt_bias\"], None, None, reverse=True,",
                             "w[\"D\"], w[\"dt_bias\"], None, None, reverse=False,"),
}


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_catch_python_mutant(name, tmp_path):
    old, new = PY_MUTANTS[name]
    pkg = tmp_path / "oracle"
    shutil.copytree(os.path.join(ROOT, "oracle"), pkg, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    init = pkg / "__init__.py"
    src = init.read_text()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    init.write_text(src.replace(old, new))
    env = dict(os.environ, R2L_ORACLE_PKG_DIR=str(tmp_path))
    env.pop("R2L_ORACLE_LIB", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pin suite:\n{r.stdout[-2000:]}"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut_c = tmp_path / "mutant.c"
    mut_c.write_text(src.replace(old, new))
    mut_so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-o", str(mut_so), str(mut_c), "-lm"])
    env = dict(os.environ, R2L_ORACLE_LIB=str(mut_so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pin suite:\n{r.stdout[-2000:]}"
