"""Plant plausible mistakes in copies of the oracle and check the pins catch each.

Every mutant is a one-line text substitution in the oracle's C source (a
dropped term, a wrong index or sign, a transposed operand, a wrong scale),
compiled into a temporary library on the CPU.  The pins of oracle_pins.py are
re-run against it; the test passes when at least one pin fails.  All mutants
keep every memory access in bounds.
"""
import os

import pytest

import oracle
import oracle.build as obuild
import oracle_pins

MUTANTS = {
    "drop_last_tap": ("int64_t smax = t < L - 1 ? t : L - 1;", "int64_t smax = t < L - 2 ? t : L - 2;"),
    "overwrite_not_accumulate": ("acc += kr[s] * x;", "acc = kr[s] * x;"),
    "input_not_reversed": ("double x = wr ? ur[t - s] * wr[t - s] : ur[t - s];",
                           "double x = wr ? ur[s] * wr[s] : ur[s];"),
    "drop_skip_term": ("acc += (*Dh) * x;", "acc += 0.0 * (*Dh) * x;"),
    "skip_on_u_not_x": ("double x = wr ? ur[t] * wr[t] : ur[t];", "double x = ur[t];"),
    "drop_gate": ("if (vr) acc *= vr[t];", "if (vr) acc *= 1.0;"),
    "gate_on_input_index": ("if (vr) acc *= vr[t];", "if (vr) acc *= vr[0];"),
    "conv2d_kernel_transposed": ("acc += kc[p * Kw + q] * ui[(i - p) * Ws + (j - q)];",
                                 "acc += kc[q * Kw + p] * ui[(i - p) * Ws + (j - q)];"),
    "conv2d_drop_last_row": ("int64_t pmax = i < Kh - 1 ? i : Kh - 1;",
                             "int64_t pmax = i < Kh - 2 ? i : Kh - 2;"),
    "dft_inverse_sign": ("unit_root(-f * t, M, &c, &s); /* exp(+2 pi i f t / M) */",
                         "unit_root(f * t, M, &c, &s);"),
    "dft_wrong_scale": ("y[t] = acc / (double)M;", "y[t] = acc / (double)N;"),
    "dft_product_sign": ("double pr = Xr[f] * Kr[f] - Xi[f] * Ki[f];",
                         "double pr = Xr[f] * Kr[f] + Xi[f] * Ki[f];"),
    "dft2_inverse_sign": ("acc += Pr[fh * Mw + fw] * c - Pi[fh * Mw + fw] * s;",
                         "acc += Pr[fh * Mw + fw] * c + Pi[fh * Mw + fw] * s;"),
    "bwd_correlation_as_convolution": ("double g = v ? dyr[t + j] * v[r * N + t + j] : dyr[t + j];",
                                       "double g = v ? dyr[t - j < 0 ? 0 : t - j] * v[r * N + t + j] : "
                                       "dyr[t - j < 0 ? 0 : t - j];"),
    "bwd_drop_last_lag": ("int64_t jmax = (L - 1 < N - 1 - t) ? L - 1 : N - 1 - t;",
                          "int64_t jmax = (L - 2 < N - 1 - t) ? L - 2 : N - 1 - t;"),
    "bwd_du_not_gated": ("du[r * N + t] = acc * w[r * N + t];", "du[r * N + t] = acc;"),
    "bwd_dw_times_w": ("dw[r * N + t] = acc * ur[t];", "dw[r * N + t] = acc * w[r * N + t];"),
    "bwd_dk_lag_sign": ("double x = w ? u[r * N + t - j] * w[r * N + t - j] : u[r * N + t - j];",
                        "double x = w ? u[r * N + t] * w[r * N + t] : u[r * N + t];"),
    "bwd_dD_ungated_g": ("                    double g = v ? dy[r * N + t] * v[r * N + t] : dy[r * N + t];\n"
                         "                    double x = w ? u[r * N + t] * w[r * N + t] : u[r * N + t];",
                         "                    double g = dy[r * N + t];\n"
                         "                    double x = w ? u[r * N + t] * w[r * N + t] : u[r * N + t];"),
    "dynamic_channel_filter": ("        const double* kr = k + r * L;\n        const double* Dh = D ? D + h : NULL;\n"
                               "        for (int64_t t = 0; t < N; ++t)\n            y[r * N + t] = conv1d_point",
                               "        const double* kr = k + h * L;\n        const double* Dh = D ? D + h : NULL;\n"
                               "        for (int64_t t = 0; t < N; ++t)\n            y[r * N + t] = conv1d_point"),
    "ssm_power_sign": ("double ang = (double)t * atan2(li, lr);", "double ang = -(double)t * atan2(li, lr);"),
    "ssm_drop_imag_part": ("acc += c_re[h * d + j] * pr - c_im[h * d + j] * pi;", "acc += c_re[h * d + j] * pr;"),
    "ssm_power_off_by_one": ("double mag = pow(sqrt(lr * lr + li * li), (double)t);",
                             "double mag = pow(sqrt(lr * lr + li * li), (double)(t + 1));"),
    "conv2d_offset_ignored": ("int64_t fi = i + oy, fj = j + ox;", "int64_t fi = i, fj = j + ox;"),
    "conv2d_offset_clip": ("if (a < 0 || a >= Hs) continue;", "if (a < 0 || a >= Hs - 1) continue;"),
    "conv3d_no_depth_shift": ("acc += k[(e * Kh + p) * Kw + q] * u[((d - e) * Hs + (i - p)) * Ws + (j - q)];",
                              "acc += k[(e * Kh + p) * Kw + q] * u[(d * Hs + (i - p)) * Ws + (j - q)];"),
    "conv3d_drop_last_depth_tap": ("int64_t emax = d < Kd - 1 ? d : Kd - 1;",
                                   "int64_t emax = d < Kd - 2 ? d : Kd - 2;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(obuild.SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique in the oracle source"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    lib = obuild.build(force=True, src=str(mpath), out=str(tmp_path / "libmutant.so"))
    saved = oracle._lib
    oracle._lib = oracle.bind(lib)
    failed = []
    try:
        for check in oracle_pins.ALL_CHECKS:
            try:
                check()
            except AssertionError:
                failed.append(check.__name__)
    finally:
        oracle._lib = saved
    assert failed, f"mutant {name} passed every pin"
    assert os.path.exists(lib)
