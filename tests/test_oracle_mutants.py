"""Planted mistakes in a copy of the oracle must each fail at least one pin.

Each mutant is the oracle's C source with one plausible slip substituted (a
clamped border, swapped dy/dx channels, a dropped bias or mask, a flipped sign,
transposed kernel taps, a wrong group, a wrong derivative sign...). The copy is
compiled into a temporary library and run through the pins of
``oracle_pins.py``; a mutant that passes every pin would mean the pins cannot
see that kind of error. The oracle's own source is never modified.
"""
import os

import pytest

import oracle
import oracle_pins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "dcn_oracle.c")).read()

MUTANTS = {
    "clamp_border": ("if (r < 0 || r >= s->H || q < 0 || q >= s->W) return 0.0;",
                     "if (r < 0) r = 0; if (r >= s->H) r = s->H - 1; if (q < 0) q = 0; if (q >= s->W) q = s->W - 1;"),
    "swap_dy_dx": ("g * 2 * K2 + 2 * k) * plane + pix];\n    double dx",
                   "g * 2 * K2 + 2 * k + 1) * plane + pix];\n    double dx"),
    "drop_bias": ("yrow[o] = bias ? bias[o] : 0.0;", "yrow[o] = 0.0;"),
    "drop_mask": ("double v = m * bilinear(x, s, b, c, py, px);", "double v = bilinear(x, s, b, c, py, px);"),
    "pad_sign": ("*py = (double)(ho * s->stride - s->pad + i * s->dil) + dy;",
                 "*py = (double)(ho * s->stride + s->pad + i * s->dil) + dy;"),
    "transposed_taps": ("return (((size_t)o * s->K + i) * s->K + j) * s->Cin + c;",
                        "return (((size_t)o * s->K + j) * s->K + i) * s->Cin + c;"),
    "group_zero_offsets": ("double dy = off[((size_t)b * 2 * s->G * K2 + (size_t)g * 2 * K2",
                           "double dy = off[((size_t)b * 2 * s->G * K2 + (size_t)0 * 2 * K2"),
    "round_not_floor": ("double y0 = floor(py), x0 = floor(px);\n    double v = 0.0;",
                        "double y0 = trunc(py), x0 = trunc(px);\n    double v = 0.0;"),
    "dpy_sign": ("*dpy = (1.0 - lx) * (v10 - v00) + lx * (v11 - v01);",
                 "*dpy = (1.0 - lx) * (v00 - v10) + lx * (v11 - v01);"),
    "dpx_weights_swapped": ("*dpx = (1.0 - ly) * (v01 - v00) + ly * (v11 - v10);",
                            "*dpx = ly * (v01 - v00) + (1.0 - ly) * (v11 - v10);"),
    "grad_x_missing_mask": ("+= gcol * m * gq;", "+= gcol * gq;"),
    "grad_weight_missing_mask": ("gwb[weight_index(s, o, i, j, c)] += gyrow[o] * m * v;",
                                 "gwb[weight_index(s, o, i, j, c)] += gyrow[o] * v;"),
    "grad_mask_times_mask": ("gm += gcol * v;", "gm += gcol * m * v;"),
    "column_grad_transposed": ("acc += gyrow[o] * w[weight_index(s, o, i, j, c)];",
                               "acc += gyrow[o] * w[weight_index(s, o, j, i, c)];"),
    "stride_ignored_in_x": ("*px = (double)(wo * s->stride - s->pad + j * s->dil) + dx;",
                            "*px = (double)(wo - s->pad + j * s->dil) + dx;"),
    "dilation_ignored": ("*py = (double)(ho * s->stride - s->pad + i * s->dil) + dy;",
                         "*py = (double)(ho * s->stride - s->pad + i) + dy;"),
    "predictor_sigmoid_sign": ("= 1.0 / (1.0 + exp(-acc));", "= 1.0 / (1.0 + exp(acc));"),
    "predictor_mask_not_squashed": ("= 1.0 / (1.0 + exp(-acc));", "= acc;"),
    "predictor_dilation_ignored_in_x": ("wo * s->stride - s->pad + j * s->dil, c);",
                                        "wo * s->stride - s->pad + j, c);"),
    "droi_offset_not_scaled_by_roi": ("gamma * off[(size_t)r * 2 * kk + 2 * t] * h : 0.0;",
                                      "gamma * off[(size_t)r * 2 * kk + 2 * t] : 0.0;"),
    "droi_swap_dy_dx": ("const double dy = off ? gamma * off[(size_t)r * 2 * kk + 2 * t] * h : 0.0;",
                        "const double dy = off ? gamma * off[(size_t)r * 2 * kk + 2 * t + 1] * h : 0.0;"),
    "droi_mean_over_rows_only": ("yb[c] = n > 0 ? m * acc / n : 0.0;", "yb[c] = n > 0 ? m * acc / (u1 - u0) : 0.0;"),
    "droi_corner_x_for_y": ("acc += bilinear(x, s, b, c, roi[2] + u + dy, roi[1] + v + dx);",
                            "acc += bilinear(x, s, b, c, roi[1] + u + dy, roi[1] + v + dx);"),
    "droi_grad_x_missing_mask": ("gx[(((size_t)b * s->H + rr) * s->W + qq) * C + c] += g * m * wt;",
                                 "gx[(((size_t)b * s->H + rr) * s->W + qq) * C + c] += g * wt;"),
    "droi_grad_offset_missing_width": ("goff[(size_t)r * 2 * kk + 2 * t + 1] = g_dx * gamma * w;",
                                       "goff[(size_t)r * 2 * kk + 2 * t + 1] = g_dx * gamma;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, "mutation site not found: %s" % name
    src = tmp_path / ("oracle_%s.c" % name)
    src.write_text(SRC.replace(old, new, 1))
    lib = oracle.load(oracle.build(force=True, src=str(src), out=str(tmp_path / ("lib_%s.so" % name))))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "mutant %s passed every pin" % name
