"""Plants plausible mistakes in copies of the CPU oracle and checks that the
pins catch every one of them (each mutant must fail at least one pin).

The mutants are built from a textual edit of the committed oracle source
into a temporary directory; the committed oracle is never modified.
"""
import os
import shutil

import pytest

import oracle
from oracle import build as obuild
import oracle_pins

SRC = obuild.SOURCE

# (name, exact text in the oracle, replacement, count of occurrences to edit)
MUTANTS = [
    ("swap_dx_dy", "orc_position(p, ho, wo, i, j, t[3 * k], t[3 * k + 1], &x, &y);\n"
                   "                            orc_splat_sample",
     "orc_position(p, ho, wo, i, j, t[3 * k + 1], t[3 * k], &x, &y);\n"
     "                            orc_splat_sample", 1),
    ("drop_corner_11", "if (yy < 0 || yy >= H || xx < 0 || xx >= W)",
     "if ((a && b) || yy < 0 || yy >= H || xx < 0 || xx >= W)", 1),
    ("swap_lx_weights", "double wx = b ? lx : 1.0 - lx;\n            const float",
     "double wx = b ? 1.0 - lx : lx;\n            const float", 1),
    ("transpose_taps", "int k = i * p->kw + j;\n                            float x, y;\n"
                       "                            orc_position(p, ho, wo, i, j, t[3 * k], t[3 * k + 1], &x, &y);\n"
                       "                            orc_splat_sample(input + (size_t)n * img, p->H, p->W, p->C,\n"
                       "                                             g * D, D, x, y, wk[k], o);",
     "int k = j * p->kh + i;\n                            float x, y;\n"
     "                            orc_position(p, ho, wo, i, j, t[3 * k], t[3 * k + 1], &x, &y);\n"
     "                            orc_splat_sample(input + (size_t)n * img, p->H, p->W, p->C,\n"
     "                                             g * D, D, x, y, wk[k], o);", 1),
    ("ignore_offset_scale", "float tx = dx * p->offset_scale;", "float tx = dx;", 1),
    ("stride_ignored", "float bx = (float)(wo * p->sw - p->pw + j * p->dw);",
     "float bx = (float)(wo - p->pw + j * p->dw);", 1),
    ("dilation_ignored", "float by = (float)(ho * p->sh - p->ph + i * p->dh);",
     "float by = (float)(ho * p->sh - p->ph + i);", 1),
    ("pad_sign", "float bx = (float)(wo * p->sw - p->pw + j * p->dw);",
     "float bx = (float)(wo * p->sw + p->pw + j * p->dw);", 1),
    ("left_edge_closed", "if (!(x > -1.0f && x < (float)W", "if (!(x > 0.0f && x < (float)W", 1),
    ("grad_dx_sign", "gx += (b ? wy : -wy) * dot;", "gx += (b ? -wy : wy) * dot;", 1),
    ("grad_dy_uses_wy", "gy += (a ? wx : -wx) * dot;", "gy += (a ? wy : -wy) * dot;", 1),
    ("grad_m_unweighted", "gm += wy * wx * dot;", "gm += dot;", 1),
    ("grad_in_wrong_weight", "gin_n[at + d] += m * (wy * wx) * (double)go[d];",
     "gin_n[at + d] += m * (wy * (1.0 - wx)) * (double)go[d];", 1),
    ("grad_offset_scale_missing", "gt[3 * k] = (double)p->offset_scale * m * gx;",
     "gt[3 * k] = m * gx;", 1),
    ("softplus_no_relu", "float sp = fmaxf(raw, 0.0f) + log1pf(expf(-fabsf(raw)));",
     "float sp = log1pf(expf(-fabsf(raw)));", 1),
    ("clamp_from_below", "if (s > smax)\n        s = smax;", "if (s < smax)\n        s = smax;", 1),
    ("msdcn_scale_per_group_ignored", "float s = orc_msdcn_scale(scale_raw[pix * p->G + g], s0[g], smax);",
     "float s = orc_msdcn_scale(scale_raw[pix * p->G + g], s0[0], smax);", 1),
    ("msdcn_grad_dir_missing_s", "gt[3 * k] = gdx == 0.0 ? 0.0 : (double)s * gdx;",
     "gt[3 * k] = gdx;", 1),
    ("msdcn_nan_scale_dir_grad_unguarded", "gt[3 * k] = gdx == 0.0 ? 0.0 : (double)s * gdx;",
     "gt[3 * k] = (double)s * gdx;", 1),
    ("msdcn_sigmoid_sign", "return (double)s0 / (1.0 + exp(-(double)raw));",
     "return (double)s0 / (1.0 + exp((double)raw));", 1),
    ("msdcn_clamp_gradient_kept", "if (!(u <= smax))\n        return 0.0;",
     "if (isnan(u))\n        return 0.0;", 1),
    ("msdcn_grad_raw_dirs_swapped",
     "*tx = (double)dirx * (double)p->offset_scale;\n        *ty = (double)diry * (double)p->offset_scale;",
     "*tx = (double)diry * (double)p->offset_scale;\n        *ty = (double)dirx * (double)p->offset_scale;", 1),
    ("msdcn_bwd_unscaled_offsets",
     "orc_position_ms(p, ho, wo, i, j, s, t[3 * k], t[3 * k + 1], &x, &y,\n"
     "                                            &tx, &ty);\n                            double m",
     "orc_position_ms(p, ho, wo, i, j, 1.0f, t[3 * k], t[3 * k + 1], &x, &y,\n"
     "                                            &tx, &ty);\n                            double m", 1),
    ("softmax_no_max_shift", "w[k] = exp((double)t[3 * k + 2] - mx);", "w[k] = exp((double)t[3 * k + 2]);", 1),
    ("softmax_unnormalised", "        w[k] /= sum;", "        w[k] /= 9.0;", 1),
    ("softmax_grad_missing_sum", "dotw += wk[k] * gwk[k];", "dotw += 0.0 * gwk[k];", 1),
    ("softmax_grad_input_raw_logit", "double m = wk[k];", "double m = (double)t[3 * k + 2];", 1),
    ("dilation_centre_off", "float cx = (float)(wo * p->sw - p->pw) + 0.5f * (float)((p->kw - 1) * p->dw);",
     "float cx = (float)(wo * p->sw - p->pw);", 1),
    ("dilation_grid_unscaled", "*x = cx + sx;", "*x = cx + kx + s * ox;", 1),
    ("dilation_ds_missing_grid", "*tx = (double)ux;", "*tx = (double)ox;", 1),
    ("producer_dw_bias_dropped", "double acc = dw_b[c];", "double acc = 0.0;", 1),
    ("producer_lin_bias_dropped", "double acc = lin_b[j];", "double acc = 0.0;", 1),
    ("producer_lin_transposed", "(double)lin_w[(size_t)j * C + c]", "(double)lin_w[(size_t)c * J + j]", 1),
    ("producer_taps_transposed", "dw_w[(i * 3 + j) * C + c]", "dw_w[(j * 3 + i) * C + c]", 1),
    ("producer_pad_shift", "const int yy = y + i - 1, xs = xx + j - 1;",
     "const int yy = y + i - 1, xs = xx + j;", 1),
    ("flops_factor", "return 4.0 * p->kh * p->kw * (double)p->N * Ho * Wo * p->C;",
     "return 2.0 * p->kh * p->kw * (double)p->N * Ho * Wo * p->C;", 1),
    ("ideal_offsets_per_channel", "double ow = 3.0 * p->kh * p->kw * (double)p->N * Ho * Wo * p->G;",
     "double ow = 3.0 * p->kh * p->kw * (double)p->N * Ho * Wo * p->C;", 1),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(mutant_dir, name, old, new, count):
    src = open(SRC).read()
    assert src.count(old) >= count, f"mutation site for {name} not found"
    mutated = src.replace(old, new, count)
    assert mutated != src
    path = os.path.join(str(mutant_dir), f"{name}.c")
    with open(path, "w") as f:
        f.write(mutated)
    lib = obuild.build(source=path, output=path[:-2] + ".so", force=True)
    o = oracle.Oracle(lib)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} survived every pin"


def test_gcc_available():
    assert shutil.which("gcc"), "gcc builds the oracle"
