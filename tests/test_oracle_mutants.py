"""Planted mistakes: each builds a copy of the oracle with one plausible error
(a wrong sign, index, operand or dropped term) and checks that some pin fails.
This is what makes the pins worth trusting: none of these errors slips by."""
import os

import pytest

import oracle
from tests import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "winattn_oracle.c")

MUTANTS = {
    "clockwise_rotation": [
        ("vec[2 * k] = x0 * cos(ay) - x1 * sin(ay);", "vec[2 * k] = x0 * cos(ay) + x1 * sin(ay);"),
        ("vec[2 * k + 1] = x0 * sin(ay) + x1 * cos(ay);", "vec[2 * k + 1] = -x0 * sin(ay) + x1 * cos(ay);"),
    ],
    "halves_swapped": [("double ay = i * th, ax = j * th;", "double ay = j * th, ax = i * th;")],
    "pair_members_swapped": [("double x0 = vec[2 * k], x1 = vec[2 * k + 1];",
                              "double x0 = vec[2 * k + 1], x1 = vec[2 * k];")],
    "mask_dropped": [("if (la != lc)", "if (0)")],
    "mask_inverted": [("if (la != lc)", "if (la == lc && a != c)")],
    "label_off_by_one": [("yr >= p->Hp - p->shift", "yr > p->Hp - p->shift")],
    "scale_dropped": [("const double scale = 1.0 / sqrt((double)d);", "const double scale = 1.0;")],
    "roll_reversed": [
        ("int y = (yr + p->shift) % p->Hp;", "int y = (yr - p->shift + p->Hp) % p->Hp;"),
        ("int x = (xr + p->shift) % p->Wp;", "int x = (xr - p->shift + p->Wp) % p->Wp;"),
    ],
    "scores_transposed": [("dot += w->q[(size_t)a * d + e] * w->k[(size_t)c * d + e];",
                           "dot += w->q[(size_t)c * d + e] * w->k[(size_t)a * d + e];")],
    "sum_not_divided": [("row[c] /= sum;", "row[c] /= 1.0;")],
    "value_index": [("acc += w->s[(size_t)a * N + c] * w->v[(size_t)c * d + e];",
                     "acc += w->s[(size_t)a * N + c] * w->v[(size_t)a * d + e];")],
    "bias_sides_swapped": [
        ("size_t ub = (((size_t)h * 2 + 0) * N + a) * r;", "size_t ub = (((size_t)h * 2 + 1) * N + a) * r;"),
        ("size_t wb = (((size_t)h * 2 + 1) * N + c) * r;", "size_t wb = (((size_t)h * 2 + 0) * N + c) * r;"),
    ],
    "bias_scaled": [("sc += bd;", "sc += scale * bd;")],
    "bias_dropped": [("sc += bd;", "sc += 0.0 * bd;")],
    "scatter_unrolled": [(
        "int64_t off = rolled_token_offset(p, b, wy * p->M + i, wx * p->M + j, h);\n                    if",
        "int64_t off = rolled_token_offset(p, b, (wy * p->M + i + p->Hp - p->shift) % p->Hp, "
        "(wx * p->M + j + p->Wp - p->shift) % p->Wp, h);\n                    if")],
    # padding (maps that are not multiples of M)
    "pad_keys_attended": [("            if (w->off[c] < 0)\n                w->s[(size_t)a * N + c] = -INFINITY;",
                           "            if (0)\n                w->s[(size_t)a * N + c] = -INFINITY;")],
    "lse_without_max": [("w->lse[a] = mx + log(sum);", "w->lse[a] = log(sum);")],
    "linear_without_relu": [("kq[t * d + c] = qr > 0.0 ? qr : 0.0;", "kq[t * d + c] = qr;")],
    "residual_sign_flipped": [("dst[e] += o[a * d + e] - (den > 0.0 ? num[e] / den : 0.0);",
                               "dst[e] += o[a * d + e] + (den > 0.0 ? num[e] / den : 0.0);")],
    "linear_mask_dropped": [("if (w.off[c] < 0 || wrap_label(&p, wy * M + (int)c / M, wx * M + (int)c % M) != la)",
                             "if (w.off[c] < 0)")],
    "rib_axes_swapped": [("f[k] = sin(w * cy);", "f[k] = sin(w * cx);"),
                         ("f[8 + k] = cos(w * cy);", "f[8 + k] = cos(w * cx);")],
    "rib_octave_off_by_one": [("const double w = ldexp(acos(-1.0), k);", "const double w = ldexp(acos(-1.0), k + 1);")],
    "rib_no_tanh": [("hid[c] = tanh(acc);", "hid[c] = acc;")],
    "cla_convolution_flipped": [("acc += dw[ch * 9 + (dy + 1) * 3 + (dx + 1)] *",
                                 "acc += dw[ch * 9 + (1 - dy) * 3 + (1 - dx)] *")],
    "cla_pointwise_transposed": [("acc += pw[(size_t)co * C + ci] * y[ci];", "acc += pw[(size_t)ci * C + co] * y[ci];")],
    "roll_over_unpadded_map": [
        ("int y = (yr + p->shift) % p->Hp;", "int y = (yr + p->shift) % p->H;"),
        ("int x = (xr + p->shift) % p->Wp;", "int x = (xr + p->shift) % p->W;"),
    ],
    "query_coords_global": [(
        "rope_rotate(w->q + (size_t)t * d, d, (double)i, (double)j, th);",
        "rope_rotate(w->q + (size_t)t * d, d, (double)(i + wy * M), (double)j, th);")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    with open(SRC) as f:
        src = f.read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
        src = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    lib = oracle.build(str(path), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(oracle.load(lib))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name!r} passed every pin"
