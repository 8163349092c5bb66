"""The oracle's pins catch plausible mistakes (CPU only).

Each case copies the oracle source, plants one mistake (a swapped operand, a
dropped term, a wrong sign or index), builds the copy and runs the pin suite
against it in a subprocess: the suite must fail.  Nothing here touches a GPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dcn4_ref.cpp")

MUTATIONS = {
    "dx_dy_swapped": ("const double dx = load(offset_mask, p->dtype, om + 2 * k);\n                        const double dy = load(offset_mask, p->dtype, om + 2 * k + 1);\n                        const double m = a[k];\n                        double h, w;\n                        sample_location(p, ho, wo, cells[k], dx, dy, &h, &w);\n                        const Bilinear b = bilinear_cell(p, h, w);\n                        y +=",
                      "const double dy = load(offset_mask, p->dtype, om + 2 * k);\n                        const double dx = load(offset_mask, p->dtype, om + 2 * k + 1);\n                        const double m = a[k];\n                        double h, w;\n                        sample_location(p, ho, wo, cells[k], dx, dy, &h, &w);\n                        const Bilinear b = bilinear_cell(p, h, w);\n                        y +="),
    "k_order_row_major": ("for (int iw = 0; iw < p->kw; ++iw) {\n        for (int ih = 0; ih < p->kh; ++ih) {",
                          "for (int ih = 0; ih < p->kh; ++ih) {\n        for (int iw = 0; iw < p->kw; ++iw) {"),
    "corner_dropped": ("for (int bb = 0; bb < 2; ++bb) {\n            const int y = b.h0 + a;",
                       "for (int bb = 0; bb < 1; ++bb) {\n            const int y = b.h0 + a;"),
    "weights_transposed": ("const double wt = (a ? b.lh : 1.0 - b.lh) * (bb ? b.lw : 1.0 - b.lw);",
                           "const double wt = (a ? b.lw : 1.0 - b.lw) * (bb ? b.lh : 1.0 - b.lh);"),
    "scale_on_grid_too": ("*h = static_cast<double>(base_h) + p->offset_scale * dy;",
                          "*h = p->offset_scale * (static_cast<double>(base_h) + dy);"),
    "dSdh_sign": ("(1 - b.lw) * (v[1][0] - v[0][0])", "(1 - b.lw) * (v[0][0] - v[1][0])"),
    "grad_offset_without_mask": ("= s * m * gdw;", "= s * gdw;"),
    "grad_value_without_mask": ("+= m * wt * gy;", "+= wt * gy;"),
    "stride_ignored": ("const int base_w = wo * p->sw - p->pw + c.iw * p->dw;",
                       "const int base_w = wo - p->pw + c.iw * p->dw;"),
    "location_two_roundings": ("*h = static_cast<double>(std::fmaf(s, static_cast<float>(dy), static_cast<float>(base_h)));",
                               "*h = static_cast<double>(static_cast<float>(s * static_cast<float>(dy)) + static_cast<float>(base_h));"),
    # single-scale deformable attention
    "attn_softmax_not_normalised": ("for (int k = 0; k < p->K; ++k) a[k] /= sum;", ""),
    "attn_dx_dy_swapped": ("*h = static_cast<double>(ry) + p->offset_scale * dy;\n        *w = static_cast<double>(rx) + p->offset_scale * dx;",
                           "*h = static_cast<double>(ry) + p->offset_scale * dx;\n        *w = static_cast<double>(rx) + p->offset_scale * dy;"),
    "attn_jacobian_without_sum": ("= a[k] * (gw[k] - dot);", "= a[k] * gw[k];"),
    "attn_offset_grad_without_weight": ("= s * a[k] * gdw;", "= s * gdw;"),
    "attn_corner_row_swapped": ("v[a2][b2] = attn_pixel(p, value, n, h0 + a2, w0 + b2, g, c);",
                                "v[a2][b2] = attn_pixel(p, value, n, h0 + 1 - a2, w0 + b2, g, c);"),
    "bilinear_ceil_cell": ("const double fh = std::floor(h);", "const double fh = std::ceil(h) - 1.0;"),
    # softmax variant
    "softmax_not_normalised": ("for (int k = 0; k < K; ++k) a[k] /= sum;", ""),
    "softmax_largest_not_subtracted": ("a[k] = std::exp(a[k] - mx);", "a[k] = std::exp(a[k]);"),
    "softmax_jacobian_without_sum": ("p->softmax ? a[k] * (gw[k] - dot) : gw[k]", "p->softmax ? a[k] * gw[k] : gw[k]"),
    # storage rounding and the offset/mask linear layer
    "encode_f16_truncates": ("double q = std::nearbyint(std::ldexp(a, 10 - E));", "double q = std::floor(std::ldexp(a, 10 - E));"),
    "encode_bf16_ties_away": ("double q = std::nearbyint(std::ldexp(a, 7 - E));", "double q = std::round(std::ldexp(a, 7 - E));"),
    "encode_f16_subnormal_unit": ("std::nearbyint(std::ldexp(a, 24));", "std::nearbyint(std::ldexp(a, 25));"),
    "linear_drops_bias": ("if (bias) acc += load(bias, dtype, j);", ""),
    "linear_weight_transposed": ("load(weight, dtype, static_cast<int64_t>(j) * Cin + c)",
                                 "load(weight, dtype, static_cast<int64_t>(c % Cout) * Cin + (j % Cin))"),
    "linear_bwd_weight_transposed": ("load(g, dtype, m * Cout + j) * load(weight, dtype, static_cast<int64_t>(j) * Cin + c)",
                                     "load(g, dtype, m * Cout + j) * load(weight, dtype, static_cast<int64_t>(c % Cout) * Cin + (j % Cin))"),
    "linear_bwd_x_row_shifted": ("acc[c] += gj * load(x, dtype, m * Cin + c);",
                                 "acc[c] += gj * load(x, dtype, ((m + 1) % M) * Cin + c);"),
    "linear_bwd_bias_skips_first_row": ("bsum += gj;", "if (m > 0) bsum += gj;"),
    "softmax_ignored_in_backward_offsets": ("const double m = a[k];\n                        double h, w;\n                        sample_location(p, ho, wo, cells[k], dx, dy, &h, &w);\n                        const Bilinear b = bilinear_cell(p, h, w);\n                        if (!b.any) continue;",
                                            "const double m = load(offset_mask, p->dtype, om + 2 * K + k);\n                        double h, w;\n                        sample_location(p, ho, wo, cells[k], dx, dy, &h, &w);\n                        const Bilinear b = bilinear_cell(p, h, w);\n                        if (!b.any) continue;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation {name} no longer applies"
    mutated = src.replace(old, new)
    cpp = tmp_path / "dcn4_ref.cpp"
    cpp.write_text(mutated)
    (tmp_path / "dcn4_ref.h").write_text(open(os.path.join(ROOT, "oracle", "dcn4_ref.h")).read())
    lib = tmp_path / "liboracle.so"
    subprocess.run(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-pthread", "-fPIC", "-shared",
                    "-o", str(lib), str(cpp)], check=True)
    env = dict(os.environ, DCN4_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"
