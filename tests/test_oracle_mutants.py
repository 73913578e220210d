"""Plants plausible mistakes in copies of the oracle source (on the CPU) and checks that at
least one pin catches each of them, so the pins are strong enough to trust the oracle."""
import os

import pytest

import oracle
import oracle_pins

# (name, original text, mistaken text): each replaces exactly one span of the source.
MUTANTS = [
    ("window_upper_bound", "for (int32_t dy = -(kh / 2); dy <= (kh - 1) / 2; ++dy)\n        for (int32_t dx = -(kw / 2); dx <= (kw - 1) / 2; ++dx) {\n          const int32_t y = cy + dy, x = cx + dx;\n          if (y < 0 || y >= H || x < 0 || x >= W) continue; /* out",
     "for (int32_t dy = -((kh - 1) / 2); dy <= kh / 2; ++dy)\n        for (int32_t dx = -((kw - 1) / 2); dx <= kw / 2; ++dx) {\n          const int32_t y = cy + dy, x = cx + dx;\n          if (y < 0 || y >= H || x < 0 || x >= W) continue; /* out"),
    ("xnor_weight_sign", "return bin_pm1(xt) * (wbit ? 1.0 : -1.0);", "return bin_pm1(xt) * (wbit ? -1.0 : 1.0);"),
    ("sign_of_zero", "static double bin_pm1(double xt) { return ((float)xt < 0.0f)",
     "static double bin_pm1(double xt) { return ((float)xt <= 0.0f)"),
    ("and_polarity", "return bin_01(xt) * (wbit ? 1.0 : 0.0);", "return (1.0 - bin_01(xt)) * (wbit ? 1.0 : 0.0);"),
    ("bw_weight_map", "return xt * (wbit ? 1.0 : -1.0);", "return xt * (wbit ? 1.0 : 0.0);"),
    ("input_terms_order", "return s * x + b;", "return s * (x + b);"),
    ("channel_mean_divisor", "return acc / (double)ni;", "return acc / (double)(ni + 1);"),
    ("beta_divides_by_valid_taps",
     "double acc = 0.0;\n      for (int32_t dy = -(kh / 2); dy <= (kh - 1) / 2; ++dy)\n        for (int32_t dx = -(kw / 2); dx <= (kw - 1) / 2; ++dx) {\n          const int32_t y = cy + dy, x = cx + dx;\n          if (y < 0 || y >= H || x < 0 || x >= W) continue;\n          acc += channel_mean_abs(in, in_scale, in_bias, ((int64_t)n * H + y) * W + x, Ni);\n        }\n      beta = acc / ((double)kh * (double)kw);",
     "double acc = 0.0; int nv = 0;\n      for (int32_t dy = -(kh / 2); dy <= (kh - 1) / 2; ++dy)\n        for (int32_t dx = -(kw / 2); dx <= (kw - 1) / 2; ++dx) {\n          const int32_t y = cy + dy, x = cx + dx;\n          if (y < 0 || y >= H || x < 0 || x >= W) continue;\n          ++nv; acc += channel_mean_abs(in, in_scale, in_bias, ((int64_t)n * H + y) * W + x, Ni);\n        }\n      beta = acc / (double)nv;"),
    ("beta_divides_by_valid_taps_2", "beta = acc / ((double)kh * (double)kw);", "beta = acc / ((double)kh * (double)kw - 1.0);"),
    ("weight_axes_transposed", "(((int64_t)c * kh + ky) * kw + kx) * Ni", "(((int64_t)c * kw + kx) * kh + ky) * Ni"),
    ("bias_before_scale", "double yv = acc * (double)scale[c] * beta + (double)bias[c];\n      if (d->relu",
     "double yv = (acc + (double)bias[c]) * (double)scale[c] * beta;\n      if (d->relu"),
    ("scale_index", "double yv = acc * (double)scale[c] * beta + (double)bias[c];\n      if (d->relu",
     "double yv = acc * (double)scale[0] * beta + (double)bias[c];\n      if (d->relu"),
    ("stride_centre", "const int32_t cy = oy * d->stride_y, cx = ox * d->stride_x;",
     "const int32_t cy = oy * d->stride_y + d->stride_y / 2, cx = ox * d->stride_x + d->stride_x / 2;"),
    ("relu_before_bias", "      if (d->relu && yv < 0.0) yv = 0.0;\n      if (y_out)",
     "      if (d->relu && yv < (double)bias[c]) yv = (double)bias[c];\n      if (y_out)"),
    ("fc_beta_divisor", "beta = acc / ((double)H * (double)W);", "beta = acc / ((double)H * (double)H);"),
    ("fc_weight_flatten", "const uint8_t* wrow = wbits + (int64_t)c * K;\n      double acc = 0.0;\n      for (int64_t k = 0; k < K; ++k) {\n        const int32_t f = (int32_t)(k % Ni);\n        acc += op_term(type, transformed_input(img, in_scale, in_bias, k / Ni, Ni, f), wrow[k]);",
     "const uint8_t* wrow = wbits + (int64_t)c * K;\n      double acc = 0.0;\n      for (int64_t k = 0; k < K; ++k) {\n        const int32_t f = (int32_t)(k % Ni);\n        acc += op_term(type, transformed_input(img, in_scale, in_bias, k / Ni, Ni, f), wrow[(k % Ni) * (K / Ni) + k / Ni]);"),
    ("binarize_polarity", "if (bits) bits[p * C + c] = (uint8_t)bin_01(v);",
     "if (bits) bits[p * C + c] = (uint8_t)(1.0 - bin_01(v));"),
    ("binarize_sign_in_double", "if (bits) bits[p * C + c] = (uint8_t)bin_01(v);",
     "if (bits) bits[p * C + c] = (uint8_t)(v < 0.0 ? 0 : 1);"),
    ("binarize_without_terms", "const double v = transformed_input(x, in_scale, in_bias, p, C, c);",
     "const double v = transformed_input(x, NULL, NULL, p, C, c);"),
    ("binarize_A_of_first_pixel", "if (A) A[p] = channel_mean_abs(x, in_scale, in_bias, p, C);",
     "if (A) A[p] = channel_mean_abs(x, in_scale, in_bias, 0, C);"),
]


@pytest.mark.parametrize("name,orig,mutated", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, orig, mutated, tmp_path):
    with open(oracle.SOURCE_PATH) as f:
        src = f.read()
    assert src.count(orig) >= 1, f"mutant {name}: original text not found"
    lib = oracle.compile_source(src.replace(orig, mutated, 1), os.path.join(tmp_path, f"lib_{name}.so"))
    variant = oracle.Variant(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(variant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
