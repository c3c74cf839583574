"""Planted mistakes in the oracle are caught by its pins.

Each case copies the oracle (its C source and Python wrapper), the pin tests with their golden
files, and the seeded input generators into a scratch directory. It then plants ONE plausible
mistake in the copy with a single textual edit: a wrong sign, a dropped term or stage, a wrong
index, constant, clamp or tie rule, a transposed or swapped operand, or a skipped rounding. The
copy is built there and the pin tests run against it; at least one pin must fail. The
repository's own oracle is never modified.

An unmodified copy ("control") must pass, so a failure is the planted mistake and not the
harness. Every planted edit keeps each access inside its buffer: a mutant is caught by a pin's
assertion (pytest exit status 1), never by a crash.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
C = "oracle/sq_oracle.c"
PY = "oracle/__init__.py"
PIN_FILES = ["tests/test_oracle_pins.py", "tests/test_oracle_pins_g64.py",
             "tests/test_oracle_pins_int8.py", "tests/test_oracle_pins_svd.py"]

# id -> (file, text, replacement, which occurrence of text)
MUTANTS = {
    # rotation ("Rotation": block-diagonal normalised Hadamard-256)
    "fwht_butterfly_sign": (C, "v[j + h] = a - b;", "v[j + h] = b - a;", 0),
    "fwht_scale": (C, "v[j] = v[j] * 0.0625f;", "v[j] = v[j] * 0.125f;", 0),
    "fwht_drops_last_stage": (C, "for (int h = 1; h < 256; h <<= 1)", "for (int h = 1; h < 128; h <<= 1)", 0),
    # narrowing conversions
    "round_ties_away": (C, "return nearbyint(a / spacing) * spacing;",
                        "return floor(a / spacing + 0.5) * spacing;", 0),
    "bf16_fraction_bits": (C, "round_to_grid(fabs((double)v), 7, -126)", "round_to_grid(fabs((double)v), 8, -126)", 0),
    "f16_overflow_edge": (C, "if (r > 65504.0)", "if (r >= 65504.0)", 0),
    "ue4m3_saturation": (C, "if (r > 448.0)\n        r = 448.0;", "if (r > 480.0)\n        r = 480.0;", 0),
    "ue4m3_subnormal_quantum": (C, "return (uint8_t)(r / ldexp(1.0, -9));", "return (uint8_t)(r / ldexp(1.0, -10));", 0),
    "e2m1_saturation": (C, "if (r > 6.0)\n        r = 6.0;", "if (r > 4.0)\n        r = 4.0;", 0),
    "e2m1_drops_sign": (C, "return (uint8_t)(sign | c);", "return (uint8_t)(c);", 0),
    # int4 group-32 codec ("Residual codecs": MSE-swept fractions)
    "int4_fraction_grid": (C, "return (float)(50 + 2 * j) / 100.0f;", "return (float)(52 + 2 * j) / 100.0f;", 0),
    "int4_divisor": (C, "float s7 = fa / 7.0f;", "float s7 = fa / 8.0f;", 0),
    "int4_clamp": (C, "if (rq > 7.0f)\n                    rq = 7.0f;", "if (rq > 8.0f)\n                    rq = 8.0f;", 0),
    "int4_tie_rule": (C, "if (best_j < 0 || mse < best) {", "if (best_j < 0 || mse <= best) {", 0),
    "int4_error_sum_drops_stage": (C, "for (int d = 16; d >= 1; d >>= 1) {", "for (int d = 16; d >= 2; d >>= 1) {", 0),
    "int4_unrounded_scale": (C, "float s = or_f16_to_f32(sh);", "float s = s7;", 0),
    "int4_zero_scale_error": (C, "p[i] = r[i] * r[i];", "p[i] = 0.0f;", 0),
    "int4_nibble_order": (C, "codes[n * (K / 2) + (b + 32 * g + i) / 2] = (uint8_t)(lo | (hi << 4));",
                          "codes[n * (K / 2) + (b + 32 * g + i) / 2] = (uint8_t)(hi | (lo << 4));", 0),
    # int4 group-64 variant
    "g64_drops_second_half": (C, "float mse = half[0] + half[1];", "float mse = half[0];", 0),
    "g64_divisor": (C, "float s7 = fa / 7.0f;", "float s7 = fa / 8.0f;", 1),
    "g64_tie_rule": (C, "if (best_j < 0 || mse < best) {", "if (best_j < 0 || mse <= best) {", 1),
    # NVFP4 codec and the tiled scale layout
    "sf_layout_line_word_swap": (C, "(r % 32) * 16 + ((r % 128) / 32) * 4", "(r % 32) * 4 + ((r % 128) / 32) * 16", 0),
    "nvfp4_global_divisor": (C, "return A / 2688.0f;", "return A / 3072.0f;", 0),
    "nvfp4_six_g": (C, "float sixg = 6.0f * g;", "float sixg = 4.0f * g;", 0),
    "nvfp4_den_drops_g": (C, "float den = dec * g;", "float den = dec;", 0),
    "nvfp4_block_amax_half": (C, "for (int i = 0; i < 16; i++) {\n        float m = fabsf(r[i]);\n        if (m > b)",
                              "for (int i = 0; i < 8; i++) {\n        float m = fabsf(r[i]);\n        if (m > b)", 0),
    "nvfp4_nibble_order": (C, "codes8[i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));",
                           "codes8[i] = (uint8_t)(c[2 * i + 1] | (c[2 * i] << 4));", 0),
    # activation quant and the low-rank input
    "act_t_transposed_down": (C, "(double)or_bf16_to_f32(lora_down[k * 32 + rr]);",
                              "(double)or_bf16_to_f32(lora_down[rr * K + k]);", 0),
    "act_static_scale_ignored": (C, "if (!static_g)", "if (1)", 0),
    # forwards
    "fwd_nvfp4_drops_g_w": (C, "double out = (double)g_x * (double)g_w * acc;", "double out = (double)g_x * acc;", 0),
    "fwd_nvfp4_lora_index": (C, "out += t[m * 32 + r] * (double)or_bf16_to_f32(U[n * 32 + r]);",
                             "out += t[m * 32 + r] * (double)or_bf16_to_f32(U[n * 32 + (31 - r)]);", 0),
    "fwd_nvfp4_sf_column": (C, "(double)or_ue4m3_to_f32(wsf[or_sf_offset(n, k / 16, C)]);",
                            "(double)or_ue4m3_to_f32(wsf[or_sf_offset(n, k / 32, C)]);", 0),
    "fwd_int4_sign_extend": (C, "int q = nib >= 8 ? nib - 16 : nib;", "int q = nib >= 8 ? nib - 8 : nib;", 0),
    "fwd_int4_unrounded_x": (C, "xb[i * K + k] = (double)or_bf16_to_f32(or_f32_to_bf16(xrot[rows[i] * K + k]));",
                             "xb[i * K + k] = (double)xrot[rows[i] * K + k];", 0),
    "fwd_int4_scale_group": (C, "float s = or_f16_to_f32(scales[n * (K / group) + k / group]);",
                             "float s = or_f16_to_f32(scales[n * (K / group) + k / 64]);", 0),
    "fwd_int4_drops_lora": (C, "acc += t[m * 32 + r] * (double)or_bf16_to_f32(U[n * 32 + r]);",
                            "acc += 0.0 * t[m * 32 + r] * (double)or_bf16_to_f32(U[n * 32 + r]);", 0),
    # int8 per-row codec, rank 16 ("v3.1 -- int8-residual mode")
    "int8_divisor": (C, "float s = fa / 127.0f;", "float s = fa / 128.0f;", 0),
    "int8_clamp": (C, "if (rq > 127.0f)\n                    rq = 127.0f;", "if (rq > 126.0f)\n                    rq = 126.0f;", 0),
    "int8_row_error_last_block": (C, "E = (b == 0) ? g[0] : E + g[0];", "E = g[0];", 0),
    "int8_tie_rule": (C, "if (best_j < 0 || E < best) {", "if (best_j < 0 || E <= best) {", 0),
    "int8_fwd_rank15": (C, "for (int r = 0; r < 16; r++)\n                    acc += t[m * 16 + r]",
                        "for (int r = 0; r < 15; r++)\n                    acc += t[m * 16 + r]", 0),
    "int8_fwd_unrounded_w": (C, "wb[k] = (double)or_bf16_to_f32(or_f32_to_bf16(d));\n        }\n        for (int64_t i = 0; i < n_rows; i++) {\n            int64_t m = rows[i];\n            double acc = 0.0;\n            for (int64_t k = 0; k < K; k++)\n                acc += xb[i * K + k] * wb[k];\n            if (t)\n                for (int r = 0; r < 16",
                             "wb[k] = (double)d;\n        }\n        for (int64_t i = 0; i < n_rows; i++) {\n            int64_t m = rows[i];\n            double acc = 0.0;\n            for (int64_t k = 0; k < K; k++)\n                acc += xb[i * K + k] * wb[k];\n            if (t)\n                for (int r = 0; r < 16", 0),
    # reconstruct
    "recon_nvfp4_drops_g_w": (C, "v[i] = ed * g_w;", "v[i] = ed;", 0),
    "recon_skips_inverse_rotation": (C, "            or_fwht256(v);\n            for (int i = 0; i < 256; i++) {\n                int64_t k = b + i;\n                float out = v[i];",
                                     "            for (int i = 0; i < 256; i++) {\n                int64_t k = b + i;\n                float out = v[i];", 0),
    "recon_lora_index": (C, "L = fmaf(or_bf16_to_f32(U[n * rank + r]), or_bf16_to_f32(D[k * rank + r]), L);",
                         "L = fmaf(or_bf16_to_f32(U[n * rank + r]), or_bf16_to_f32(D[k * rank + (rank - 1 - r)]), L);", 0),
    "recon_lora_sign": (C, "out = L + v[i];", "out = v[i] - L;", 0),
    "recon_int8_row_scale": (C, "((const float *)scales)[n];", "((const float *)scales)[0];", 0),
    "recon_int4_sign_extend": (C, "int q = nib >= 8 ? (int)nib - 16 : (int)nib;", "int q = (int)nib;", 0),
    # backward of the input
    "bwd_dy_column": (C, "double a = (double)or_bf16_to_f32(dy[rows[i] * N + n]);",
                      "double a = (double)or_bf16_to_f32(dy[rows[i] * N + (N - 1 - n)]);", 0),
    # decoders, rotation of whole rows, absmax and rounding inside the codecs
    "e2m1_decode_table": (C, "{0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};",
                          "{0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 5.0f};", 0),
    "ue4m3_decode_bias": (C, "return (float)ldexp(8.0 + m, e - 7 - 3);", "return (float)ldexp(8.0 + m, e - 8 - 3);", 0),
    "f16_decode_bias": (C, "v = ldexp(1024.0 + m, e - 15 - 10);", "v = ldexp(1024.0 + m, e - 14 - 10);", 0),
    "rotate_first_block_only": (C, "v[i] = in[r * K + b + i];", "v[i] = in[r * K + i];", 0),
    "int4_build_skips_rotation": (C, "            or_fwht256(v);\n            for (int g = 0; g < 8; g++) {",
                                  "            for (int g = 0; g < 8; g++) {", 0),
    "int4_scale_index": (C, "int64_t gi = n * (K / 32) + (b / 32) + g;", "int64_t gi = n * (K / 32) + g;", 0),
    "int4_amax_half": (C, "for (int i = 0; i < 32; i++) {\n        float m = fabsf(r[i]);",
                       "for (int i = 0; i < 16; i++) {\n        float m = fabsf(r[i]);", 0),
    "int4_truncates": (C, "float rq = nearbyintf(v);", "float rq = truncf(v);", 0),
    "g64_amax_half": (C, "for (int i = 0; i < 64; i++) {\n        float m = fabsf(r[i]);",
                      "for (int i = 0; i < 32; i++) {\n        float m = fabsf(r[i]);", 0),
    "g64_truncates": (C, "float rq = nearbyintf(v);", "float rq = truncf(v);", 1),
    "nvfp4_absmax_unrotated": (C, "float A = absmax_f32(rot_scratch, N * K);", "float A = absmax_f32(R, N * K);", 0),
    "nvfp4_sf_byte": (C, "sf_tiled[or_sf_offset(r, c, C)] = sf;", "sf_tiled[or_sf_offset(r, c, C) ^ 1] = sf;", 0),
    "int8_build_skips_rotation": (C, "            or_fwht256(row + b);\n", "", 0),
    "int8_amax_first_block": (C, "for (int64_t k = 0; k < K; k++) {\n        float m = fabsf(r[k]);",
                              "for (int64_t k = 0; k < 256; k++) {\n        float m = fabsf(r[k]);", 0),
    "int8_truncates": (C, "float rq = nearbyintf(v);", "float rq = truncf(v);", 2),
    "lowrank_input_transposed": (C, "(double)or_bf16_to_f32(lora_down[k * rank + rr]);",
                                 "(double)or_bf16_to_f32(lora_down[rr * K + k]);", 0),
    "fwd_int8_row_scale": (C, "float d = (float)codes[n * K + k] * scales[n];",
                           "float d = (float)codes[n * K + k] * scales[0];", 0),
    # row subsets of the sampled forwards and backward, and the backward's zero skip
    "fwd_nvfp4_x_scale_row": (C, "(double)or_ue4m3_to_f32(xsf[or_sf_offset(m, k / 16, C)]);",
                              "(double)or_ue4m3_to_f32(xsf[or_sf_offset(i, k / 16, C)]);", 0),
    "fwd_int4_x_row": (C, "xb[i * K + k] = (double)or_bf16_to_f32(or_f32_to_bf16(xrot[rows[i] * K + k]));",
                       "xb[i * K + k] = (double)or_bf16_to_f32(or_f32_to_bf16(xrot[i * K + k]));", 0),
    "fwd_int8_x_row": (C, "xb[i * K + k] = (double)or_bf16_to_f32(or_f32_to_bf16(xrot[rows[i] * K + k]));",
                       "xb[i * K + k] = (double)or_bf16_to_f32(or_f32_to_bf16(xrot[i * K + k]));", 1),
    "bwd_dy_row": (C, "double a = (double)or_bf16_to_f32(dy[rows[i] * N + n]);",
                   "double a = (double)or_bf16_to_f32(dy[i * N + n]);", 0),
    "bwd_skips_nonzero": (C, "if (a == 0.0)\n                continue;", "if (a != 0.0)\n                continue;", 0),
    # SVD init (the "Low-rank branch" paragraph)
    "svd_residual_sign": (C, "R[n * K + k] = W[n * K + k] - L;", "R[n * K + k] = W[n * K + k] + L;", 0),
    "svd_residual_index": (C, "L = fmaf(or_bf16_to_f32(up[n * rank + r]), or_bf16_to_f32(down[k * rank + r]), L);",
                           "L = fmaf(or_bf16_to_f32(up[n * rank + r]), or_bf16_to_f32(down[k * rank + (rank - 1 - r)]), L);", 0),
    "svd_sigma_not_split": (C, "double rs = sqrt(sigma[i]);", "double rs = sigma[i];", 0),
    "svd_down_not_split": (C, "down[k * rank + i] = or_f64_to_bf16(v[k * 32 + i] * rs);",
                           "down[k * rank + i] = or_f64_to_bf16(v[k * 32 + i]);", 0),
    "svd_skips_top_vector": (C, "const double *ui = B + (int64_t)ord[i] * N, *vi = VJ + (int64_t)ord[i] * K;",
                             "const double *ui = B + (int64_t)ord[i + 1] * N, *vi = VJ + (int64_t)ord[i + 1] * K;", 0),
    "svd_rounds_through_f32": (C, "up[n * rank + i] = or_f64_to_bf16(u[n * 32 + i] * rs);",
                               "up[n * rank + i] = or_f32_to_bf16((float)(u[n * 32 + i] * rs));", 0),
    "svd_jacobi_rotation_sign": (C, "bi[e] = c * x - s * y;", "bi[e] = c * x + s * y;", 0),
    "svd_sorted_ascending": (C, "S[ord[b2]] > S[ord[b2 - 1]]", "S[ord[b2]] < S[ord[b2 - 1]]", 0),
    "svd_stops_early": (C, "worst <= 1e-13 * s0", "worst <= 1e-3 * s0", 0),
    "f64_bf16_fraction_bits": (C, "round_to_grid(fabs(v), 7, -126)", "round_to_grid(fabs(v), 6, -126)", 0),
}


def plant(text, old, new, occ):
    parts = text.split(old)
    assert len(parts) > occ + 1, f"text to mutate not found (occurrence {occ}): {old!r}"
    return old.join(parts[:occ + 1]) + new + old.join(parts[occ + 1:])


def make_copy(dst, mutant):
    for rel in [C, PY, "synth_inputs.py", "tests/conftest.py"] + PIN_FILES:
        os.makedirs(os.path.join(dst, os.path.dirname(rel)), exist_ok=True)
        shutil.copyfile(os.path.join(ROOT, rel), os.path.join(dst, rel))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    if mutant is not None:
        rel, old, new, occ = MUTANTS[mutant]
        path = os.path.join(dst, rel)
        with open(path) as f:
            text = f.read()
        with open(path, "w") as f:
            f.write(plant(text, old, new, occ))


def run_pins(dst):
    env = dict(os.environ, OMP_NUM_THREADS="1", PYTHONDONTWRITEBYTECODE="1")
    env.pop("PYTHONPATH", None)
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"] + PIN_FILES,
                       cwd=dst, env=env, capture_output=True, text=True, timeout=600)
    return p.returncode, (p.stdout + p.stderr)[-3000:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    base = tmp_path_factory.mktemp("mutants")
    cases = ["control"] + list(MUTANTS)

    def one(name):
        dst = str(base / name)
        make_copy(dst, None if name == "control" else name)
        return name, run_pins(dst)

    workers = max(1, min(8, (os.cpu_count() or 2)))
    with ThreadPoolExecutor(workers) as ex:
        return dict(ex.map(one, cases))


def test_unmodified_copy_passes(outcomes):
    rc, log = outcomes["control"]
    assert rc == 0, log


@pytest.mark.parametrize("mutant", list(MUTANTS))
def test_planted_mistake_fails_a_pin(outcomes, mutant):
    rc, log = outcomes[mutant]
    assert rc == 1 and " failed" in log, f"mutant {mutant} survived the pins (exit {rc}):\n{log}"
