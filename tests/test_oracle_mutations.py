"""Plant a plausible mistake in a copy of the oracle (on the CPU) and check that the pins
catch it.  Each mutation edits one expression of qg_oracle.c; the pin named beside it must
then fail.  This shows the pins constrain the oracle's arithmetic, not just its shape."""
import pytest

import oracle
import test_oracle_awq_pins as awq
import test_oracle_gptq_pins as gptq
import test_oracle_outlier_pins as outl
import test_oracle_pins as pins
import test_oracle_sparse24_pins as sp24

MUTATIONS = [
    # (original text, mutated text, pins that must fail)
    ("nearbyintf(v / s) + z, 0, 15)", "nearbyintf(v / s), 0, 15)",
     [pins.test_w4_asym_round_trip_bound_and_ranges]),
    ("float s32 = r / 15.0f;", "float s32 = r / 16.0f;",
     [lambda: pins.test_w4_asym_hand_examples(0)]),
    ("uint16_t s16 = qgo_f32_to_f16_ru(s32);", "uint16_t s16 = (uint16_t)(qgo_f32_to_f16_ru(s32) - (qgo_f32_to_f16_ru(s32) > 0 && qgo_f16_to_f32(qgo_f32_to_f16_ru(s32)) != s32));",
     [lambda: pins.test_w4_asym_hand_examples(0)]),
    ("<< (4 * i);", "<< (4 * (7 - i));", [lambda: pins.test_pack_hand_words(0)]),
    ("return (double)(q - (int)zeros[g * N + n])", "return (double)((int)zeros[g * N + n] - q)",
     [pins.test_w4a16_ref_reduces_to_integer_matmul]),
    ("int64_t g = k / group;\n    int q = nib(packed, N, k, n);", "int64_t g = n % (K_UNUSED + 1);\n    int q = nib(packed, N, k, n);",
     [pins.test_w4a16_ref_reduces_to_integer_matmul]),
    ("sj = sqrtf(ax) / sqrtf(aw);", "sj = sqrtf(aw) / sqrtf(ax);", [pins.test_smooth_half_alpha_equalises_ranges]),
    ("int qw = v >= 8 ? v - 16 : v;", "int qw = v;", [pins.test_w4a8_partials_and_reference]),
    # W4A8 output: binary64 accumulation instead of binary32, and t applied twice
    ("float acc = 0.0f;", "double acc = 0.0;",
     [pins.test_w4a8_output_sums_groups_in_ascending_order_in_binary32]),
    ("qgo_f32_to_bf16_rn(acc * t[m]);", "qgo_f32_to_bf16_rn(acc * t[m] * t[m]);",
     [pins.test_w4a8_output_exact_case_is_rounded_integer_product]),
    ("float tm = a / 127.0f;", "float tm = a / 128.0f;", [pins.test_act_i8_closed_form_and_brute_force]),
    ("float s = amax / 7.0f;", "float s = amax / 8.0f;", [pins.test_w4_sym_absmax_bound_brute_force]),
    # AWQ search
    ("sum += fabs((double)X[m * K + c]);", "sum += (double)X[m * K + c];", [awq.test_act_mean_closed_form]),
    ("(float)pow((double)xm[c], alpha);", "(float)pow((double)xm[c], 1.0 - alpha);",
     [awq.test_scales_closed_forms, awq.test_alpha_one_is_exact_on_the_constructed_layer]),
    ("qgo_bf16_to_f32(qgo_f32_to_bf16_rn(X[m * K + k] * inv_s[k]))", "qgo_bf16_to_f32(qgo_f32_to_bf16_rn(X[m * K + k] * s[k]))",
     [awq.test_alpha_one_is_exact_on_the_constructed_layer]),
    ("int status = qgo_quantize_w4_asym(W, s, K, N, group, codes, sc, z);",
     "int status = qgo_quantize_w4_asym(W, inv_s, K, N, group, codes, sc, z);",
     [awq.test_alpha_one_is_exact_on_the_constructed_layer]),
    ("if (status == OR_OK && mse[i] < mse[bi]) bi = i;", "if (status == OR_OK && mse[i] <= mse[bi]) bi = i;",
     [awq.test_zero_weights_tie_goes_to_the_first_point]),
    ("(double)i / (double)(n_grid - 1)", "(double)i / (double)n_grid", [awq.test_grid_points]),
    ("xs_bf16[m * K + k] = qgo_f32_to_bf16_rn(X[m * K + k] * inv_s[k]);",
     "xs_bf16[m * K + k] = qgo_f32_to_bf16_rn(X[m * K + k] / inv_s[k]);", [awq.test_scale_act_rounds_once_to_bf16]),
    # INT8 outlier side path
    ("if (a > bm) { bm = a; best = i; }", "if (a >= bm) { bm = a; best = i; }", [outl.test_selection_matches_a_stable_sort]),
    ("float sc = amax / 127.0f;", "float sc = amax / 128.0f;", [outl.test_int8_codes_closed_form]),
    ("W_dense[(g * group + pick[r]) * N + n] = 0.0f; /* reading R */", "/* outlier left in the dense part */",
     [outl.test_dense_remainder]),
    ("int64_t k = g * group + idx[(g * count + r) * N + n];", "int64_t k = idx[(g * count + r) * N + n];",
     [outl.test_side_path_product_against_numpy]),
    # 2:4 sparsity
    ("if (a > best) { best = a; keep[r] = i; }", "if (a >= best) { best = a; keep[r] = i; }",
     [sp24.test_hand_column, sp24.test_selection_matches_a_stable_sort]),
    ("meta[(b / 8) * N + n] |= (uint32_t)((i1 << 2) | i0) << (4 * (b % 8));",
     "meta[(b / 8) * N + n] |= (uint32_t)((i0 << 2) | i1) << (4 * (b % 8));", [sp24.test_hand_column]),
    ("int64_t k = 4 * b + pos[j], kv = 2 * b + j, g = k / group;", "int64_t k = 4 * b + j, kv = 2 * b + j, g = k / group;",
     [sp24.test_reference_product_against_numpy]),
    # GPTQ
    ("for (int64_t j = k + 1; j < K; ++j) Wc[j * N + n] -= e * Hinv[k * K + j];",
     "for (int64_t j = k + 1; j < K; ++j) Wc[j * N + n] += e * Hinv[k * K + j];",
     [gptq.test_cholesky_form_agrees, gptq.test_lower_layer_error_than_round_to_nearest]),
    ("for (int64_t b = k + 1; b < K; ++b) Hinv[a * K + b] -= f * Hinv[k * K + b];",
     "for (int64_t b = k + 1; b < K; ++b) Hinv[a * K + b] -= 0.0 * f * Hinv[k * K + b];",
     [gptq.test_cholesky_form_agrees]),
    ("double lambda = tr > 0.0 ? damp * tr / (double)K : damp;", "double lambda = tr > 0.0 ? damp * tr : damp;",
     [gptq.test_hessian_hand_case]),
    ("H[a * K + b] = 2.0 * s / (double)Mc;", "H[a * K + b] = s / (double)Mc;", [gptq.test_hessian_hand_case]),
    ("for (int i = 0; i < group; ++i) gv[i] = (float)Wc[(k + i) * N + n];",
     "for (int i = 0; i < group; ++i) gv[i] = W[(k + i) * N + n];", [gptq.test_cholesky_form_agrees]),
    ("double d = yref[i] - yq[i];", "double d = yref[i] - 0.5 * yq[i];", [awq.test_alpha_zero_is_the_plain_int4_layer]),
]


@pytest.mark.parametrize("idx", range(len(MUTATIONS)))
def test_planted_mistake_is_caught(idx, tmp_path):
    orig, mutated, must_fail = MUTATIONS[idx]
    src = oracle.source_text()
    assert orig in src, f"mutation anchor not found: {orig!r}"
    text = src.replace(orig, mutated)
    if "K_UNUSED" in mutated:
        text = "#define K_UNUSED 0\n" + text
    L = oracle.build_variant(text, str(tmp_path / f"mut{idx}.so"))
    with oracle.use_library(L):
        for pin in must_fail:
            with pytest.raises(AssertionError):
                pin()
