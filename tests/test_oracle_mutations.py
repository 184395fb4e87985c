"""Plants plausible mistakes in copies of the oracle's C source, on the CPU,
and checks that the oracle's pins catch every one of them.  This shows the
pins have teeth: an oracle with any of these slips would not pass."""
import json
import os
import shutil

import numpy as np
import pytest

import oracle
import test_oracle as pins

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "oracle.c")

# (name, text in oracle.c, replacement, pins that must catch it)
MUTATIONS = [
    ("rmsnorm_drops_eps", "sqrt(ss / (double)H + eps)", "sqrt(ss / (double)H)",
     [pins.test_rmsnorm_eps_inside_the_root]),
    ("rmsnorm_eps_outside_root", "sqrt(ss / (double)H + eps)", "(sqrt(ss / (double)H) + eps)",
     [pins.test_rmsnorm_eps_inside_the_root]),
    ("rmsnorm_wrong_weight_index", "* bf16_to_double(w[j])", "* bf16_to_double(w[H - 1 - j])",
     [pins.test_rmsnorm_matches_torch_fp64, pins.test_rmsnorm_hand_example]),
    ("rmsnorm_mean_over_h_minus_1", "sqrt(ss / (double)H + eps)", "sqrt(ss / (double)(H - 1) + eps)",
     [pins.test_rmsnorm_hand_example, pins.test_rmsnorm_matches_torch_fp64]),
    ("matmul_transposed_weight", "s += bf16_to_double(am[k]) * bf16_to_double(wn[k]);",
     "s += bf16_to_double(am[k]) * bf16_to_double(w[k * N + n]);",
     [pins.test_matmul_small_integers_brute_force, pins.test_matmul_matches_torch_fp64]),
    ("matmul_drops_last_k", "for (int64_t k = 0; k < K; ++k)\n                s += bf16_to_double(am[k])",
     "for (int64_t k = 0; k < K - 1; ++k)\n                s += bf16_to_double(am[k])",
     [pins.test_matmul_identity_weight, pins.test_matmul_hand_example]),
    ("kv_write_wrong_offset", "off = slot % ORACLE_PAGE", "off = (slot + 1) % ORACLE_PAGE",
     [pins.test_kv_write_matches_direct_scatter]),
    ("attention_wrong_gqa_map", "int32_t g = h / group;", "int32_t g = h % Hkv;",
     [pins.test_attention_gqa_head_mapping]),
    ("attention_causal_off_by_one", "int64_t n = (int64_t)t + 1;", "int64_t n = (int64_t)t;",
     [pins.test_attention_identical_keys_give_prefix_mean, pins.test_attention_is_causal]),
    ("attention_drops_scale", "double p = exp(s * scale - mx);", "double p = exp(s - mx);",
     [pins.test_attention_matches_torch_sdpa_fp64, pins.test_attention_dominant_logit_closed_form]),
    ("attention_lse_drops_max", "lse[r] = mx + log(l);", "lse[r] = log(l);",
     [pins.test_attention_identical_keys_give_prefix_mean, pins.test_attention_brute_force_tiny]),
    ("attention_wrong_slot", "j % ORACLE_PAGE) * d;\n            const uint16_t *kj",
     "(j + 1) % ORACLE_PAGE) * d;\n            const uint16_t *kj",
     [pins.test_attention_paging_is_transparent, pins.test_attention_matches_torch_sdpa_fp64]),
    ("attention_values_not_normalised", "orow[i] /= l;", "orow[i] /= 1.0;",
     [pins.test_attention_identical_keys_give_prefix_mean]),
    ("embedding_off_by_one_row", "memcpy(out + t * H, table + id * H,",
     "memcpy(out + t * H, table + ((id + 1) % V) * H,",
     [pins.test_embedding_rows_carry_their_ids, pins.test_embedding_matches_fancy_indexing]),
    ("rope_sin_sign_flipped", "orow[i] = a * c - b * s;", "orow[i] = a * c + b * s;",
     [pins.test_rope_hand_example, pins.test_rope_matches_complex_rotation]),
    ("rope_interleaved_pairs", "b = bf16_to_double(xr[i + half]);",
     "b = bf16_to_double(xr[i ^ 1]);",
     [pins.test_rope_hand_example, pins.test_rope_matches_complex_rotation]),
    ("rope_frequency_exponent_i_over_d", "pow(theta, -2.0 * (double)i / (double)d)",
     "pow(theta, -1.0 * (double)i / (double)d)",
     [pins.test_rope_hand_example, pins.test_rope_matches_complex_rotation]),
    ("swiglu_gate_and_up_swapped", "double g = bf16_to_double(gu[t * 2 * F + j]);",
     "double g = bf16_to_double(gu[t * 2 * F + F + j]);",
     [pins.test_swiglu_closed_forms, pins.test_swiglu_matches_torch_fp64]),
    ("swiglu_sigmoid_not_silu", "out[t * F + j] = g / (1.0 + exp(-g)) * u;",
     "out[t * F + j] = 1.0 / (1.0 + exp(-g)) * u;",
     [pins.test_swiglu_closed_forms, pins.test_swiglu_matches_torch_fp64]),
    ("add_rmsnorm_norm_ignores_delta", "            ss += v * v;\n        }\n        double mean_sq",
     "            ss += bf16_to_double(x[r * H + i]) * bf16_to_double(x[r * H + i]);\n        }\n        double mean_sq",
     [pins.test_add_rmsnorm_constant_sum_closed_form, pins.test_add_rmsnorm_matches_torch_fp64]),
    ("add_rmsnorm_eps_outside_root", "sqrt(mean_sq + eps)", "(sqrt(mean_sq) + eps)",
     [pins.test_add_rmsnorm_constant_sum_closed_form, pins.test_add_rmsnorm_matches_torch_fp64]),
    ("philox_hi_lo_swapped", "c[1] = lo1;", "c[1] = hi1;",
     [pins.test_philox_known_answer_vectors]),
    ("philox_key_not_bumped", "k[0] += 0x9E3779B9u;", "k[0] += 0u;",
     [pins.test_philox_known_answer_vectors]),
    ("sample_temperature_multiplies", "w[j] = exp((double)row[j] / (double)temperature[t] - mx);",
     "w[j] = exp((double)row[j] * (double)temperature[t] - mx);",
     [pins.test_sample_frequencies_follow_the_softmax]),
    ("sample_ties_dropped", "if (w[j] >= tau) zk += w[j];", "if (w[j] > tau) zk += w[j];",
     [pins.test_sample_ties_at_the_threshold_are_all_kept]),
    ("sample_wrong_word", "double u = (double)(rnd[0] >> 8)", "double u = (double)(rnd[1] >> 8)",
     [pins.test_sample_uniform_logits_closed_form]),
    ("sample_nucleus_ignored", "double need = (double)top_p[t] * total", "double need = total",
     [pins.test_sample_nucleus_drops_the_tail, pins.test_sample_dominant_logit_and_tiny_top_p]),
    ("moe_route_ties_to_higher_index", "if (best < 0 || row[e] > row[best]) best = e;",
     "if (best < 0 || row[e] >= row[best]) best = e;",
     [pins.test_moe_route_hand_example, pins.test_moe_route_matches_a_stable_sort]),
    ("moe_route_weights_not_renormalised", "weights[t * k + i] = exp((double)row[ex[i]] - (double)row[ex[0]]) / sum;",
     "weights[t * k + i] = exp((double)row[ex[i]] - (double)row[ex[0]]);",
     [pins.test_moe_route_hand_example, pins.test_moe_route_matches_a_stable_sort]),
    ("moe_dispatch_wrong_position", "pos[i] = p;", "pos[i] = p + 1;",
     [pins.test_moe_dispatch_groups_by_expert_stably]),
    ("moe_combine_ignores_weights", "out[t * H + h] += weights[t * k + i] * bf16_to_double(yr[h]);",
     "out[t * H + h] += bf16_to_double(yr[h]);",
     [pins.test_moe_combine_closed_forms]),
    ("argmax_ties_take_highest_index", "if (row[j] > row[best]) best = j;",
     "if (row[j] >= row[best]) best = j;",
     [pins.test_argmax_ties_take_the_lowest_index, pins.test_argmax_matches_numpy_first_occurrence]),
    ("fold_indexes_w_by_row", "* bf16_to_double(w[k]);", "* bf16_to_double(w[n % K]);",
     [pins.test_fold_norm_weight_closed_forms, pins.test_fold_norm_weight_small_integers]),
    ("rmsnorm_matmul_drops_eps", "sqrt(sum_sq / (double)K + eps)", "sqrt(sum_sq / (double)K)",
     [pins.test_rmsnorm_matmul_one_hot_rows_closed_form]),
    ("rmsnorm_matmul_mean_over_n", "sqrt(sum_sq / (double)K + eps)", "sqrt(sum_sq / (double)N + eps)",
     [pins.test_rmsnorm_matmul_hand_example, pins.test_rmsnorm_matmul_one_hot_rows_closed_form]),
    ("rmsnorm_matmul_not_normalised", "s += (bf16_to_double(xm[k]) / root) * bf16_to_double(wn[k]);",
     "s += bf16_to_double(xm[k]) * bf16_to_double(wn[k]);",
     [pins.test_rmsnorm_matmul_hand_example, pins.test_rmsnorm_matmul_matches_torch_fp64]),
    ("rmsnorm_matmul_transposed_weight",
     "s += (bf16_to_double(xm[k]) / root) * bf16_to_double(wn[k]);",
     "s += (bf16_to_double(xm[k]) / root) * bf16_to_double(wf[(k * N + n) % (N * K)]);",
     [pins.test_rmsnorm_matmul_hand_example, pins.test_rmsnorm_matmul_matches_torch_fp64]),
    ("rope_angles_exponent_i_over_d", "pow(theta, -(double)(2 * i) / (double)d)",
     "pow(theta, -(double)(i) / (double)d)",
     [pins.test_rope_angles_closed_forms, pins.test_rope_angles_rotate_like_rope]),
    ("rope_angles_cos_sin_swapped", "* 2] = cos((double)p * freq);", "* 2] = sin((double)p * freq);",
     [pins.test_rope_angles_closed_forms]),
    ("rmsnorm_backward_r_squared", "bf16_to_double(x[r * H + j]) * inv * inv * inv / (double)H * dot;",
     "bf16_to_double(x[r * H + j]) * inv * inv / (double)H * dot;",
     [pins.test_rmsnorm_backward_matches_finite_differences, pins.test_rmsnorm_backward_closed_forms]),
    ("rmsnorm_backward_dw_without_r",
     "acc += bf16_to_double(dy[m * H + j]) * bf16_to_double(x[m * H + j]) * rs[m];",
     "acc += bf16_to_double(dy[m * H + j]) * bf16_to_double(x[m * H + j]);",
     [pins.test_rmsnorm_backward_matches_finite_differences, pins.test_rmsnorm_backward_closed_forms]),
    ("rmsnorm_backward_dot_without_w", "dot += bf16_to_double(w[i]) * bf16_to_double(dy[r * H + i]) * xi;",
     "dot += bf16_to_double(dy[r * H + i]) * xi;",
     [pins.test_rmsnorm_backward_matches_finite_differences]),
    ("attention_backward_ds_without_mean", "const double ds = wt[key] * (dp[key] - mean_dp);",
     "const double ds = wt[key] * dp[key];",
     [pins.test_attention_backward_matches_finite_differences, pins.test_attention_backward_closed_forms]),
    ("attention_backward_dk_without_scale", "dk[off[key] + i] += scale * ds * bf16_to_double(qr[i]);",
     "dk[off[key] + i] += ds * bf16_to_double(qr[i]);",
     [pins.test_attention_backward_matches_finite_differences]),
    ("attention_backward_dv_from_ds", "dv[off[key] + i] += wt[key] * bf16_to_double(gr[i]);",
     "dv[off[key] + i] += (wt[key] - 0.5 * (dp[key] - mean_dp)) * bf16_to_double(gr[i]);",
     [pins.test_attention_backward_matches_finite_differences, pins.test_attention_backward_closed_forms]),
    ("attention_backward_sees_one_key_less", "const int64_t visible = (int64_t)row_pos[r] + 1;",
     "const int64_t visible = (int64_t)row_pos[r] + (row_pos[r] > 0 ? 0 : 1);",
     [pins.test_attention_backward_matches_finite_differences, pins.test_attention_backward_closed_forms]),
    ("swiglu_backward_drops_sigmoid_slope", "dy * up * sig * (1.0 + gate * (1.0 - sig));",
     "dy * up * sig;",
     [pins.test_swiglu_backward_matches_finite_differences]),
    ("swiglu_backward_dup_uses_up", "dgu[t * 2 * F + F + j] = dy * gate * sig;",
     "dgu[t * 2 * F + F + j] = dy * up * sig;",
     [pins.test_swiglu_backward_matches_finite_differences]),
    ("rope_backward_rotates_forward", "xr[i] = lo * cs + hi * sn;", "xr[i] = lo * cs - hi * sn;",
     [pins.test_rope_backward_is_the_inverse_rotation]),
    ("matmul_residual_drops_residual", "c[m * N + n] = bf16_to_double(r[m * N + n]) + dot;",
     "c[m * N + n] = dot;",
     [pins.test_matmul_residual_small_integers_brute_force, pins.test_matmul_residual_degenerate_cases]),
    ("matmul_residual_transposed_residual", "c[m * N + n] = bf16_to_double(r[m * N + n]) + dot;",
     "c[m * N + n] = bf16_to_double(r[(n * M + m) % (M * N)]) + dot;",
     [pins.test_matmul_residual_small_integers_brute_force, pins.test_matmul_residual_degenerate_cases]),
]


def _catches(pin, orc):
    try:
        if pin is pins.test_rmsnorm_constant_row_closed_form:
            pin(orc, 0.001)
        else:
            pin(orc)
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("name,find,repl,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, find, repl, catchers):
    src = open(SRC).read()
    assert src.count(find) == 1, "mutation anchor must occur exactly once: %r" % find
    mut = tmp_path / ("oracle_%s.c" % name)
    mut.write_text(src.replace(find, repl))
    lib = oracle.build(force=True, src=str(mut), out=str(tmp_path / ("lib_%s.so" % name)))
    orc = oracle.Oracle(lib)
    caught = [p.__name__ for p in catchers if _catches(p, orc)]
    assert caught, "no pin caught the planted mistake %s" % name


def test_unmutated_copy_passes_every_listed_pin(tmp_path):
    dst = tmp_path / "oracle_copy.c"
    shutil.copy(SRC, dst)
    orc = oracle.Oracle(oracle.build(force=True, src=str(dst), out=str(tmp_path / "lib.so")))
    for _, _, _, catchers in MUTATIONS:
        for p in catchers:
            assert not _catches(p, orc), p.__name__


def test_oracle_matches_its_regression_fixture():
    """tests/golden/oracle_tiny.json was written by make_oracle_tiny.py from
    the oracle; any change to the oracle's arithmetic shows up here."""
    with open(os.path.join(HERE, "golden", "oracle_tiny.json")) as f:
        g = json.load(f)
    u16 = lambda a: np.asarray(a, dtype=np.uint16)  # noqa: E731
    r = g["rmsnorm"]
    np.testing.assert_array_equal(oracle.rmsnorm(u16(r["x"]), u16(r["w"]), r["eps"]), r["y"])
    m = g["matmul"]
    np.testing.assert_array_equal(oracle.matmul(u16(m["a"]), u16(m["w"])), m["c"])
    a = g["attention"]
    q = u16(a["q"])
    rows = oracle.decode_rows(q, a["seq_lens"])
    o, lse = oracle.attention(*rows, a["Hq"], u16(a["k_cache"]), u16(a["v_cache"]),
                              np.asarray(a["block_table"], dtype=np.int32), want_lse=True)
    np.testing.assert_allclose(o, a["o"], rtol=1e-15, atol=0)
    np.testing.assert_allclose(lse, a["lse"], rtol=1e-15, atol=0)
