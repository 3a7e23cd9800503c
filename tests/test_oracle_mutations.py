"""Plants plausible mistakes in a copy of the oracle (on the CPU) and checks
that at least one pin catches each: the pins are only worth something if a
dropped term, a wrong sign or index, or a transposed operand fails them."""
import importlib.util
import os
import shutil
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, HERE)
import test_oracle_attn as attn_pins  # noqa: E402
import test_oracle_mlp as mlp_pins  # noqa: E402
import test_oracle_pins as pins  # noqa: E402
import test_oracle_gptq as gptq_pins  # noqa: E402
import test_oracle_scale as scale_pins  # noqa: E402
import test_oracle_state16 as state16_pins  # noqa: E402

# (name, original text, planted text, pins expected to catch it)
MUTATIONS = [
    ("philox_weyl_constant", "W0 = 0x9E3779B9u", "W0 = 0x9E3779B8u",
     ["test_philox_known_answers"]),
    ("philox_swapped_words", "uint32_t n0 = hi1 ^ c1 ^ k0;",
     "uint32_t n0 = hi0 ^ c1 ^ k0;", ["test_philox_known_answers"]),
    ("uniform_bits", "((double)(x >> 9) + 0.5)", "((double)(x >> 8) + 0.5)",
     ["test_u01_exact_open_interval"]),
    ("gumbel_sign", "g[k] = -log(-log((double)u[k]));",
     "g[k] = log(-log((double)u[k]));", ["test_softmax_is_library_softmax"]),
    ("dropped_temperature", "z[k] = (l[k] + g[k]) / tau;", "z[k] = (l[k] + g[k]);",
     ["test_softmax_is_library_softmax", "test_gradients_match_central_differences"]),
    ("jacobian_sign", "acc += yy[j] * (cand[p] - cand[j]);",
     "acc += yy[j] * (cand[j] - cand[p]);",
     ["test_gradients_match_central_differences"]),
    ("ternary_dropped_p0", "double gm = a * (qp - qm) * p1 * p0;",
     "double gm = a * (qp - qm) * p1;", ["test_gradients_match_central_differences"]),
    ("scale_grad_dropped_v", "dsg += dw * v[c];", "dsg += dw;",
     ["test_gradients_match_central_differences"]),
    ("weight_grad_transposed", "double d = dY[t * N + n];", "double d = dY[n * N + t];",
     ["test_loss_and_weight_grad_equal_library_gemm"]),
    ("output_grad_factor", "dY[t * N + n] = (float)gsqo_bf16_round(2.0 * e);",
     "dY[t * N + n] = (float)gsqo_bf16_round(e);",
     ["test_loss_and_weight_grad_equal_library_gemm"]),
    ("lion_beta_swap", "float c = fmaf(beta1, m, omb1 * g);",
     "float c = fmaf(beta2, m, omb2 * g);", ["test_lion_second_step_closed_form"]),
    ("rtn_ties_last", "if (d < bestd) {", "if (d <= bestd) {",
     ["test_init_scales_and_rtn_bruteforce"]),
    ("ternary_init_sign_of_zero", "(lev == 1 && !(w < 0.0f))", "(lev == 1 && (w > 0.0f))",
     ["test_init_logits_layout"]),
    ("local_shift_no_upper_clamp", "if (j > 7) j = 7;\n            c[k]", "c[k]",
     ["test_local_shift_clamped_exhaustive"]),
    ("ternary_harden_sign", "lev = nonzero ? (plus ? 2 : 0) : 1;",
     "lev = nonzero ? (plus ? 0 : 2) : 1;", ["test_harden_bruteforce_and_pack_roundtrip"]),
    ("pack_msb_first", "packed[n * wpr + bit / 32] |= (1u << (bit % 32));",
     "packed[n * wpr + bit / 32] |= (1u << (31 - bit % 32));",
     ["test_harden_bruteforce_and_pack_roundtrip"]),
    ("mlp_silu_derivative", "double dsilu = sg * (1.0 + av * (1.0 - sg));",
     "double dsilu = sg * (1.0 - av * (1.0 - sg));", ["mlp:test_mlp_matches_torch_autograd"]),
    ("mlp_dropped_up_factor", "double gav = dh * b[t * F + f] * dsilu;",
     "double gav = dh * dsilu;", ["mlp:test_mlp_matches_torch_autograd"]),
    ("attn_no_score_scale",
     "const double scale = 1.0 / sqrt((double)d);\n    #pragma omp parallel for collapse(2)",
     "const double scale = 1.0;\n    #pragma omp parallel for collapse(2)",
     ["attn:test_probs_match_torch"]),
    ("attn_rope_sign", "x[i + half] = b * cs + a * sn;\n            }\n            for (int64_t g",
     "x[i + half] = b * cs - a * sn;\n            }\n            for (int64_t g",
     ["attn:test_probs_match_torch", "attn:test_rotary_relative_position_property"]),
    ("attn_causal_strict", "for (int64_t k = 0; k <= q; ++k) {\n                    const double* kv",
     "for (int64_t k = 0; k < q + (q == 0); ++k) {\n                    const double* kv",
     ["attn:test_probs_match_torch"]),
    ("attn_wrong_group", "const int64_t g = h / grp;\n            for (int64_t q = 0; q < S; ++q)\n                for (int64_t j",
     "const int64_t g = h % nkv;\n            for (int64_t q = 0; q < S; ++q)\n                for (int64_t j",
     ["attn:test_vo_matches_torch_autograd"]),
    ("mlp_down_grad_transposed", "for (int64_t t = 0; t < T; ++t) acc += dp[t * H + n] * h[t * F + f];",
     "for (int64_t t = 0; t < T; ++t) acc += dp[t * H + n] * h[t * F + (F - 1 - f)];",
     ["mlp:test_mlp_matches_torch_autograd"]),
    ("scale_grad_uses_level_index",
     "acc += (double)dW[n * K + k] * gsqo_level_value(mode, lev[n * K + k]);",
     "acc += (double)dW[n * K + k] * (double)lev[n * K + k];",
     ["scale:test_scale_grad_central_differences"]),
    ("scale_weight_unscaled",
     "double w = (double)s[n * G + k / group] * gsqo_level_value(mode, lev[c]);\n        wq[c]",
     "double w = gsqo_level_value(mode, lev[c]);\n        wq[c]",
     ["scale:test_scale_grad_central_differences", "scale:test_scale_step_on_grid_weight_is_a_fixed_point"]),
    ("state16_logits_to_nearest", "logits[p * NK + i] = gsqo_bf16_sr(logits[p * NK + i], w[p]);",
     "logits[p * NK + i] = (float)gsqo_bf16_round((double)logits[p * NK + i]);",
     ["state16:test_rounding_follows_fp32_lion_on_average",
      "state16:test_thresholds_are_next_step_philox_words"]),
    ("state16_thresholds_this_step",
     "coord_words(mode, seed, t_next, coord, w);",
     "coord_words(mode, seed, t_next - 1u, coord, w);",
     ["state16:test_thresholds_are_next_step_philox_words"]),
    ("quad_word_fixed", "w[4] = out[coord % 4];", "w[4] = out[0];",
     ["test_counter_layout"]),
    ("quad_block_per_coordinate", "uint64_t q = coord - coord % 4;", "uint64_t q = coord;",
     ["test_counter_layout"]),
    ("state16_threshold_scale", "b += (r9 & 0x1FFu) << 7;", "b += (r9 & 0x1FFu) << 6;",
     ["state16:test_stochastic_rounding_brackets_and_is_unbiased"]),
    ("state16_momenta_truncated",
     "mom[p * NK + i] = (float)gsqo_bf16_round((double)mom[p * NK + i]);",
     "mom[p * NK + i] = gsqo_bf16_sr(mom[p * NK + i], 0u);",
     ["state16:test_momenta_round_to_nearest"]),
    ("gptq_update_transposed", "W[:, j + 1:] -= np.outer(e, U[j, j + 1:])",
     "W[:, j + 1:] -= np.outer(e, U[j + 1:, j])",
     ["gptq:test_first_column_update_is_damped_least_squares", "gptq:test_loss_identity_over_the_loop"]),
    ("gptq_no_diagonal_division", "e = (W[:, j] - q) / U[j, j]", "e = (W[:, j] - q)",
     ["gptq:test_first_column_update_is_damped_least_squares", "gptq:test_loss_identity_over_the_loop"]),
    ("gptq_scale_from_group_start_only", "absmax = np.abs(W[:, j:j + group]).max(axis=1)",
     "absmax = np.abs(W[:, j:j + 1]).max(axis=1)",
     ["gptq:test_diagonal_hessian_is_round_to_nearest"]),
]

MODES = {"test_softmax_is_library_softmax": [0, 2]}


def _load_mutant(tmp_path, name, old, new):
    dst = tmp_path / f"oracle_{name}"
    shutil.copytree(os.path.join(ROOT, "oracle"), dst,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    target = "gptq.py" if name.startswith("gptq_") else "gsq_oracle.c"
    src = (dst / target).read_text()
    assert src.count(old) == 1, f"mutation anchor not unique: {name}"
    (dst / target).write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_{name}", dst / "__init__.py",
                                                  submodule_search_locations=[str(dst)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new, catchers):
    mod = _load_mutant(tmp_path, name, old, new)
    caught = []
    for tname in catchers:
        module = {"mlp": mlp_pins, "attn": attn_pins, "scale": scale_pins,
                  "gptq": gptq_pins, "state16": state16_pins}.get(
            tname.split(":")[0], pins) \
            if ":" in tname else pins
        tname = tname.split(":")[-1]
        fn = getattr(module, tname)
        params = getattr(fn, "pytestmark", [])
        modes = MODES.get(tname)
        if modes is None:
            modes = [0, 1, 2] if any(m.name == "parametrize" for m in params) else [None]
        for mode in modes:
            try:
                fn(mod) if mode is None else fn(mod, mode)
            except AssertionError:
                caught.append((tname, mode))
    assert caught, f"no pin caught the planted mistake {name}"
