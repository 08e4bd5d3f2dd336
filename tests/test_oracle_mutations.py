"""The pins must catch plausible mistakes: each case plants one mistake in a
copy of the oracle's C source (never in the CUDA path), builds it, and checks
that at least one pin fails against the mutant."""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kvq_oracle.c")

MUTATIONS = {
    "scale uses 2^b instead of 2^b-1": ("s = range / (float)qmax;", "s = range / (float)(qmax + 1u);"),
    "round half up instead of half to even": ("float r = nearbyintf(t);", "float r = floorf(t + 0.5f);"),
    "MSB-first bit packing": ("(uint8_t)(1u << (bit % 8))", "(uint8_t)(0x80u >> (bit % 8))"),
    "MSB-first bit unpacking": ("if ((group_bytes[bit / 8] >> (bit % 8)) & 1u)",
                                "if ((group_bytes[bit / 8] >> (7 - bit % 8)) & 1u)"),
    "min term dropped from the affine value": ("out[r * head_dim + g * ORACLE_GROUP + i] = mn + s * (double)c;",
                                               "out[r * head_dim + g * ORACLE_GROUP + i] = s * (double)c;"),
    "interleaved instead of consecutive GQA head map": ("const int h = hk * group_q + j;",
                                                        "const int h = j * n_kv_heads + hk;"),
    "softmax scale dropped": ("logit[t] = softmax_scale * acc;", "logit[t] = acc;"),
    "keys and values swapped": ("acc += qd[d] * kh[t * D + d];", "acc += qd[d] * vh[t * D + d];"),
    "bf16 truncation instead of rounding": ("if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;",
                                            "if (0) kept += 1u;"),
    "negative zero kept as min": ("if (mn == 0.0f) mn = 0.0f; /* -0 -> +0 */", "/* zero sign kept */"),
    "window keys lost": ("kh[(n_packed + t) * D + d] = bf16_to_f32(k_win[((int64_t)hk * n_window + t) * D + d]);",
                         "kh[(n_packed + t) * D + d] = 0.0;"),
}

CHECKS = [
    (pins.test_packing_closed_form_every_position_and_value, dict(bits=3)),
    (pins.test_packing_b4_nibbles_and_b8_identity, {}),
    (pins.test_on_grid_round_trip_is_exact, dict(bits=4, k=3)),
    (pins.test_round_half_to_even, {}),
    (pins.test_constant_groups, {}),
    (pins.test_error_bound_endpoints_and_brute_force, dict(bits=2)),
    (pins.test_dequantize_matches_library_rounding, dict(bits=4)),
    (pins.test_bf16_rounding_ties, {}),
    (pins.test_attention_matches_numpy_scipy_brute_force, {}),
    (pins.test_attention_matches_torch_sdpa_fp64, {}),
    (pins.test_window_only_view_is_textbook_bf16_attention, {}),
    (pins.test_softmax_rows_sum_to_one_and_match_probs, {}),
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-o",
                    str(lib), str(mutant), "-lm"], check=True)
    caught = []
    with oracle.use_library(str(lib)):
        for fn, kw in CHECKS:
            try:
                fn(**kw)
            except (AssertionError, ValueError):
                caught.append(fn.__name__)
    assert caught, f"no pin caught: {name}"


# ---- the oracle's numpy functions (sequences, top-K, width allocation):
# each case rewrites one line of one function's source, runs the mutant in
# the oracle module's namespace, and checks that a pin fails against it

import inspect

PY_MUTATIONS = {
    "segments: window rows dropped": (
        "decode_attn_segments", "            ks.append(_bf16_to_f64(kw))\n            vs.append(_bf16_to_f64(seg[\"v_win\"]))",
        "            pass"),
    "segments: values taken from the key codes": (
        "decode_attn_segments", "vs.append(affine(seg[\"v_codes\"], seg[\"v_sm\"], D, seg[\"bits\"]))",
        "vs.append(affine(kc, seg[\"k_sm\"], D, seg[\"bits\"]))"),
    "segments: only the first segment attended": (
        "decode_attn_segments", "    for seg in segments:", "    for seg in segments[:1]:"),
    "top-K: score from the group's first query head only": (
        "sparse_decode_attn", "for h in heads]), axis=0)", "for h in heads][:1]), axis=0)"),
    "top-K: ties to the higher index": (
        "sparse_decode_attn", "order = np.argsort(-score, kind=\"stable\")",
        "order = (n_p - 1 - np.argsort(-score[::-1], kind=\"stable\"))"),
    "top-K: window left out of the active set": (
        "sparse_decode_attn", "k = np.concatenate([kp[hk][sel], kw[hk]], axis=0)",
        "k = np.concatenate([kp[hk][sel], kw[hk][:0]], axis=0)"),
    "top-K: one token too many": (
        "sparse_decode_attn", "sel = np.sort(order[:min(top_k, n_p)])", "sel = np.sort(order[:min(top_k + 1, n_p)])"),
    "sensitivity: value term dropped": (
        "width_sensitivity", "ev = np.sqrt((64 * (rv / 2) ** 2).sum())", "ev = 0.0"),
    "sensitivity: key ranges halved twice": (
        "width_sensitivity", "delta = softmax_scale * (l1 * rk / 2).sum(axis=1).max()",
        "delta = softmax_scale * (l1 * rk / 4).sum(axis=1).max()"),
    "sensitivity: group ranges from the first token only": (
        "width_sensitivity", "rk = (kg.max(axis=2) - kg.min(axis=2)).max(axis=0)",
        "rk = (kg.max(axis=2) - kg.min(axis=2))[0]"),
    "allocation: error per width with 2^b instead of 2^b - 1": (
        "allocate_widths", "err = float(sens[i]) / (2 ** b - 1)", "err = float(sens[i]) / (2 ** b)"),
    "allocation: costs rounded down": (
        "allocate_widths", "            cost = -(-(int(capacity[i]) * 2 * n_kv_heads * (head_dim * b // 8 + head_dim // 64 * 8)) // unit)",
        "            cost = (int(capacity[i]) * 2 * n_kv_heads * (head_dim * b // 8 + head_dim // 64 * 8)) // unit"),
    "allocation: scale/min bytes left out of the cost": (
        "allocate_widths", "            cost = -(-(int(capacity[i]) * 2 * n_kv_heads * (head_dim * b // 8 + head_dim // 64 * 8)) // unit)",
        "            cost = -(-(int(capacity[i]) * 2 * n_kv_heads * (head_dim * b // 8)) // unit)"),
}

PY_CHECKS = {
    "decode_attn_segments": [(pins.test_one_segment_is_the_view_attention, {}),
                             (pins.test_view_split_into_segments_changes_nothing, dict(cut=17)),
                             (pins.test_segments_of_different_widths_match_brute_force_and_order, {}),
                             (pins.test_identical_keys_over_segments_give_mean_of_all_values, {})],
    "sparse_decode_attn": [(pins.test_sparse_with_every_token_selected_is_dense, dict(top_k=45)),
                           (pins.test_sparse_error_within_discarded_mass_bound, dict(bits=4, top_k=5)),
                           (pins.test_sparse_selects_a_planted_key_and_attends_it_with_the_window, {}),
                           (pins.test_sparse_score_takes_the_group_maximum_and_ties_go_low, {})],
    "width_sensitivity": [(pins.test_sensitivity_bounds_the_error_of_quantizing_recent_tokens, dict(bits=b))
                          for b in (2, 3, 4, 8)] + [(pins.test_sensitivity_of_a_constant_window_is_zero, {}),
                                                    (pins.test_sensitivity_closed_form, {})],
    "allocate_widths": [(pins.test_allocation_matches_brute_force, dict(seed=s)) for s in range(6)] +
                       [(pins.test_allocation_extremes, {})],
}


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_pins_catch_python_oracle_mutation(name, monkeypatch):
    fn, old, new = PY_MUTATIONS[name]
    src = inspect.getsource(getattr(oracle, fn))
    assert src.count(old) == 1, f"mutation anchor not found: {old}"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutant {fn}>", "exec"), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    caught = []
    for check, kw in PY_CHECKS[fn]:
        try:
            check(**kw)
        except Exception:  # noqa: BLE001  (a failing pin is what we want)
            caught.append(check.__name__)
    assert caught, f"no pin caught: {name}"
