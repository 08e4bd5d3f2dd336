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
