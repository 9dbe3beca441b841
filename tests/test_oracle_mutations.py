"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle's C source, plants one mistake (a wrong index, a dropped term, a
transposed layout, a wrong exponent bias...), builds the copy on the CPU, swaps it in for the
real oracle and runs the pins: at least one pin must fail.  Nothing here touches a GPU.
"""
import os
import subprocess
import sys

import pytest

import oracle
from oracle import build as obuild
import tests.test_oracle_pins as pins
import tests.test_oracle_pins_fp8 as pins8

MUTATIONS = {
    "block index uses modulo": ("int64_t p = bt[(size_t)s * maxB + t / B];\n        int o = t % B;\n        double acc",
                                "int64_t p = bt[(size_t)s * maxB + t % B];\n        int o = t % B;\n        double acc"),
    "kv head grouping strided": ("int hk = h / g;", "int hk = h % Hkv;"),
    "scale dropped": ("x[t] = scale * acc;", "x[t] = acc;"),
    "denominator dropped": ("den += w;\n", "den += 1.0;\n"),
    "pool layout transposed": ("return (((size_t)p * Hkv + hk) * B + o) * D + d;",
                               "return (((size_t)p * B + o) * Hkv + hk) * D + d;"),
    "binary16 exponent bias": ("v = ldexp((double)(1024 + f), e - 25);",
                               "v = ldexp((double)(1024 + f), e - 24);"),
    "bfloat16 fraction width": ("v = ldexp((double)(128 + f), e - 134);",
                                "v = ldexp((double)(256 + f), e - 135);"),
    "kv_write offset swapped": ("int off = (int)(slot % B);", "int off = (int)(slot / B % B);"),
    "merge weight dropped": ("den += c * l[p];", "den += l[p];"),
    "one token too many": ("for (int t = 0; t < L; ++t) {\n        int64_t p = bt[(size_t)s * maxB + t / B];\n        int o = t % B;\n        double acc",
                           "for (int t = 0; t < L + (L % B != 0); ++t) {\n        int64_t p = bt[(size_t)s * maxB + t / B];\n        int o = t % B;\n        double acc"),
    "e4m3 exponent bias": ("v = ldexp((double)(8 + f), e - 10);",
                           "v = ldexp((double)(8 + f), e - 9);"),
    "e4m3 encoder truncates": ("int n = (int)nearbyint(a / ldexp(1.0, e - 3));",
                               "int n = (int)floor(a / ldexp(1.0, e - 3));"),
    "fp8 V written untransposed": (
        "return ((((size_t)blk * Hkv + h) * (size_t)(B / 16) + (size_t)(off / 16)) * D + d) * 16 +\n"
        "           (size_t)orc_v_slot(off % 16);",
        "return ((((size_t)blk * Hkv + h) * (size_t)(B / 16) + (size_t)(off / 16)) * 16 +\n"
        "           (size_t)orc_v_slot(off % 16)) * D + d;"),
    "fp8 V halves of a 32-token block swapped": (
        "(size_t)(B / 16) + (size_t)(off / 16)) * D + d) * 16 +",
        "(size_t)(B / 16) + (size_t)((B / 16 - 1) - off / 16)) * D + d) * 16 +"),
    "fp8 V slot order ignored": ("if (2 * (p / 4) + p % 2 + 8 * ((p / 2) % 2) == t) return p;",
                                 "if (p == t) return p;"),
    "fp8 K scale dropped": ("(orc_e4m3_to_f64(k_pool[(((size_t)p * Hkv + hk) * B + t % B) * D + d]) * ks)",
                            "(orc_e4m3_to_f64(k_pool[(((size_t)p * Hkv + hk) * B + t % B) * D + d]))"),
    "copy skips v pool": ("memmove((char *)v_pool + (size_t)dst * blk_bytes,",
                          "if (0) memmove((char *)v_pool + (size_t)dst * blk_bytes,"),
}

PINS = [
    pins.test_f16_decoder_matches_ieee_binary16_for_all_patterns,
    pins.test_bf16_decoder_matches_upper_half_of_binary32_for_all_patterns,
    lambda: pins.test_oracle_matches_bruteforce_contiguous_attention(4, 2, 32, 16),
    lambda: pins.test_oracle_matches_bruteforce_contiguous_attention(4, 2, 32, 32),
    pins.test_oracle_matches_torch_sdpa_fp64_on_contiguous_layout,
    pins.test_oracle_16bit_inputs_match_bruteforce_on_upcast_values,
    pins.test_golden_closed_form_example,
    pins.test_len1_returns_v0_exactly,
    pins.test_zero_query_or_zero_scale_gives_mean_of_values,
    pins.test_gqa_consecutive_grouping_equals_mha_with_replicated_kv_heads,
    pins.test_tokens_past_context_len_are_not_read,
    lambda: pins.test_split_lse_merge_equals_one_pass(48),
    pins.test_kv_write_places_rows_at_their_slots_and_nothing_else,
    pins.test_kv_copy_blocks_copies_whole_blocks,
    pins8.test_e4m3_decoder_matches_torch_for_all_codes,
    pins8.test_e4m3_encoder_matches_torch_rounding_in_range,
    lambda: pins8.test_kv_write_fp8_quantises_into_the_two_layouts(16),
    lambda: pins8.test_kv_write_fp8_quantises_into_the_two_layouts(32),
    lambda: pins8.test_fp8_decode_matches_bruteforce_on_dequantised_values(16),
    lambda: pins8.test_fp8_decode_matches_bruteforce_on_dequantised_values(32),
]


def _build_mutant(tmp_path, name, old, new):
    with open(obuild.SRC) as f:
        src = f.read()
    assert src.count(old) >= 1, "mutation anchor not found: %s" % name
    src = src.replace(old, new, 1)
    c = tmp_path / "mutant.c"
    so = tmp_path / "mutant.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(c),
                           "-o", str(so), "-lm"])
    return str(so)


def run_pins():
    """Run every pin; return the names of those that failed."""
    caught = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, oracle.OracleError):
            caught.append(getattr(pin, "__name__", "lambda"))
    return caught


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    """A mutant counts as caught when a pin fails or the mutant crashes its process (an
    out-of-bounds read planted by the mistake)."""
    old, new = MUTATIONS[name]
    so = _build_mutant(tmp_path, name, old, new)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys; import tests.test_oracle_mutations as m; "
            "c = m.run_pins(); print(c); sys.exit(3 if c else 0)")
    env = dict(os.environ, PKV_ORACLE_LIB=so, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode != 0, "no pin caught the planted mistake '%s'" % name


def test_unmutated_oracle_passes_every_pin():
    assert run_pins() == []
