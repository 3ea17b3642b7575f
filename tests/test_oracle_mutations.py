"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a private copy of oracle/rans_oracle.c
(a transposed lane mapping, a dropped term, a shifted cumulative frequency,
wrong word order, wrong rounding, wrong exponent bias, a transposed scale
index ...), builds it into a temporary library and checks that at least one
of the pins in test_oracle_rans.py / test_oracle_formats.py fails on it.
Nothing here touches the real oracle build or any GPU.
"""
import os
import subprocess

import pytest

import test_oracle_formats as F
import test_oracle_huffman as H
import test_oracle_rans as R

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "rans_oracle.c")
HUFF_SRC = os.path.join(os.path.dirname(SRC), "huffman_oracle.c")

MUTATIONS = {
    # symbol j -> lane j mod 32 instead of 8-symbol groups per lane
    "lane_mapping": ("return GROUP_SYMS * (step / GROUP) + GROUP * lane + (step % GROUP);",
                     "return GROUP_SYMS * (step / GROUP) + lane * 1 + LANES * (step % GROUP);",
                     [R.test_hand_derived_examples]),
    # decoder drops the "- cum_s" term
    "decode_drops_cum": ("x[l] = (uint64_t)f[s] * (x[l] / PROB_TOTAL) + slot - cum[s];",
                         "x[l] = (uint64_t)f[s] * (x[l] / PROB_TOTAL) + slot;",
                         [R.test_every_tail_shape]),
    # cumulative frequency off by one for every symbol after the first
    "cum_shift": ("cum[s] = c;", "cum[s] = c + (s > 0 && c > 0);",
                  [R.test_hand_derived_examples, R.test_every_tail_shape]),
    # encoder swaps quotient and remainder
    "encode_swapped": ("x[l] = (x[l] / fs) * PROB_TOTAL + (x[l] % fs) + cum[s];",
                       "x[l] = (x[l] % fs) * PROB_TOTAL + (x[l] / fs) + cum[s];",
                       [R.test_hand_derived_examples]),
    # emitted words appended instead of prepended (wrong order for the decoder)
    "word_order": ("words[words_cap - 1 - w] = (uint16_t)(x[l] & 0xFFFFu);",
                   "words[words_cap - 1 - (w ^ 1)] = (uint16_t)(x[l] & 0xFFFFu);",
                   [R.test_every_tail_shape]),
    # renormalisation reads a word only once the state is far too small
    "renorm_threshold": ("if (x[l] < STATE_LOW) {\n                if (p >= n_words)",
                         "if (x[l] < 4096u) {\n                if (p >= n_words)",
                         [R.test_hand_derived_examples, R.test_every_tail_shape]),
    # frequency table rounds down instead of to nearest
    "freq_round_down": ("uint64_t q = (2u * counts[s] * PROB_TOTAL + n) / (2u * n);",
                        "uint64_t q = (counts[s] * PROB_TOTAL) / n;",
                        [R.test_quantized_table_rounds_to_nearest]),
    # bf16 rounding: half up instead of half to even
    "bf16_half_up": ("return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);",
                     "return (uint16_t)((b + 0x8000u) >> 16);",
                     [F.test_bf16_rne_all_high_halves_against_torch]),
    # E4M3 exponent bias 8 instead of 7
    "e4m3_bias": ("else v = ldexp(1.0 + m / 8.0, e - 7);", "else v = ldexp(1.0 + m / 8.0, e - 8);",
                  [F.test_e4m3_values_match_torch_all_codes]),
    # E4M3 subnormals scaled by 2^-7 instead of 2^-6
    "e4m3_subnormal": ("if (e == 0) v = ldexp(m / 8.0, -6);", "if (e == 0) v = ldexp(m / 8.0, -7);",
                       [F.test_e4m3_values_match_torch_all_codes]),
    # Int8 read as unsigned
    "int8_unsigned": ("return b < 128 ? (double)b : (double)b - 256.0;", "return (double)b;",
                      [F.test_int8_values_all_codes]),
    # scale indexed by column instead of row (transposed operand)
    "scale_index": ("out[k] = orc_dequant_one(dtype, sym[k], scales[i / cols]);",
                    "out[k] = orc_dequant_one(dtype, sym[k], scales[i % cols]);",
                    [F.test_dequant_int8_matches_torch]),
    # fp32 product rounded toward zero instead of to nearest even
    "mul_truncates": ("return (float)p;",
                      "float r = (float)p; if (fabs((double)r) > fabs(p)) r = nextafterf(r, 0.0f); return r;",
                      [F.test_fp32_mul_rn_against_numpy]),
    # frequency fix-up goes to the largest byte value instead of the largest f
    "freq_fixup_target": ("if (f[s] > f[best]) best = s;", "if (s > best && f[s]) best = s;",
                          [R.test_quantized_table_rounds_to_nearest]),
}


# the same, planted in a copy of oracle/huffman_oracle.c
HUFF_MUTATIONS = {
    # canonical codes: no shift when the length grows
    "canonical_no_shift": ("if (prev_len) c = (c + 1) << (L - prev_len);", "if (prev_len) c = c + 1;",
                           [H.test_rfc1951_canonical_codes]),
    # bits stored least significant first
    "bit_order": ("bits[l][nbits[l]++] = (uint8_t)((code[sym[j]] >> (L - 1 - b)) & 1u);",
                  "bits[l][nbits[l]++] = (uint8_t)((code[sym[j]] >> b) & 1u);",
                  [H.test_hand_derived_interleaving, H.test_hand_derived_interleaving_multibit_codes]),
    # refill threshold 11 bits instead of 12 (in the encoder's schedule)
    "refill_threshold": ("            if (held[l] < HUF_MAX_LEN) {\n                uint32_t w = 0;",
                         "            if (held[l] < HUF_MAX_LEN - 1) {\n                uint32_t w = 0;",
                         [H.test_hand_derived_interleaving, H.test_exhaustive_round_trip_tiny]),
    # package-merge keeps one item too few (suboptimal or invalid lengths)
    "package_merge_count": ("for (int i = 0; i < 2 * n - 2; ++i)", "for (int i = 0; i < 2 * n - 3; ++i)",
                            [H.test_textbook_lengths, H.test_lengths_optimal_against_dynamic_program]),
    # merge prefers packages on equal weights (still optimal, different lengths on ties)
    # is not a mistake; a merge that ignores package weights is:
    "merge_order": ("if (b >= p || (a < n && leaves[a].w <= next[b].w)) merged[k++] = leaves[a++];",
                    "if (b >= p || a < n) merged[k++] = leaves[a++];",
                    [H.test_textbook_lengths, H.test_lengths_optimal_against_dynamic_program]),
    # decoder skips the end check of the padding bits
    "no_padding_check": ("            if (q[l][(head[l] + b) % 64]) return HUF_ERR_CORRUPT;", "            ;",
                         [H.test_corruption_detected]),
}


@pytest.mark.parametrize("name", sorted(HUFF_MUTATIONS))
def test_huffman_pins_catch_planted_mistake(orc, tmp_path, name):
    old, new, pins = HUFF_MUTATIONS[name]
    src = open(HUFF_SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant = tmp_path / "mutant_huffman.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared",
                           "-fPIC", "-o", str(so), SRC, str(mutant), "-lm"])
    orc._use_library(str(so))
    try:
        caught = 0
        for pin in pins:
            try:
                if pin is H.test_lengths_optimal_against_dynamic_program:
                    for seed in range(6):
                        pin(orc, seed)
                else:
                    pin(orc)
            except (AssertionError, orc.OracleError, pytest.fail.Exception):
                caught += 1
        assert caught >= 1, f"planted mistake {name} passed every pin"
    finally:
        orc._use_library(None)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(orc, tmp_path, name):
    old, new, pins = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared",
                           "-fPIC", "-o", str(so), str(mutant), HUFF_SRC, "-lm"])
    orc._use_library(str(so))
    try:
        caught = 0
        for pin in pins:
            try:
                pin(orc)
            except (AssertionError, orc.OracleError):
                caught += 1
        assert caught >= 1, f"planted mistake {name} passed every pin"
    finally:
        orc._use_library(None)
