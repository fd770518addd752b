"""The pins have teeth: each plausible mistake planted in a copy of the oracle is caught.

Every mutant is a textual edit of ``oracle/w3_oracle.c`` compiled into a
temporary directory (the committed oracle is never touched).  The mutants stay
inside the buffers they are given, so a wrong answer is the only effect.
"""
import os
import subprocess

import pytest

import oracle
from oracle_checks import ALL_CHECKS

SRC = os.path.join(os.path.dirname(oracle.__file__), "w3_oracle.c")

# (name, text to replace, replacement, expected number of occurrences)
MUTANTS = [
    ("offset_c_minus_3", "code_at(row, k) - 4", "code_at(row, k) - 3", 2),
    ("code_bits_msb_first", "c |= stream_bit(row, 3 * k + i) << i;", "c |= stream_bit(row, 3 * k + i) << (2 - i);", 1),
    ("word_bits_msb_first_both_sides",
     "(row[b / 32] >> (b % 32)) & 1u", "(row[b / 32] >> (31 - b % 32)) & 1u", 1),
    ("group_index_reversed", "scales[n * G + k / ORACLE_GROUP]", "scales[n * G + (K - 1 - k) / ORACLE_GROUP]", 2),
    ("output_transposed", "y[m * N + n] = dot_row", "y[n * M + m] = dot_row", 2),
    ("dropped_last_term", "for (int64_t k = 0; k < K; ++k)\n        acc +=", "for (int64_t k = 0; k < K - 1; ++k)\n        acc +=", 1),
    ("x_reversed_along_k", "x[m * K + k]", "x[m * K + (K - 1 - k)]", 1),
    ("sign_flipped", "(int)code_at(row, k) - 4", "4 - (int)code_at(row, k)", 2),
    ("scale_not_applied_in_product",
     "wrow[k] = (float)q * bf16_bits_to_float(scales[n * G + k / ORACLE_GROUP]);", "wrow[k] = (float)q;", 1),
    ("words_per_row_4bit_container", "return K * 3 / 32;", "return K * 4 / 32;", 1),
    ("ct4_level_offset_7", "int q = (int)field - 8;", "int q = (int)field - 7;", 1),
    ("ct4_field_bits_msb_first", "field |= stream_bit(in, 4 * k + i) << i;",
     "field |= stream_bit(in, 4 * k + i) << (3 - i);", 1),
    ("ct4_clamp_not_counted", "                q = 3;\n                ++*out_of_range;", "                q = 3;", 1),
    ("ct4_pack_offset_7", "unsigned field = (unsigned)(q + 8);", "unsigned field = (unsigned)(q + 7);", 1),
    # the native block order, changed the same way in both directions (so the round trip still holds)
    ("native_lane_row_and_block_swapped", "int64_t row = 32 * b + l / 4 + 8 * h;",
     "int64_t row = 32 * b + l % 4 + 8 * h;", 2),
    ("native_row_stride_4", "int64_t row = 32 * b + l / 4 + 8 * h;", "int64_t row = 32 * b + l / 4 + 4 * h;", 2),
    ("native_words_of_lane_block", "int64_t word = 12 * g + 3 * (l % 4) + i;",
     "int64_t word = 12 * g + 3 * (l / 8) + i;", 2),
    # the row norms that scale every parity tolerance: a wrong norm would loosen the GPU tests
    ("norm_without_sqrt", "out[n] = sqrt(ss);", "out[n] = ss;", 1),
    ("norm_of_first_group_only", "for (int64_t k = 0; k < K; ++k) ss +=", "for (int64_t k = 0; k < 128; ++k) ss +=", 1),
    # the multi-threaded product (the full-size parity tests use it) dropping its last output row
    ("threads_skip_last_row", "        for (int64_t n = 0; n < N; ++n) {\n            if (!wrow) continue;",
     "        for (int64_t n = 0; n < N - 1; ++n) {\n            if (!wrow) continue;", 1),
]


def _pack_only_msb(src: str) -> str:
    # the word-bit-order mutant must change the packer consistently, or it is not plausible
    return src.replace("row[b / 32] |= bit << (b % 32);", "row[b / 32] |= bit << (31 - b % 32);")


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, count):
    src = open(SRC).read()
    assert src.count(old) == count, f"mutation site for {name} not found as expected"
    mutated = src.replace(old, new)
    if name == "word_bits_msb_first_both_sides":
        mutated = _pack_only_msb(mutated)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "libmutant.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so_path), str(c_path), "-lm"])
    orc = oracle.Oracle(oracle.load_library(str(so_path)))
    caught = []
    for check in ALL_CHECKS:
        try:
            check(orc)
        except (AssertionError, ValueError):
            caught.append(check.__name__)
    assert caught, f"mutant {name} passed every pin"
