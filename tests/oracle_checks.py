"""Pins for the CPU oracle, written as plain functions of an ``Oracle``.

Each check raises ``AssertionError`` when the oracle disagrees with something
fixed outside the oracle itself: a fact printed on the GSQ model card, a
hand-derived word pattern, a closed form, exact rational arithmetic on the raw
codes, or a numpy library product.  ``test_oracle_pins.py`` runs them against
the real oracle; ``test_oracle_mutants.py`` runs them against deliberately
broken copies to show that each plausible mistake is caught by at least one.
"""
from __future__ import annotations

import json
import os
from decimal import ROUND_HALF_UP, Decimal
from fractions import Fraction

import numpy as np

from w3a16_gemv_b200.inputs import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name: str):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16(values) -> np.ndarray:
    """bf16 bit patterns of values that are exactly representable (asserted)."""
    a = np.asarray(values, dtype=np.float32)
    b = f32_to_bf16_bits(a)
    assert np.array_equal(bf16_bits_to_f32(b), a), "fixture value not exact in bf16"
    return b


def _block_codes(spec) -> np.ndarray:
    c = np.zeros(32, dtype=np.uint8)
    if spec == "all7":
        c[:] = 7
    elif spec == "jmod8":
        c[:] = np.arange(32) % 8
    else:
        for j, v in spec.items():
            c[int(j)] = v
    return c


# --- the storage example and the bits-per-weight figure on the card ----------------

def check_worked_example_shapes(orc):
    g = load_golden("gsq_storage_example.json")
    N, K = g["original_shape"]
    assert [N, orc.words_per_row(K)] == g["weight_shape"]
    assert [N, orc.groups_per_row(K)] == g["weight_scale_shape"]
    assert g["quantization_config"]["weight_scale_group_size"] == 128
    # pack a few full-width rows and check the produced width (and no overrun)
    rng = np.random.Generator(np.random.PCG64(1))
    codes = rng.integers(0, 8, size=(3, K), dtype=np.uint8)
    packed = orc.pack(codes)
    assert packed.shape == (3, g["weight_shape"][1])


def check_bits_per_weight(orc):
    g = load_golden("gsq_storage_example.json")
    N, K = g["original_shape"]
    for (n, k) in [(N, K), (4096, 4096), (8192, 28672), (1024, 8192), (1, 128)]:
        bits = (4 * n * orc.words_per_row(k) + 2 * n * orc.groups_per_row(k)) * 8
        assert Fraction(bits, n * k) == Fraction(25, 8)  # 3 + 16/128 exactly
    printed = Decimal(g["effective_bits_per_weight_printed"])
    assert Decimal("3.125").quantize(Decimal("0.01"), rounding=ROUND_HALF_UP) == printed


# --- bit order ------------------------------------------------------------------------

def check_golden_word_patterns(orc):
    g = load_golden("bitorder_words.json")
    for case in g["cases"]:
        codes = _block_codes(case["codes"])[None, :]
        want = np.array([int(w, 16) for w in case["words"]], dtype=np.uint32)[None, :]
        got = orc.pack(codes)
        assert np.array_equal(got, want), f"{case['name']}: {[hex(v) for v in got[0]]}"
        assert np.array_equal(orc.unpack(want, 32), codes), case["name"]


def _block_as_int(words) -> int:
    return int(words[0]) | (int(words[1]) << 32) | (int(words[2]) << 64)


def check_block_is_base8_number(orc):
    # one-hot codes: every position j, every value v
    for j in range(32):
        codes = np.zeros((8, 32), dtype=np.uint8)
        codes[:, j] = np.arange(8)
        packed = orc.pack(codes)
        for v in range(8):
            assert _block_as_int(packed[v]) == v * 8 ** j, (j, v)
    # random blocks (several blocks per row): block t of a row = sum_j c_j 8^j
    rng = np.random.Generator(np.random.PCG64(2))
    codes = rng.integers(0, 8, size=(5, 256), dtype=np.uint8)
    packed = orc.pack(codes)
    for n in range(5):
        for t in range(8):
            digits = codes[n, 32 * t:32 * t + 32]
            assert _block_as_int(packed[n, 3 * t:3 * t + 3]) == sum(int(c) * 8 ** j for j, c in enumerate(digits))


def check_round_trips(orc):
    rng = np.random.Generator(np.random.PCG64(3))
    for N, K in [(1, 128), (3, 256), (7, 1152), (2, 4096)]:
        codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
        assert np.array_equal(orc.unpack(orc.pack(codes), K), codes)
        words = rng.integers(0, 2 ** 32, size=(N, orc.words_per_row(K)), dtype=np.uint64).astype(np.uint32)
        assert np.array_equal(orc.pack(orc.unpack(words, K)), words)


# --- signed level and scale grouping --------------------------------------------------

def check_levels_and_offset(orc):
    codes = np.tile(np.arange(8, dtype=np.uint8), 16)[None, :]  # K = 128
    w = orc.dequant_f32(orc.pack(codes), _bf16([[1.0]]), 128)
    assert np.array_equal(w[0, :8], np.arange(-4, 4, dtype=np.float32))
    gsq = load_golden("gsq_storage_example.json")["gsq_levels"]
    assert list(w[0, 2:7]) == gsq  # codes 2..6 are the GSQ levels -2..+2


def check_group_scales_exact(orc):
    rng = np.random.Generator(np.random.PCG64(4))
    N, K = 3, 512
    G = K // 128
    codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    # a distinct power of two per (row, group), so any wrong row/group index shows
    exps = np.arange(N * G).reshape(N, G) - 6
    scales = _bf16(np.ldexp(1.0, exps))
    w = orc.dequant_f32(orc.pack(codes), scales, K)
    for n in range(N):
        for k in range(K):
            assert w[n, k] == (int(codes[n, k]) - 4) * 2.0 ** float(exps[n, k // 128]), (n, k)
    # random bf16 scales: q*s is exact in fp32, so it equals the fp64 product
    scales = f32_to_bf16_bits(rng.lognormal(-4, 1.0, size=(N, G)).astype(np.float32))
    w = orc.dequant_f32(orc.pack(codes), scales, K)
    s64 = bf16_bits_to_f32(scales).astype(np.float64)
    for n in range(N):
        for k in range(K):
            assert float(w[n, k]) == (int(codes[n, k]) - 4) * s64[n, k // 128]


# --- the product ----------------------------------------------------------------------

# The single-threaded product and its multi-threaded variant (rows spread over threads) are
# both held to every pin of the product.
PRODUCT_THREADS = (None, 2)

def check_brute_force_tiny(orc):
    rng = np.random.Generator(np.random.PCG64(5))
    for M, N, K in [(1, 1, 128), (2, 3, 128), (2, 3, 256), (3, 2, 384)]:
        G = K // 128
        codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
        xi = rng.integers(-8, 9, size=(M, K))
        se = rng.integers(-4, 3, size=(N, G))
        for threads in PRODUCT_THREADS:
            y = orc.gemm_f64(_bf16(xi), orc.pack(codes), _bf16(np.ldexp(1.0, se)), threads=threads)
            assert y.shape == (M, N)
            for m in range(M):
                for n in range(N):
                    exact = sum(Fraction(int(xi[m, k])) * (int(codes[n, k]) - 4) *
                                Fraction(2) ** int(se[n, k // 128]) for k in range(K))
                    assert Fraction(y[m, n]) == exact, (M, N, K, m, n, threads)


def check_position_probe(orc):
    rng = np.random.Generator(np.random.PCG64(6))
    N, K = 5, 256
    codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    scales = f32_to_bf16_bits(rng.lognormal(-4, 0.5, size=(N, K // 128)).astype(np.float32))
    s = bf16_bits_to_f32(scales).astype(np.float64)
    packed = orc.pack(codes)
    eye = np.eye(K, dtype=np.float32)
    for threads in PRODUCT_THREADS:
        y = orc.gemm_f64(_bf16(eye), packed, scales, threads=threads)  # row k of x is e_k
        for k in range(K):
            for n in range(N):
                assert y[k, n] == (int(codes[n, k]) - 4) * s[n, k // 128], (k, n, threads)


def check_closed_forms(orc):
    rng = np.random.Generator(np.random.PCG64(7))
    M, N, K = 3, 4, 640
    xi = rng.integers(-16, 17, size=(M, K))
    x = _bf16(xi)
    # all codes 4 -> q = 0 -> y == 0 exactly
    y = orc.gemm_f64(x, orc.pack(np.full((N, K), 4, np.uint8)), _bf16(np.full((N, K // 128), 0.375)))
    assert np.all(y == 0.0)
    # constant code c and scale s -> y[m,n] = (c-4) * s * sum_k x[m,k]
    for c, s in [(7, 0.25), (0, 1.5), (2, 3.0)]:
        y = orc.gemm_f64(x, orc.pack(np.full((N, K), c, np.uint8)), _bf16(np.full((N, K // 128), s)))
        for m in range(M):
            assert np.all(y[m] == (c - 4) * s * int(xi[m].sum()))
    # x = 1, s = 1 -> y[0,n] = sum_k q[n,k]
    codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    for threads in PRODUCT_THREADS:
        y = orc.gemm_f64(_bf16(np.ones((1, K))), orc.pack(codes), _bf16(np.ones((N, K // 128))), threads=threads)
        assert np.array_equal(y[0], np.array([int(codes[n].astype(np.int64).sum()) - 4 * K for n in range(N)],
                                             float))
    # the multi-threaded product on a constant code
    y = orc.gemm_f64(x, orc.pack(np.full((N, K), 7, np.uint8)), _bf16(np.full((N, K // 128), 0.25)), threads=3)
    for m in range(M):
        assert np.all(y[m] == 3 * 0.25 * int(xi[m].sum()))


def check_numpy_cross_check(orc):
    rng = np.random.Generator(np.random.PCG64(8))
    M, N, K = 4, 37, 1024
    codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    scales = f32_to_bf16_bits(rng.lognormal(-4, 0.5, size=(N, K // 128)).astype(np.float32))
    x = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    W = (codes.astype(np.float64) - 4.0) * np.repeat(bf16_bits_to_f32(scales).astype(np.float64), 128, axis=1)
    X = bf16_bits_to_f32(x).astype(np.float64)
    ref = X @ W.T
    y = orc.gemm_f64(x, orc.pack(codes), scales)
    assert np.all(np.abs(y - ref) <= 1e-12 * (np.abs(X) @ np.abs(W).T) + 1e-300)
    yt = orc.gemm_f64(x, orc.pack(codes), scales, threads=3)
    assert np.all(np.abs(yt - ref) <= 1e-12 * (np.abs(X) @ np.abs(W).T) + 1e-300)
    # sampled entries agree with the full product bit for bit
    ms, ns = rng.integers(0, M, 50), rng.integers(0, N, 50)
    assert np.array_equal(orc.gemm_f64_entries(x, orc.pack(codes), scales, ms, ns), y[ms, ns])


def check_weight_row_norms(orc):
    K = 256  # sqrt(K) = 16 exactly
    codes = np.stack([np.full(K, 7), np.full(K, 0), np.full(K, 4)]).astype(np.uint8)
    scales = _bf16([[0.5, 0.5], [0.25, 0.25], [8.0, 8.0]])
    norms = orc.weight_row_norms(orc.pack(codes), scales, K)
    assert list(norms) == [3 * 0.5 * 16, 4 * 0.25 * 16, 0.0]


def check_rejects_bad_arguments(orc):
    assert orc.words_per_row(100) == -1 and orc.groups_per_row(96) == -1
    bad = np.zeros((1, 128), np.uint8)
    bad[0, 5] = 8
    try:
        orc.pack(bad)
    except ValueError:
        pass
    else:
        raise AssertionError("a code of 8 was accepted")


def check_ct4_container_words(orc):
    """The 4-bit container pins: hand-derived words for packing and for the re-pack with clamping."""
    g = load_golden("ct4_container_words.json")
    for case in g["pack_cases"]:
        codes = np.full((1, 128), 4, dtype=np.uint8)  # level 0 everywhere
        for pos, level in case["levels"].items():
            codes[0, int(pos)] = level + 4
        words = orc.pack_ct4(codes)
        assert words.shape == (1, 16), case["name"]
        assert int(words[0, 0]) == int(case["word"], 16), case["name"]
        assert np.all(words[0, 1:] == 0x88888888), case["name"]
    for case in g["repack_cases"]:
        ct4 = np.full((1, 16), 0x88888888, dtype=np.uint32)
        ct4[0, 0] = int(case["word"], 16)
        packed, clamped = orc.repack_ct4(ct4, 128)
        codes = orc.unpack(packed, 128)
        assert list(codes[0, :8]) == case["codes"], case["name"]
        assert np.all(codes[0, 8:] == 4), case["name"]
        assert clamped == case["out_of_range"], case["name"]


def check_ct4_repack_equals_direct_pack(orc):
    """Re-packing the container of any codes gives the exact-width words of the same codes."""
    rng = np.random.Generator(np.random.PCG64(7))
    codes = rng.integers(0, 8, size=(5, 384), dtype=np.uint8)
    packed, clamped = orc.repack_ct4(orc.pack_ct4(codes), 384)
    assert clamped == 0
    assert np.array_equal(packed, orc.pack(codes))


# --- the kernel-native block layout ---------------------------------------------------

def check_native_layout_golden_words(orc):
    """Hand-derived positions of the native block order (tests/golden/native_layout_words.json)."""
    g = json.load(open(os.path.join(GOLDEN, "native_layout_words.json")))
    N, K = g["N"], g["K"]
    W = orc.words_per_row(K)
    packed = (1000 * np.arange(N, dtype=np.uint32)[:, None] + np.arange(W, dtype=np.uint32)[None, :] + 1)
    native = orc.native_from_packed(packed.astype(np.uint32), K)
    assert native.size == g["native_words"] == orc.native_words(N, K)
    for e in g["entries"]:
        assert int(native[e["index"]]) == e["value"], e


def check_native_layout_round_trip_and_padding(orc):
    rng = np.random.Generator(np.random.PCG64(21))
    for N, K in [(32, 128), (33, 256), (100, 384), (7, 1152)]:
        packed = orc.pack(rng.integers(0, 8, size=(N, K), dtype=np.uint8))
        native = orc.native_from_packed(packed, K)
        assert native.size == -(-N // 32) * 32 * orc.words_per_row(K)
        assert np.array_equal(orc.packed_from_native(native, N, K), packed)
        # every word of a real row appears once; padded rows are zero
        assert np.array_equal(np.sort(native[native != 0]), np.sort(packed[packed != 0].ravel()))
    assert orc.native_words(5, 100) == -1


def check_native_lane_blocks_decode_to_their_rows(orc):
    """Read as a little-endian 96-bit integer, lane l's words 3h..3h+2 of group g of block b are
    sum_j c[32b + l/4 + 8h, 128g + 32(l%4) + j] * 8^j (the base-8 form of the row bit order)."""
    rng = np.random.Generator(np.random.PCG64(22))
    N, K = 70, 256
    codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    native = orc.native_from_packed(orc.pack(codes), K)
    G = K // 128
    for b in range(-(-N // 32)):
        for gg in range(G):
            for lane in range(32):
                for h in range(4):
                    base = ((b * G + gg) * 32 + lane) * 12 + 3 * h
                    v = int(native[base]) | int(native[base + 1]) << 32 | int(native[base + 2]) << 64
                    row = 32 * b + lane // 4 + 8 * h
                    want = 0
                    if row < N:
                        for j in range(32):
                            want += int(codes[row, 128 * gg + 32 * (lane % 4) + j]) * 8 ** j
                    assert v == want, (b, gg, lane, h)


ALL_CHECKS = [
    check_worked_example_shapes,
    check_bits_per_weight,
    check_golden_word_patterns,
    check_block_is_base8_number,
    check_round_trips,
    check_levels_and_offset,
    check_group_scales_exact,
    check_brute_force_tiny,
    check_position_probe,
    check_closed_forms,
    check_numpy_cross_check,
    check_weight_row_norms,
    check_rejects_bad_arguments,
    check_ct4_container_words,
    check_ct4_repack_equals_direct_pack,
    check_native_layout_golden_words,
    check_native_layout_round_trip_and_padding,
    check_native_lane_blocks_decode_to_their_rows,
]
