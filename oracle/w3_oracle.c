/*
 * w3_oracle.c -- plain, slow CPU oracle for the W3A16 group-128 format.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link, load or call this file.  Only the
 * tests, the smoke check and the CPU-baseline leg of the benchmark use it.  It
 * shares no code with the CUDA kernels: it is written at the level of single
 * bits and single multiply-adds so that a reader can check it against the
 * format definition by eye.
 *
 * What it follows (all from the GSQ model card "Llama-3.1-70B-Instruct-3Bit-GSQ",
 * section "Storage layout (why the HF UI shows I32 + BF16)" and the
 * quantization_config block under it):
 *   - a weight of shape [N, K] (out_features, in_features) is stored as uint3
 *     codes with exact-width packing: no code is padded into a wider field, so
 *     a row of K codes takes K*3/32 int32 words ("8192 x 3 / 32 = 768");
 *   - one bf16 scale per group of 128 consecutive weights along K, shape
 *     [N, K/128] ("8192 / 128 = 64"), weight_scale_type "group",
 *     weight_scale_group_size 128;
 *   - symmetric, has_zero_point false: a weight is (signed level) x scale;
 *   - section "Quantization details": the GSQ codebook is the 5-level integer
 *     set {-2,-1,0,1,+2} times the group scale.
 *
 * Readings where the card is silent (each is also listed with the design notes):
 *   - bit order: one LSB-first bitstream per row.  Code k of row n occupies
 *     stream bits 3k, 3k+1, 3k+2 (bit 0 of the code first), and stream bit b
 *     is bit (b mod 32) of word floor(b/32) of that row.  Equivalently, the 3
 *     words of each 32-code block, read as one little-endian 96-bit integer,
 *     equal sum_j c_j * 8^j.
 *   - signed level: q = c - 4 for every code c in 0..7, so the GSQ levels
 *     -2..2 are the codes 2..6.
 *   - int32 container: a raw 32-bit pattern (handled here as uint32_t).
 *   - the product y = x * W^T (nn.Linear convention), W[n,k] = q[n,k]*s[n,k/128].
 *
 * Precision: the fp32 dequantized weight q*s is exact (|q| <= 4 is a 3-bit
 * integer and a bf16 scale has 8 significant bits, so the product has at most
 * 11), and the matrix product is accumulated in fp64 in plain k order.
 *
 * Every function returns 0 on success and -1 on an invalid argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 128

/* Words of packed storage per row: K codes x 3 bits / 32 bits per word. */
int64_t oracle_words_per_row(int64_t K) {
    if (K <= 0 || (K * 3) % 32 != 0) return -1;
    return K * 3 / 32;
}

/* Scale groups per row: one bf16 scale per 128 weights along K. */
int64_t oracle_groups_per_row(int64_t K) {
    if (K <= 0 || K % ORACLE_GROUP != 0) return -1;
    return K / ORACLE_GROUP;
}

/* bf16 is the upper half of an IEEE binary32: widen by appending 16 zero bits. */
static float bf16_bits_to_float(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Read one bit of row `row` (a pointer to its first word) at stream position b. */
static unsigned stream_bit(const uint32_t *row, int64_t b) {
    return (unsigned)((row[b / 32] >> (b % 32)) & 1u);
}

/* The 3-bit code c[n,k], assembled bit by bit from the row's bitstream. */
static unsigned code_at(const uint32_t *row, int64_t k) {
    unsigned c = 0;
    for (int i = 0; i < 3; ++i)
        c |= stream_bit(row, 3 * k + i) << i;
    return c;
}

/* codes: [N,K] bytes, each 0..7.  packed: [N, K*3/32] words, fully written. */
int oracle_pack(const uint8_t *codes, uint32_t *packed, int64_t N, int64_t K) {
    int64_t W = oracle_words_per_row(K);
    if (!codes || !packed || N < 0 || W < 0) return -1;
    for (int64_t n = 0; n < N; ++n) {
        uint32_t *row = packed + n * W;
        for (int64_t w = 0; w < W; ++w) row[w] = 0;
        for (int64_t k = 0; k < K; ++k) {
            unsigned c = codes[n * K + k];
            if (c > 7) return -1;
            for (int i = 0; i < 3; ++i) {
                int64_t b = 3 * k + i;
                uint32_t bit = (c >> i) & 1u;
                row[b / 32] |= bit << (b % 32);
            }
        }
    }
    return 0;
}

/* packed: [N, K*3/32] words.  codes: [N,K] bytes, each written with 0..7. */
int oracle_unpack(const uint32_t *packed, uint8_t *codes, int64_t N, int64_t K) {
    int64_t W = oracle_words_per_row(K);
    if (!codes || !packed || N < 0 || W < 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            codes[n * K + k] = (uint8_t)code_at(packed + n * W, k);
    return 0;
}

/* w[n,k] = (c[n,k] - 4) * s[n, k/128] in fp32 (exact).  scales: bf16 bits [N, K/128]. */
int oracle_dequant_f32(const uint32_t *packed, const uint16_t *scales, float *w,
                       int64_t N, int64_t K) {
    int64_t W = oracle_words_per_row(K), G = oracle_groups_per_row(K);
    if (!packed || !scales || !w || N < 0 || W < 0 || G < 0) return -1;
    for (int64_t n = 0; n < N; ++n) {
        const uint32_t *row = packed + n * W;
        for (int64_t k = 0; k < K; ++k) {
            int q = (int)code_at(row, k) - 4;
            float s = bf16_bits_to_float(scales[n * G + k / ORACLE_GROUP]);
            w[n * K + k] = (float)q * s;
        }
    }
    return 0;
}

/* One output element: sum over k of x[m,k] * W[n,k], fp64, k ascending. */
static double dot_row(const uint16_t *x, const float *wrow, int64_t m, int64_t K) {
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k)
        acc += (double)bf16_bits_to_float(x[m * K + k]) * (double)wrow[k];
    return acc;
}

/* Dequantize row n of W into wrow (K floats). */
static void dequant_row(const uint32_t *packed, const uint16_t *scales, int64_t n,
                        int64_t K, float *wrow) {
    int64_t W = K * 3 / 32, G = K / ORACLE_GROUP;
    const uint32_t *row = packed + n * W;
    for (int64_t k = 0; k < K; ++k) {
        int q = (int)code_at(row, k) - 4;
        wrow[k] = (float)q * bf16_bits_to_float(scales[n * G + k / ORACLE_GROUP]);
    }
}

/*
 * y[m,n] = sum_k x[m,k] * W[n,k]   (y = x W^T), y in fp64, row-major [M,N].
 * x: bf16 bits [M,K]; packed: [N,K*3/32]; scales: bf16 bits [N,K/128].
 */
int oracle_gemm_f64(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                    double *y, int64_t M, int64_t N, int64_t K) {
    if (!x || !packed || !scales || !y || M < 0 || N < 0) return -1;
    if (oracle_words_per_row(K) < 0 || oracle_groups_per_row(K) < 0) return -1;
    float *wrow = (float *)malloc((size_t)K * sizeof(float));
    if (!wrow) return -1;
    for (int64_t n = 0; n < N; ++n) {
        dequant_row(packed, scales, n, K, wrow);
        for (int64_t m = 0; m < M; ++m)
            y[m * N + n] = dot_row(x, wrow, m, K);
    }
    free(wrow);
    return 0;
}

/*
 * The same y as oracle_gemm_f64, with the output rows n spread over `threads`
 * OpenMP threads (0: the OpenMP default, all cores).  Every element is still
 * one fp64 dot product in ascending k computed by one thread, so the result is
 * bit-identical to oracle_gemm_f64; only the wall time changes.
 */
int oracle_gemm_f64_threads(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                            double *y, int64_t M, int64_t N, int64_t K, int threads) {
    if (!x || !packed || !scales || !y || M < 0 || N < 0 || threads < 0) return -1;
    if (oracle_words_per_row(K) < 0 || oracle_groups_per_row(K) < 0) return -1;
    int failed = 0;
#ifdef _OPENMP
    const int nt = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel num_threads(nt)
#endif
    {
        float *wrow = (float *)malloc((size_t)K * sizeof(float));
        if (!wrow) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
        for (int64_t n = 0; n < N; ++n) {
            if (!wrow) continue;
            dequant_row(packed, scales, n, K, wrow);
            for (int64_t m = 0; m < M; ++m)
                y[m * N + n] = dot_row(x, wrow, m, K);
        }
        free(wrow);
    }
    return failed ? -1 : 0;
}

/* Threads oracle_gemm_f64_threads(..., 0) uses: the OpenMP default (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * The same product for a list of `count` single entries (ms[i], ns[i]), for
 * checking sampled outputs of shapes too large for the full triple loop.
 */
int oracle_gemm_f64_entries(const uint16_t *x, const uint32_t *packed,
                            const uint16_t *scales, int64_t M, int64_t N, int64_t K,
                            const int64_t *ms, const int64_t *ns, int64_t count,
                            double *out) {
    if (!x || !packed || !scales || !ms || !ns || !out || count < 0) return -1;
    if (oracle_words_per_row(K) < 0 || oracle_groups_per_row(K) < 0) return -1;
    float *wrow = (float *)malloc((size_t)K * sizeof(float));
    if (!wrow) return -1;
    for (int64_t i = 0; i < count; ++i) {
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) { free(wrow); return -1; }
        dequant_row(packed, scales, ns[i], K, wrow);
        out[i] = dot_row(x, wrow, ms[i], K);
    }
    free(wrow);
    return 0;
}

/* ||W[n,:]||_2 of the dequantized row, in fp64 (used by the output tolerance). */
int oracle_weight_row_norms(const uint32_t *packed, const uint16_t *scales,
                            int64_t N, int64_t K, double *out) {
    if (!packed || !scales || !out || N < 0) return -1;
    if (oracle_words_per_row(K) < 0 || oracle_groups_per_row(K) < 0) return -1;
    float *wrow = (float *)malloc((size_t)K * sizeof(float));
    if (!wrow) return -1;
    for (int64_t n = 0; n < N; ++n) {
        dequant_row(packed, scales, n, K, wrow);
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += (double)wrow[k] * (double)wrow[k];
        out[n] = sqrt(ss);
    }
    free(wrow);
    return 0;
}

/* ---- the 4-bit container written before the exact-width re-pack -------------------
 *
 * The card's note under "Storage layout" says that GSQ training first writes its
 * shards in the compressed-tensors pack-quantized format, the 3-bit codebook
 * padded into a 4-bit INT32 container, and that convert_to_humming.py re-packs
 * them into the exact-width storage above.  The card does not print that
 * container's layout.  Reading used here: eight 4-bit fields per int32 word,
 * LSB first (level k of a row in bits 4*(k mod 8) .. 4*(k mod 8)+3 of word k/8),
 * each field the signed level plus 8 (an unsigned nibble 0..15 for -8..7), so a
 * row of K levels takes K/8 words.
 */

/* Container words per row: K levels x 4 bits / 32 bits per word. */
int64_t oracle_ct4_words_per_row(int64_t K) {
    if (K <= 0 || K % 8 != 0) return -1;
    return K / 8;
}

/* codes [N,K] (0..7, level c - 4) -> container [N, K/8] words, fully written. */
int oracle_pack_ct4(const uint8_t *codes, uint32_t *ct4, int64_t N, int64_t K) {
    int64_t W = oracle_ct4_words_per_row(K);
    if (!codes || !ct4 || N < 0 || W < 0) return -1;
    for (int64_t n = 0; n < N; ++n) {
        uint32_t *row = ct4 + n * W;
        for (int64_t w = 0; w < W; ++w) row[w] = 0;
        for (int64_t k = 0; k < K; ++k) {
            unsigned c = codes[n * K + k];
            if (c > 7) return -1;
            int q = (int)c - 4;
            unsigned field = (unsigned)(q + 8);
            for (int i = 0; i < 4; ++i) {
                int64_t b = 4 * k + i;
                row[b / 32] |= ((field >> i) & 1u) << (b % 32);
            }
        }
    }
    return 0;
}

/* container [N, K/8] -> exact-width packed [N, 3K/32].  A level outside -4..3 has
 * no 3-bit code: it is clamped to the nearer of -4 and 3, and the number of such
 * levels is written to *out_of_range. */
int oracle_repack_ct4(const uint32_t *ct4, uint32_t *packed, int64_t N, int64_t K, int64_t *out_of_range) {
    int64_t W4 = oracle_ct4_words_per_row(K), W3 = oracle_words_per_row(K);
    if (!ct4 || !packed || !out_of_range || N < 0 || W4 < 0 || W3 < 0) return -1;
    *out_of_range = 0;
    for (int64_t n = 0; n < N; ++n) {
        const uint32_t *in = ct4 + n * W4;
        uint32_t *out = packed + n * W3;
        for (int64_t w = 0; w < W3; ++w) out[w] = 0;
        for (int64_t k = 0; k < K; ++k) {
            unsigned field = 0;
            for (int i = 0; i < 4; ++i)
                field |= stream_bit(in, 4 * k + i) << i;
            int q = (int)field - 8;
            if (q < -4) {
                q = -4;
                ++*out_of_range;
            } else if (q > 3) {
                q = 3;
                ++*out_of_range;
            }
            unsigned c = (unsigned)(q + 4);
            for (int i = 0; i < 3; ++i) {
                int64_t b = 3 * k + i;
                out[b / 32] |= ((c >> i) & 1u) << (b % 32);
            }
        }
    }
    return 0;
}

/* ---- the kernel-native block layout (a permutation of the packed words) ------------------
 *
 * The storage above keeps each row's words together.  The decode kernels read 32 rows at a
 * time, each of 32 lanes taking one 32-code block (3 words) of each of four rows, so this
 * library also defines an optional "native" order of the same words (the GLQ page's
 * decoder-native "kernel" layout is the precedent: an offline re-order of the checkpoint for
 * the kernel, behind the same format).  Rows are grouped in blocks of 32 (the last block
 * padded with zero rows); for block b, group g (128 codes), lane l = 4r + c (r = l / 4 in
 * 0..7, c = l % 4 in 0..3), word 3h + i (h in 0..3, i in 0..2):
 *     native[((b*G + g)*32 + l)*12 + 3h + i] = packed[row 32b + r + 8h][word 12g + 3c + i]
 * i.e. lane l holds 32-code block c of group g for rows r, r+8, r+16, r+24, in the row's own
 * bit order.  Size: ceil(N/32)*32 rows of 3K/32 words.
 */

/* Words of the native layout for an N x K weight (rows padded to a multiple of 32). */
int64_t oracle_native_words(int64_t N, int64_t K) {
    int64_t W = oracle_words_per_row(K);
    if (N < 0 || W < 0 || K % ORACLE_GROUP != 0) return -1;
    return (N + 31) / 32 * 32 * W;
}

/* packed [N, 3K/32] (row order) -> native (block order above); padded rows are zero. */
int oracle_native_from_packed(const uint32_t *packed, uint32_t *native, int64_t N, int64_t K) {
    int64_t W = oracle_words_per_row(K), G = oracle_groups_per_row(K), NW = oracle_native_words(N, K);
    if (!packed || !native || N < 0 || W < 0 || G < 0 || NW < 0) return -1;
    int64_t NB = (N + 31) / 32;
    for (int64_t b = 0; b < NB; ++b)
        for (int64_t g = 0; g < G; ++g)
            for (int l = 0; l < 32; ++l)
                for (int h = 0; h < 4; ++h)
                    for (int i = 0; i < 3; ++i) {
                        int64_t row = 32 * b + l / 4 + 8 * h;
                        int64_t word = 12 * g + 3 * (l % 4) + i;
                        native[((b * G + g) * 32 + l) * 12 + 3 * h + i] = row < N ? packed[row * W + word] : 0u;
                    }
    return 0;
}

/* native -> packed [N, 3K/32] (the inverse; padded rows are dropped). */
int oracle_packed_from_native(const uint32_t *native, uint32_t *packed, int64_t N, int64_t K) {
    int64_t W = oracle_words_per_row(K), G = oracle_groups_per_row(K), NW = oracle_native_words(N, K);
    if (!packed || !native || N < 0 || W < 0 || G < 0 || NW < 0) return -1;
    int64_t NB = (N + 31) / 32;
    for (int64_t b = 0; b < NB; ++b)
        for (int64_t g = 0; g < G; ++g)
            for (int l = 0; l < 32; ++l)
                for (int h = 0; h < 4; ++h)
                    for (int i = 0; i < 3; ++i) {
                        int64_t row = 32 * b + l / 4 + 8 * h;
                        int64_t word = 12 * g + 3 * (l % 4) + i;
                        if (row < N) packed[row * W + word] = native[((b * G + g) * 32 + l) * 12 + 3 * h + i];
                    }
    return 0;
}
