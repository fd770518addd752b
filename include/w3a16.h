/*
 * w3a16.h -- C ABI of libw3a16.so: W3A16 group-128 fused dequantize-and-multiply
 * for NVIDIA B200 (sm_100a).
 *
 * Format (GSQ model card "Llama-3.1-70B-Instruct-3Bit-GSQ", section "Storage
 * layout (why the HF UI shows I32 + BF16)" and its quantization_config block):
 *   - a linear layer's weight W has shape [N, K] = [out_features, in_features];
 *   - it is stored as uint3 codes with exact-width packing, 32 codes in 3
 *     int32 words, so `packed` is [N, 3K/32] int32, row-major ("8192 x 3 / 32
 *     = 768" in the card's gate_proj example);
 *   - one bf16 scale per group of 128 consecutive weights along K, so
 *     `scales` is [N, K/128] bf16, row-major ("8192 / 128 = 64");
 *   - symmetric, no zero point: W[n,k] = (c[n,k] - 4) * scales[n, k/128].
 *     The GSQ codebook (section "Quantization details") uses the levels
 *     -2..+2, i.e. codes 2..6; codes 0, 1 and 7 (levels -4, -3, +3) are valid too.
 *
 * Bit order (the card does not print one; this library fixes it): each row is
 * one LSB-first bitstream.  Code k occupies stream bits 3k..3k+2, bit 0 of
 * the code first, and stream bit b is bit (b mod 32) of word b/32 of the row.
 * Read as one little-endian 96-bit integer, the 3 words of every 32-code block
 * equal sum_j c_j * 8^j.  Codes 10 and 21 of each block straddle a word boundary.
 *
 * Conventions for every entry point:
 *   - all array pointers are DEVICE pointers (cudaMalloc'd or torch CUDA
 *     tensors) on the current device; the caller owns every buffer.  The
 *     only device memory the library allocates is the scratch of w3a16_gemm
 *     (at most 64 KB per SM, for partial sums), taken from and returned to a
 *     private stream-ordered pool on `stream` within the call, so calls on
 *     different streams never share it;
 *   - bf16 values are passed as their 16-bit patterns (uint16_t);
 *   - every array pointer must be 16-byte aligned (W3_ERR_ALIGN otherwise);
 *   - calls only enqueue work on `stream` (NULL = the legacy default stream)
 *     and return immediately; results are visible after the stream is
 *     synchronised;
 *   - the return value is the status; no call aborts, throws or exits;
 *   - arguments are checked on the host before anything is launched; a
 *     failing check returns an error and enqueues nothing;
 *   - a device-side wait that runs out of time (a hardware or driver fault,
 *     never expected) records W3_ERR_TIMEOUT in a per-device flag that
 *     w3_check_device_error() reports.
 */
#ifndef W3A16_H
#define W3A16_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same object as cudaStream_t; declared here so this header needs no CUDA headers. */
typedef struct CUstream_st *w3_stream_t;

typedef enum w3_status {
    W3_OK = 0,
    W3_ERR_NULL = 1,        /* a required pointer is NULL */
    W3_ERR_SHAPE = 2,       /* a size is out of range: M, N < 1, K < 128, K % 128 != 0, or too large */
    W3_ERR_ALIGN = 3,       /* an array pointer is not 16-byte aligned */
    W3_ERR_CUDA = 4,        /* the CUDA runtime reported an error (launch, device query) */
    W3_ERR_UNSUPPORTED = 5, /* the current device is not sm_100 (B200/GB200) */
    W3_ERR_TIMEOUT = 6,     /* a bounded device-side wait gave up (see w3_check_device_error) */
    W3_ERR_ALIAS = 7        /* the output overlaps an input */
} w3_status;

/* A short English description of a status; never NULL. */
const char *w3_status_string(w3_status status);

/* Version of this ABI (incremented on any incompatible change). */
int32_t w3_abi_version(void);

/* int32 words per packed row, 3K/32; -1 if K is not a positive multiple of 128. */
int64_t w3_packed_words_per_row(int64_t K);

/* bf16 scales per row, K/128; -1 if K is not a positive multiple of 128. */
int64_t w3_groups_per_row(int64_t K);

/*
 * w3_pack -- codes [N,K] uint8 (values 0..7; the upper 5 bits of each byte are
 * ignored) -> packed [N, 3K/32] int32 in the bit order above.
 * Storage layout from the card's "Storage layout" section.  Every output word
 * is written.  Errors: W3_ERR_NULL, W3_ERR_SHAPE (N < 1, K not a positive
 * multiple of 128), W3_ERR_ALIGN, W3_ERR_ALIAS (codes and packed overlap),
 * W3_ERR_UNSUPPORTED, W3_ERR_CUDA.
 */
w3_status w3_pack(const uint8_t *codes, int32_t *packed, int64_t N, int64_t K, w3_stream_t stream);

/*
 * w3_unpack -- packed [N, 3K/32] int32 -> codes [N,K] uint8 (each 0..7).
 * The inverse of w3_pack (same section of the card).  Same errors as w3_pack.
 */
w3_status w3_unpack(const int32_t *packed, uint8_t *codes, int64_t N, int64_t K, w3_stream_t stream);

/*
 * w3_repack_ct4 -- 4-bit container [N, K/8] int32 -> packed [N, 3K/32] int32 in
 * the exact-width format above.  The card's note under "Storage layout" says
 * GSQ training first writes shards in the compressed-tensors pack-quantized
 * format, the 3-bit codebook padded into a 4-bit INT32 container, and that
 * convert_to_humming.py re-packs them into the exact-width storage; it prints
 * no container layout.  Layout read here: eight 4-bit fields per int32, LSB
 * first (level k of a row in bits 4*(k%8)..4*(k%8)+3 of word k/8), each field
 * the signed level plus 8.  A level outside -4..3 has no 3-bit code: it is
 * clamped to -4 or 3, and if `out_of_range` (a device int64, 8-byte aligned)
 * is not NULL the call sets it to the number of clamped levels (stream-
 * ordered).  Scales are unchanged by the re-pack.  Errors: W3_ERR_NULL,
 * W3_ERR_SHAPE (N < 1, K not a positive multiple of 128), W3_ERR_ALIGN,
 * W3_ERR_ALIAS, W3_ERR_UNSUPPORTED, W3_ERR_CUDA.
 */
w3_status w3_repack_ct4(const int32_t *ct4, int32_t *packed, int64_t N, int64_t K, int64_t *out_of_range,
                        w3_stream_t stream);

/*
 * w3_dequant_f32 -- w[n,k] = (c[n,k] - 4) * scales[n, k/128] as fp32 [N,K].
 * The symmetric group-wise dequantization of the card's quantization_config
 * (weight_scale_type "group", weight_scale_group_size 128, has_zero_point
 * false).  The product is exact in fp32.  Meant for checking and debugging;
 * the product entry point below never materialises W.  Same errors as w3_pack.
 */
w3_status w3_dequant_f32(const int32_t *packed, const uint16_t *scales, float *w,
                         int64_t N, int64_t K, w3_stream_t stream);

/*
 * w3a16_gemm -- y = x * W^T (the nn.Linear product of the card's quantized
 * Linear layers), with W dequantized on the fly and never written to memory.
 *   x      [M,K] bf16, row-major
 *   packed [N, 3K/32] int32, scales [N, K/128] bf16 (the format above)
 *   y      [M,N] bf16, row-major; every element is written
 * Arithmetic: fp32 accumulation; the result is rounded once to bf16 (nearest
 * even).  For M <= 16, and for M <= 32 when N >= 256, the weight enters the
 * products exactly (q and the scale are applied in fp32; K may be split over
 * several thread blocks, whose fp32 partial sums are added in a fixed order);
 * for larger M each weight is first rounded to bf16(q*s) and fed to the
 * tensor cores.  Repeated calls
 * with the same arguments give bit-identical y (no floating-point atomics).
 * Errors: W3_ERR_NULL, W3_ERR_SHAPE (M, N < 1; K < 128 or K % 128 != 0;
 * M*K, N*K or M*N above 2^40), W3_ERR_ALIGN, W3_ERR_ALIAS (y overlaps x,
 * packed or scales), W3_ERR_UNSUPPORTED, W3_ERR_CUDA.
 */
w3_status w3a16_gemm(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y,
                     int64_t M, int64_t N, int64_t K, w3_stream_t stream);

/*
 * w3a16_gemm_noalloc -- the same product y = x * W^T as w3a16_gemm, with the
 * same arguments, checks, errors and results, that allocates nothing: the
 * 32-wide tensor-core decode (route "decode_tc32": 17 <= M <= 32, N >= 256)
 * keeps its fp32 partial sums in a fixed scratch array inside the library
 * (about 10.5 MB of device memory per device, sized for up to 160 SMs) instead
 * of a stream-ordered allocation; every other route allocates nothing in
 * either call and runs exactly as in w3a16_gemm.  The format paper has no
 * counterpart to this call; it is for callers that may not allocate.
 *   - W3_ERR_UNSUPPORTED if the decode would need more scratch than the array
 *     holds (a GPU with more than 160 SMs).
 *   - The scratch is shared by all calls on a device: calls that overlap in
 *     time (on different streams, or from different host threads) race on it
 *     and may return wrong results.  Calls on one stream are ordered and safe.
 *   - The scratch needs no initialisation: each call writes every slot it reads.
 */
w3_status w3a16_gemm_noalloc(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y,
                             int64_t M, int64_t N, int64_t K, w3_stream_t stream);

/*
 * The kernel-native block order (optional).  The decode kernels read a weight
 * 32 rows at a time, each of 32 lanes taking one 32-code block (3 words) of
 * four rows.  These calls store the same words permuted so that the words one
 * decode warp needs for a run of groups are one contiguous range (a single
 * 1-D bulk copy) and each lane's 12 words of a group are adjacent (three
 * 16-byte loads).  The GLQ page's decoder-native "kernel" layout
 * (trellis_layout "kernel") is the precedent: an offline re-order of a
 * checkpoint for its kernel; the exact-width storage above stays the
 * interchange format and the bit order inside each 3-word block is unchanged.
 * Definition: rows are grouped in blocks of 32 (the last padded with zero
 * rows); for block b, group g (128 codes), lane l = 4r + c (r = l/4 in 0..7,
 * c = l%4 in 0..3) and word 3h + i (h in 0..3, i in 0..2)
 *     native[((b*G + g)*32 + l)*12 + 3h + i] = packed[32b + r + 8h][12g + 3c + i],
 * G = K/128.  Scales keep their [N, K/128] layout.
 */

/* Words of the native order for an N x K weight: ceil(N/32)*32 * 3K/32; -1 for an invalid shape. */
int64_t w3_native_words(int64_t N, int64_t K);

/*
 * w3_pack_native -- codes [N,K] uint8 (0..7) -> native int32 [w3_native_words(N,K)]
 * (the same words w3_pack writes, in the native order; padded rows zero).
 * Errors as w3_pack.
 */
w3_status w3_pack_native(const uint8_t *codes, int32_t *native, int64_t N, int64_t K, w3_stream_t stream);

/* w3_native_from_packed -- packed [N, 3K/32] -> native order (a permutation of words). Errors as w3_pack. */
w3_status w3_native_from_packed(const int32_t *packed, int32_t *native, int64_t N, int64_t K, w3_stream_t stream);

/* w3_packed_from_native -- the inverse: native order -> packed [N, 3K/32]. Errors as w3_pack. */
w3_status w3_packed_from_native(const int32_t *native, int32_t *packed, int64_t N, int64_t K, w3_stream_t stream);

/*
 * w3a16_gemm_native -- y = x * W^T like w3a16_gemm, with W given in the native
 * order (scales [N, K/128] as usual), for decode batches: 1 <= M <= 16 and
 * N >= 32 (W3_ERR_UNSUPPORTED otherwise; larger batches use w3a16_gemm on the
 * row-major words).  Same arithmetic and determinism as w3a16_gemm's decode
 * (the weight enters exactly; fp32 accumulation; one rounding to bf16).
 * Allocates nothing.  Errors: W3_ERR_NULL, W3_ERR_SHAPE, W3_ERR_ALIGN,
 * W3_ERR_ALIAS, W3_ERR_UNSUPPORTED, W3_ERR_CUDA.
 */
w3_status w3a16_gemm_native(const uint16_t *x, const int32_t *native, const uint16_t *scales, uint16_t *y,
                            int64_t M, int64_t N, int64_t K, w3_stream_t stream);

/*
 * w3a16_gemm_route -- which kernels w3a16_gemm (and w3a16_gemm_noalloc) run for
 * an M x N x K product on a GPU with `num_sms` SMs, as a short name:
 *   "decode_sk"   persistent stream-K mma.sync decode (M <= 4, N >= 32 * num_sms,
 *                 x of the whole K range fits in shared memory);
 *   "decode_split" mma.sync decode, K split over a thread-block cluster with a
 *                 fixed-order reduction in distributed shared memory (the other
 *                 M <= 16 shapes with N >= 32 where its plan fits);
 *   "decode"      mma.sync decode with cluster split-K (the remaining M <= 16 shapes);
 *   "decode_tc32" tensor-core (tcgen05) decode, 32 columns (17 <= M <= 32, N >= 256);
 *   "prefill"     tcgen05 GEMM, weights dequantized into shared memory;
 *   "prefill_ab"  tcgen05 GEMM, weights dequantized into tensor memory;
 *   "passes"      M > 16 with K < 256: the decode routes on 16-row slices of x.
 * The choice depends only on the shape and the SM count (no device is touched,
 * so it can be asked on a machine without a GPU).  Returns NULL for a shape
 * that w3a16_gemm rejects with W3_ERR_SHAPE, or num_sms < 1.  The string is
 * static; do not free it.  No counterpart in the format's pages: it names this
 * library's kernels.
 */
const char *w3a16_gemm_route(int64_t M, int64_t N, int64_t K, int32_t num_sms);

/*
 * w3a16_gemm_launches -- how many kernels one w3a16_gemm (or w3a16_gemm_noalloc)
 * call launches for an M x N x K product on a GPU with `num_sms` SMs: 2 where
 * the tensor-core decode ("decode_tc32") splits row tiles between CTAs and a
 * fix-up kernel finishes them, one per 16-row pass for "passes", 1 for every
 * other route.  Host only, like w3a16_gemm_route; -1 where that returns NULL.
 */
int32_t w3a16_gemm_launches(int64_t M, int64_t N, int64_t K, int32_t num_sms);

/*
 * w3_check_device_error -- synchronise `stream`, then report and clear the
 * current device's error flag: W3_OK, or W3_ERR_TIMEOUT if a kernel of this
 * library gave up a bounded wait since the last check.  W3_ERR_CUDA if the
 * synchronisation itself fails.
 */
w3_status w3_check_device_error(w3_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* W3A16_H */
