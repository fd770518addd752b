// format_kernels.cuh -- pack, unpack and fp32 dequantization of the exact-width
// uint3 format (GSQ model card, section "Storage layout (why the HF UI shows
// I32 + BF16)": [N,K] codes -> [N, 3K/32] int32, bf16 scales [N, K/128]).
//
// One thread handles one 32-code block = 3 consecutive words.  Rows hold K/32
// whole blocks, so block b of the flattened matrix is words 3b..3b+2 and codes
// 32b..32b+31 regardless of the row it falls in.  Bit order: code j of a block
// is bits 3j..3j+2 of the block read as a little-endian 96-bit integer.
#pragma once

#include "common.cuh"

namespace w3 {

__device__ __forceinline__ unsigned __int128 load_block96(const uint32_t *__restrict__ p) {
    return static_cast<unsigned __int128>(p[0]) | (static_cast<unsigned __int128>(p[1]) << 32) |
           (static_cast<unsigned __int128>(p[2]) << 64);
}

__global__ void __launch_bounds__(256) pack_kernel(const uint8_t *__restrict__ codes, uint32_t *__restrict__ packed,
                                                   int64_t nblocks) {
    const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(codes + 32 * b);
    uint4 q[2] = {src[0], src[1]};
    const uint8_t *c = reinterpret_cast<const uint8_t *>(q);
    unsigned __int128 v = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) v |= static_cast<unsigned __int128>(c[j] & 7u) << (3 * j);
    uint32_t *dst = packed + 3 * b;
    dst[0] = static_cast<uint32_t>(v);
    dst[1] = static_cast<uint32_t>(v >> 32);
    dst[2] = static_cast<uint32_t>(v >> 64);
}

__global__ void __launch_bounds__(256) unpack_kernel(const uint32_t *__restrict__ packed,
                                                     uint8_t *__restrict__ codes, int64_t nblocks) {
    const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    const unsigned __int128 v = load_block96(packed + 3 * b);
    uint4 q[2];
    uint8_t *c = reinterpret_cast<uint8_t *>(q);
#pragma unroll
    for (int j = 0; j < 32; ++j) c[j] = static_cast<uint8_t>((v >> (3 * j)) & 7u);
    uint4 *dst = reinterpret_cast<uint4 *>(codes + 32 * b);
    dst[0] = q[0];
    dst[1] = q[1];
}

// w[n,k] = (c - 4) * s[n, k/128], exact in fp32.
__global__ void __launch_bounds__(256) dequant_f32_kernel(const uint32_t *__restrict__ packed,
                                                          const uint16_t *__restrict__ scales,
                                                          float *__restrict__ w, int64_t nblocks,
                                                          int64_t blocks_per_row, int64_t groups_per_row) {
    const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    const int64_t n = b / blocks_per_row;
    const int64_t t = b - n * blocks_per_row;  // block index within the row
    const float s = bf16_bits_to_f32(scales[n * groups_per_row + t / 4]);
    const unsigned __int128 v = load_block96(packed + 3 * b);
    float4 *dst = reinterpret_cast<float4 *>(w + 32 * b);
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        float4 o;
        o.x = static_cast<float>(static_cast<int>((v >> (3 * j)) & 7u) - 4) * s;
        o.y = static_cast<float>(static_cast<int>((v >> (3 * j + 3)) & 7u) - 4) * s;
        o.z = static_cast<float>(static_cast<int>((v >> (3 * j + 6)) & 7u) - 4) * s;
        o.w = static_cast<float>(static_cast<int>((v >> (3 * j + 9)) & 7u) - 4) * s;
        dst[j / 4] = o;
    }
}

inline unsigned grid_for(int64_t nblocks, int threads) {
    return static_cast<unsigned>((nblocks + threads - 1) / threads);
}

}  // namespace w3

namespace w3 {

// Re-pack from the 4-bit container GSQ training writes before the exact-width
// storage (the card's note under "Storage layout": compressed-tensors
// pack-quantized, the 3-bit codebook padded into a 4-bit INT32 container,
// re-packed by convert_to_humming.py).  The container layout is a reading (the
// card prints none): eight 4-bit fields per word, LSB first, each the level
// plus 8.  A 32-level block is 4 container words (16 bytes) in, 3 words out.
// Levels outside -4..3 have no 3-bit code: they are clamped to -4 or 3 and
// counted into *out_of_range (when given).
__global__ void __launch_bounds__(256) repack_ct4_kernel(const uint4 *__restrict__ ct4, uint32_t *__restrict__ packed,
                                                         int64_t nblocks, unsigned long long *out_of_range) {
    const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    unsigned clamped = 0;
    if (b < nblocks) {
        const uint4 q = ct4[b];
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
        unsigned __int128 v = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            int level = static_cast<int>((w[j >> 3] >> (4 * (j & 7))) & 15u) - 8;
            if (level < -4 || level > 3) {
                ++clamped;
                level = level < -4 ? -4 : 3;
            }
            v |= static_cast<unsigned __int128>(level + 4) << (3 * j);
        }
        uint32_t *dst = packed + 3 * b;
        dst[0] = static_cast<uint32_t>(v);
        dst[1] = static_cast<uint32_t>(v >> 32);
        dst[2] = static_cast<uint32_t>(v >> 64);
    }
    if (out_of_range) {
        clamped = __reduce_add_sync(0xffffffffu, clamped);
        if ((threadIdx.x & 31) == 0 && clamped) atomicAdd(out_of_range, static_cast<unsigned long long>(clamped));
    }
}

}  // namespace w3

namespace w3 {

// The kernel-native block order of the packed words (the decode kernels read 32 rows
// at a time, each lane one 32-code block of four rows): rows in blocks of 32 (the
// last padded with zero rows); for block b, group g, lane l = 4r + c, word 3h + i:
//     native[((b*G + g)*32 + l)*12 + 3h + i] = packed[row 32b + r + 8h][word 12g + 3c + i].
// One thread moves one 3-word block (t -> h = t % 4, l = t/4 % 32, g, b), so the
// writes of a warp are contiguous.
__device__ __forceinline__ void native_coords(int64_t t, int64_t G, int64_t &row, int64_t &word) {
    const int h = static_cast<int>(t & 3), l = static_cast<int>((t >> 2) & 31);
    const int64_t bg = t >> 7, g = bg % G, b = bg / G;
    row = 32 * b + (l >> 2) + 8 * h;
    word = 12 * g + 3 * (l & 3);
}

__global__ void __launch_bounds__(256) native_from_packed_kernel(const uint32_t *__restrict__ packed,
                                                                 uint32_t *__restrict__ native, int64_t N,
                                                                 int64_t K, int64_t nthreads) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= nthreads) return;
    const int64_t W = K * 3 / 32, G = K / kGroup;
    int64_t row, word;
    native_coords(t, G, row, word);
    uint32_t v[3] = {0u, 0u, 0u};
    if (row < N) {
        const uint32_t *src = packed + row * W + word;
        v[0] = src[0];
        v[1] = src[1];
        v[2] = src[2];
    }
    uint32_t *dst = native + 3 * t;
    dst[0] = v[0];
    dst[1] = v[1];
    dst[2] = v[2];
}

__global__ void __launch_bounds__(256) packed_from_native_kernel(const uint32_t *__restrict__ native,
                                                                 uint32_t *__restrict__ packed, int64_t N,
                                                                 int64_t K, int64_t nthreads) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= nthreads) return;
    const int64_t W = K * 3 / 32, G = K / kGroup;
    int64_t row, word;
    native_coords(t, G, row, word);
    if (row >= N) return;
    const uint32_t *src = native + 3 * t;
    uint32_t *dst = packed + row * W + word;
    dst[0] = src[0];
    dst[1] = src[1];
    dst[2] = src[2];
}

// codes [N,K] -> native directly: the 3 words of (row, 32-code block) packed as in
// pack_kernel and written at their native position.
__global__ void __launch_bounds__(256) pack_native_kernel(const uint8_t *__restrict__ codes,
                                                          uint32_t *__restrict__ native, int64_t N, int64_t K,
                                                          int64_t nthreads) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= nthreads) return;
    const int64_t G = K / kGroup;
    int64_t row, word;
    native_coords(t, G, row, word);
    unsigned __int128 v = 0;
    if (row < N) {
        // word 12g + 3c is 32-code block 4g + c of the row: codes 32 * (word / 3) ...
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + row * K + 32 * (word / 3));
        uint4 q[2] = {src[0], src[1]};
        const uint8_t *c = reinterpret_cast<const uint8_t *>(q);
#pragma unroll
        for (int j = 0; j < 32; ++j) v |= static_cast<unsigned __int128>(c[j] & 7u) << (3 * j);
    }
    uint32_t *dst = native + 3 * t;
    dst[0] = static_cast<uint32_t>(v);
    dst[1] = static_cast<uint32_t>(v >> 32);
    dst[2] = static_cast<uint32_t>(v >> 64);
}

}  // namespace w3
