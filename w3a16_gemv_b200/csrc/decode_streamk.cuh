// decode_streamk.cuh -- persistent, load-balanced decode for small batches
// (M padded to 1, 2 or 4), the same arithmetic as decode_gemv.cuh.
//
// Why a second schedule: a decode problem has few row blocks per SM (the
// gate_proj shape has 896 blocks of 32 rows for 148 SMs), and a kernel that
// hands out whole blocks leaves SMs unevenly loaded.  Here one CTA runs per
// SM and the CTA's blocks x groups are split into exactly equal contiguous
// ranges, one per warp, in (block, group) order ("stream-K" inside the CTA).
// A warp's range covers at most a partial first block, whole blocks, and a
// partial last block.  Whole blocks are stored directly; partial blocks are
// summed at the end through shared memory in fixed warp order (ascending
// groups), so the result is deterministic and needs no global scratch.  The
// prepared x (see decode_gemv.cuh) covers the whole K range and is built once
// per CTA.
//
// A block is 32 rows = two 16-row MMA tiles that share the B fragments.  Each
// warp streams its range through a private ring: a full stage is 3 groups of
// the 32 rows, fetched with one tiled TMA copy ([32 rows][36 words] box, dense,
// conflict-free pitch); a stage with 1 or 2 groups left in its segment uses
// 1-group boxes ([32][12 words]) so that no byte outside the range is read.
// With the kernel-native block order (NATIVE; see format_kernels.cuh) a stage
// of a block's consecutive groups is one contiguous range of memory, fetched
// with a single 1-D bulk copy, and each lane reads its 12 words of a group with
// three 16-byte shared-memory loads (lane-ordered, free of bank conflicts).
#pragma once

#include "decode_gemv.cuh"

namespace w3 {
namespace decode_sk {

using decode::unpack_block;

constexpr int kWarps = 12;
constexpr int kMaxDepth = 4;  // ring stages per warp; the launch picks 2..kMaxDepth
constexpr int kTileRows = 16;
constexpr int kBlockRows = 32;                           // rows per warp block (2 tiles)
constexpr int kStageGroups = 3;
constexpr int kPitch3 = kStageGroups * kWordsPerGroup;   // 36 words: rows of a 3-group box
constexpr int kPitch1 = kWordsPerGroup;                  // 12 words: rows of a 1-group box
constexpr int kStageBytes = kBlockRows * kPitch3 * 4;    // 4608
constexpr int kBox1Bytes = kBlockRows * kPitch1 * 4;     // 1536: one group of a block (also in the native order)
constexpr int kNativeGroupWords = kBlockRows * kPitch1;  // 384
constexpr int kXsBudgetBytes = 96 * 1024;
constexpr int kSmemLimit = 227 * 1024;
static_assert(kStageBytes % 128 == 0 && kBox1Bytes % 128 == 0,
              "a tiled TMA destination in shared memory must be 128-byte aligned");

struct SmemLayout {
    int xs_off, corr_off, cpart_off, ncorr_off, bar_off, ring_off, slot_off, total;
};

__host__ __device__ inline SmemLayout smem_layout(int G, int mt, int depth) {
    SmemLayout L;
    L.xs_off = 0;                                                          // uint2 [G][8][mt][4]
    L.corr_off = decode::align_up(L.xs_off + G * 8 * mt * 4 * 8, 16);      // float [G][8]
    L.cpart_off = decode::align_up(L.corr_off + G * 8 * 4, 16);            // float [G][mt][4]
    L.ncorr_off = decode::align_up(L.cpart_off + G * mt * 4 * 4, 16);      // float4 [G][4]
    L.bar_off = decode::align_up(L.ncorr_off + G * 4 * 16, 16);            // u64 [kWarps][depth]
    L.ring_off = decode::align_up(L.bar_off + kWarps * depth * 8, 128);    // [kWarps][depth][kStageBytes]
    L.slot_off = L.ring_off + kWarps * depth * kStageBytes;                // float4 [kWarps][2][2 tiles][32]
    L.total = L.slot_off + kWarps * 2 * 2 * 32 * 16;
    return L;
}

struct Params {
    CUtensorMap tmap3;  // packed [N][3K/32] u32, box [32 rows][36 words]
    CUtensorMap tmap1;  // same tensor, box [32 rows][12 words]
    const uint32_t *native;  // the same words in the native block order (NATIVE kernels)
    const uint16_t *x;
    const uint16_t *scales;
    uint16_t *y;
    int M, N, K;
    int ctas;   // grid size; CTA i owns blocks [NB*i/ctas, NB*(i+1)/ctas)
    int depth;  // ring stages per warp
};

// The unit range [u0, u1) of warp w among `nw` warps sharing `units` units.
__host__ __device__ __forceinline__ void warp_range(int64_t units, int w, int nw, int64_t &u0, int64_t &u1) {
    u0 = units * w / nw;
    u1 = units * (w + 1) / nw;
}

// One k-step of one tile: the four A registers of MMA k (pairs 2k and 2k+1 of
// the lane's two rows), unpacked right before the MMA.
template <int K>
__device__ __forceinline__ void tile_kstep(const uint32_t (&wa)[3], const uint32_t (&wb)[3], uint2 b,
                                           float (&d)[4], uint32_t magic) {
    const uint32_t a0 = decode::unpack_pair<2 * K>(wa[0], wa[1], wa[2], magic);
    const uint32_t a1 = decode::unpack_pair<2 * K>(wb[0], wb[1], wb[2], magic);
    const uint32_t a2 = decode::unpack_pair<2 * K + 1>(wa[0], wa[1], wa[2], magic);
    const uint32_t a3 = decode::unpack_pair<2 * K + 1>(wb[0], wb[1], wb[2], magic);
    mma_bf16_m16n8k16(d, a0, a1, a2, a3, b.x, b.y, d);
}

template <int K>
__device__ __forceinline__ void block_ksteps(const uint32_t (&w)[4][3], const uint2 (&xs_g)[8],
                                             float (&d0)[4], float (&d1)[4], uint32_t magic) {
    if constexpr (K < 8) {
        const uint2 b = xs_g[K];
        tile_kstep<K>(w[0], w[1], b, d0, magic);
        tile_kstep<K>(w[2], w[3], b, d1, magic);
        block_ksteps<K + 1>(w, xs_g, d0, d1, magic);
    }
}

// The 12 words of lane (r, c) for group j of a stage (block c of the group in rows
// r, r+8, r+16, r+24): row i, word w of group j at st[i*pitch + j*jstride + w] in
// a row-major box, or lane-ordered in the native order.
template <bool NATIVE>
__device__ __forceinline__ void lane_words(const uint32_t *st, int pitch, int jstride, int j, int r, int c,
                                           uint32_t (&w)[4][3]) {
    if constexpr (NATIVE) {
        const uint4 *q = reinterpret_cast<const uint4 *>(st + j * kNativeGroupWords + (4 * r + c) * 12);
        const uint4 a = q[0], b = q[1], d = q[2];
        w[0][0] = a.x; w[0][1] = a.y; w[0][2] = a.z;
        w[1][0] = a.w; w[1][1] = b.x; w[1][2] = b.y;
        w[2][0] = b.z; w[2][1] = b.w; w[2][2] = d.x;
        w[3][0] = d.y; w[3][1] = d.z; w[3][2] = d.w;
    } else {
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int i = 0; i < 3; ++i) w[h][i] = st[(8 * h + r) * pitch + j * jstride + 3 * c + i];
    }
}

// One group of one 32-row block: both tiles' 8 MMAs as two interleaved chains,
// each started from the group's -corr and scaled in fp32 into acc.
template <int MT, bool NATIVE>
__device__ __forceinline__ void block_group(const uint32_t *st, int pitch, int jstride, int j, int gabs,
                                            const uint2 *xs_lane, const float4 *ncorr,
                                            const uint16_t *const (&sc)[4], int r, int c,
                                            float (&acc)[2][4], uint32_t magic) {
    uint32_t w[4][3];  // block c of the group in rows r, r+8, r+16, r+24
    lane_words<NATIVE>(st, pitch, jstride, j, r, c, w);
    const float4 nc = ncorr[gabs * 4];
    float d0[4] = {nc.x, nc.y, nc.z, nc.w};
    float d1[4] = {nc.x, nc.y, nc.z, nc.w};
    // this lane's B fragments of the group's 8 k-steps
    uint2 bfr[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) bfr[k] = xs_lane[(gabs * 8 + k) * MT * 4];
    block_ksteps<0>(w, bfr, d0, d1, magic);
    float s[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) s[h] = bf16_bits_to_f32(__ldg(sc[h] + gabs));
    acc[0][0] = fmaf(s[0], d0[0], acc[0][0]);
    acc[0][1] = fmaf(s[0], d0[1], acc[0][1]);
    acc[0][2] = fmaf(s[1], d0[2], acc[0][2]);
    acc[0][3] = fmaf(s[1], d0[3], acc[0][3]);
    acc[1][0] = fmaf(s[2], d1[0], acc[1][0]);
    acc[1][1] = fmaf(s[2], d1[1], acc[1][1]);
    acc[1][2] = fmaf(s[3], d1[2], acc[1][2]);
    acc[1][3] = fmaf(s[3], d1[3], acc[1][3]);
}

// A full stage (3 groups) of one 32-row block: 3 groups x 2 tiles = 6
// independent MMA chains interleaved k-step by k-step, so that the tensor-core
// latency of one chain is covered by the others.
template <int K, int MT>
__device__ __forceinline__ void stage_ksteps(const uint32_t (&w)[3][4][3], const uint2 *xs_g,
                                             float (&d)[3][2][4], uint32_t magic) {
    if constexpr (K < 8) {
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const uint2 b = xs_g[(j * 8 + K) * MT * 4];
            tile_kstep<K>(w[j][0], w[j][1], b, d[j][0], magic);
            tile_kstep<K>(w[j][2], w[j][3], b, d[j][1], magic);
        }
        stage_ksteps<K + 1, MT>(w, xs_g, d, magic);
    }
}

template <int MT, bool NATIVE>
__device__ __forceinline__ void full_stage(const uint32_t *st, int g, const uint2 *xs_lane, const float4 *ncorr,
                                           const uint16_t *const (&sc)[4], int r, int c,
                                           float (&acc)[2][4], uint32_t magic) {
    float s[3][4];
#pragma unroll
    for (int j = 0; j < 3; ++j)
#pragma unroll
        for (int h = 0; h < 4; ++h) s[j][h] = bf16_bits_to_f32(__ldg(sc[h] + g + j));
    uint32_t w[3][4][3];
#pragma unroll
    for (int j = 0; j < 3; ++j) lane_words<NATIVE>(st, kPitch3, kWordsPerGroup, j, r, c, w[j]);
    float d[3][2][4];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const float4 nc = ncorr[(g + j) * 4];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            d[j][t][0] = nc.x;
            d[j][t][1] = nc.y;
            d[j][t][2] = nc.z;
            d[j][t][3] = nc.w;
        }
    }
    stage_ksteps<0, MT>(w, xs_lane + g * 8 * MT * 4, d, magic);
#pragma unroll
    for (int j = 0; j < 3; ++j)
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            acc[t][0] = fmaf(s[j][2 * t], d[j][t][0], acc[t][0]);
            acc[t][1] = fmaf(s[j][2 * t], d[j][t][1], acc[t][1]);
            acc[t][2] = fmaf(s[j][2 * t + 1], d[j][t][2], acc[t][2]);
            acc[t][3] = fmaf(s[j][2 * t + 1], d[j][t][3], acc[t][3]);
        }
}

__device__ __forceinline__ void store_block(uint16_t *y, int N, int M, int block, int r, int c,
                                            const float (&v)[2][4]) {
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = block * kBlockRows + 16 * t + r + ((i < 2) ? 0 : 8);
            const int m = 2 * c + (i & 1);
            if (row < N && m < M) y[static_cast<int64_t>(m) * N + row] = f32_to_bf16_rn(v[t][i]);
        }
}

template <int MT, bool NATIVE>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_sk_kernel(const __grid_constant__ Params p) {
    static_assert(MT == 1 || MT == 2 || MT == 4, "stream-K decode handles batches up to 4");
    extern __shared__ __align__(128) uint8_t smem[];
    const int M = p.M, N = p.N;
    const int G = p.K / kGroup;
    const int depth = p.depth;
    const SmemLayout L = smem_layout(G, MT, depth);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int r = lane >> 2;
    const int c = lane & 3;
    pdl_trigger();  // the next kernel in the stream may start its own set-up

    const int NB = (N + kBlockRows - 1) / kBlockRows;
    const int b_begin = static_cast<int>(static_cast<int64_t>(NB) * blockIdx.x / p.ctas);
    const int b_end = static_cast<int>(static_cast<int64_t>(NB) * (blockIdx.x + 1) / p.ctas);
    const int64_t units = static_cast<int64_t>(b_end - b_begin) * G;
    int64_t u0, u1;
    warp_range(units, warp, kWarps, u0, u1);

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off) + warp * depth;
    uint8_t *ring = smem + L.ring_off + warp * depth * kStageBytes;
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t ring0 = smem_addr(ring);
    if (lane == 0) {
        for (int s = 0; s < depth; ++s) mbar_init(bar0 + 8 * s, 1);
        mbar_init_fence();
    }
    __syncwarp();

    // The warp's work is a flat sequence of stages over [u0, u1): a stage never
    // crosses a block boundary, so segments (the pieces of the range inside one
    // block) are runs of stages.  Two cursors (block index within the CTA,
    // group) walk the range: one for issuing copies, one for computing.
    const int64_t blk0 = u0 / G;
    const int g_first0 = static_cast<int>(u0 - blk0 * G);
    const int64_t last = u1 - 1;
    const int64_t blk_last = (u1 > u0) ? last / G : blk0;
    const int g_end_last = (u1 > u0) ? static_cast<int>(last - blk_last * G) + 1 : 0;  // end group in last block
    // groups of the stage at cursor (bl, g)
    auto stage_groups = [&](int64_t bl, int g) {
        const int end = (bl == blk_last) ? g_end_last : G;
        const int left = end - g;
        return left < kStageGroups ? left : kStageGroups;
    };
    auto advance = [&](int64_t &bl, int &g, int ng) {
        g += ng;
        const int end = (bl == blk_last) ? g_end_last : G;
        if (g == end) {
            ++bl;
            g = 0;
        }
    };

    // issue the stage at cursor (bl, g) into ring slot `slot`; returns its groups
    auto issue = [&](int64_t bl, int g, int slot) -> int {
        const int ng = stage_groups(bl, g);
        const int row0 = (b_begin + static_cast<int>(bl)) * kBlockRows;
        __syncwarp();  // every lane is done reading the slot being refilled
        if (lane == 0) {
            const uint32_t bar = bar0 + 8 * slot;
            const uint32_t dst = ring0 + slot * kStageBytes;
            if constexpr (NATIVE) {
                // ng consecutive groups of one block: one contiguous range
                mbar_arrive_expect_tx(bar, ng * kBox1Bytes);
                bulk_copy_g2s(dst, p.native + (static_cast<int64_t>(row0 / kBlockRows) * G + g) * kNativeGroupWords,
                              ng * kBox1Bytes, bar);
            } else if (ng == kStageGroups) {
                mbar_arrive_expect_tx(bar, kStageBytes);
                tma_load_2d(dst, &p.tmap3, g * kWordsPerGroup, row0, bar);
            } else {
                mbar_arrive_expect_tx(bar, ng * kBox1Bytes);
                for (int j = 0; j < ng; ++j)
                    tma_load_2d(dst + j * kBox1Bytes, &p.tmap1, (g + j) * kWordsPerGroup, row0, bar);
            }
        }
        return ng;
    };

    const int nstages_total = [&] {
        int n = 0;
        int64_t bl = blk0;
        int g = g_first0;
        if (u1 <= u0) return 0;
        while (bl <= blk_last) {
            const int end = (bl == blk_last) ? g_end_last : G;
            n += (end - g + kStageGroups - 1) / kStageGroups;
            ++bl;
            g = 0;
        }
        return n;
    }();

    // stream weights before preparing x
    int64_t ibl = blk0;
    int ig = g_first0;
    int issued = 0;
    int issue_slot = 0;  // == issued % depth
    for (; issued < depth - 1 && issued < nstages_total; ++issued) {
        advance(ibl, ig, issue(ibl, ig, issue_slot));
        issue_slot = (issue_slot + 1 == depth) ? 0 : issue_slot + 1;
    }
    // x (and, at the end, y) may belong to the previous kernel in the stream: wait for it here,
    // after the first weight stages are already in flight
    pdl_wait();
    decode::Params dp;  // prepare_x reads x, M and K only
    dp.x = p.x;
    dp.M = M;
    dp.K = p.K;
    decode::SmemLayout dl;
    dl.xs_off = L.xs_off;
    dl.corr_off = L.corr_off;
    dl.cpart_off = L.cpart_off;
    decode::prepare_x<MT>(dp, smem, dl, 0, G);
    // the MMA chains start from -corr: (-corr[2c], -corr[2c+1]) for rows r and r+8
    {
        const float *cf = reinterpret_cast<const float *>(smem + L.corr_off);
        float4 *nq = reinterpret_cast<float4 *>(smem + L.ncorr_off);
        for (int it = threadIdx.x; it < G * 4; it += blockDim.x) {
            const int g = it >> 2, cc = it & 3;
            const float a = -cf[g * 8 + 2 * cc], b = -cf[g * 8 + 2 * cc + 1];
            nq[it] = make_float4(a, b, a, b);
        }
        __syncthreads();
    }

    // B fragments: lanes whose batch row r is >= MT read words of other rows;
    // the MMA keeps columns apart and those columns are never stored.
    const uint2 *xs_lane = reinterpret_cast<const uint2 *>(smem + L.xs_off) + (r * 4 + c);
    const float4 *ncorr = reinterpret_cast<const float4 *>(smem + L.ncorr_off) + c;
    float4 *slots = reinterpret_cast<float4 *>(smem + L.slot_off) + warp * 2 * 2 * 32;

    bool ok = true;
    const uint32_t magic = decode::pinned_magic();
    uint32_t phase_bits = 0;
    float acc[2][4] = {};
    const uint16_t *sc[4] = {p.scales, p.scales, p.scales, p.scales};
    int64_t cbl = blk0;  // compute cursor
    int cg = g_first0;
    int64_t sc_block = -1;
    int slot = 0;  // == s % depth
    for (int s = 0; s < nstages_total; ++s, slot = (slot + 1 == depth) ? 0 : slot + 1) {
        const int ng = stage_groups(cbl, cg);
        const int block = b_begin + static_cast<int>(cbl);
        if (cbl != sc_block) {  // scale rows of this lane in the new block (clamped to N-1)
            sc_block = cbl;
#pragma unroll
            for (int h = 0; h < 4; ++h)
                sc[h] = p.scales + static_cast<int64_t>(min(block * kBlockRows + 8 * h + r, N - 1)) * G;
        }
        if (ok && issued < nstages_total) {
            advance(ibl, ig, issue(ibl, ig, issue_slot));
            issue_slot = (issue_slot + 1 == depth) ? 0 : issue_slot + 1;
            ++issued;
        }
        if (s >= issued) break;  // only after a timeout: nothing left in flight
        const uint32_t parity = (phase_bits >> slot) & 1u;
        phase_bits ^= 1u << slot;
        // warp-uniform: a timeout seen by any lane stops the whole warp
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar0 + 8 * slot, parity) && ok);
        if (ok) {
            const uint32_t *st = reinterpret_cast<const uint32_t *>(ring + slot * kStageBytes);
            if (ng == kStageGroups) {
                full_stage<MT, NATIVE>(st, cg, xs_lane, ncorr, sc, r, c, acc, magic);
            } else {
                for (int j = 0; j < ng; ++j)
                    block_group<MT, NATIVE>(st, kPitch1, kBlockRows * kPitch1, j, cg + j, xs_lane, ncorr, sc, r, c,
                                            acc, magic);
            }
        }
        // end of a segment: store a whole block, or park a partial one in a slot
        const int g_stage = cg;
        const int64_t bl_stage = cbl;
        advance(cbl, cg, ng);
        if (cbl != bl_stage) {
            const int g_first = (bl_stage == blk0) ? g_first0 : 0;
            const bool whole = (g_first == 0) && (g_stage + ng == G);
            if (whole) {
                if (ok) store_block(p.y, N, M, block, r, c, acc);
            } else {
                // a partial block is the first or the last segment of the range
                float4 *dst = slots + ((bl_stage == blk0) ? 0 : 2) * 32;
                dst[lane] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
                dst[32 + lane] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
            }
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;
        }
    }

    __syncthreads();
    // Owners: the warp holding group 0 of a partial block adds the later warps'
    // first-segment partials, in ascending warp (= ascending group) order.
    if (ok && u1 > u0) {
        // the last block starting inside [u0, u1): if it does not end inside the
        // range it is partial, continues in later warps, and this warp owns it
        const int64_t own_u = ((u1 - 1) / G) * G;
        if (own_u >= u0 && own_u + G > u1) {
            const int block = b_begin + static_cast<int>(own_u / G);
            const float4 *mine = slots + ((own_u == u0) ? 0 : 2) * 32;
            float4 v0 = mine[lane], v1 = mine[32 + lane];
            const float4 *all = reinterpret_cast<const float4 *>(smem + L.slot_off);
            for (int w2 = warp + 1; w2 < kWarps; ++w2) {
                int64_t a0, a1;
                warp_range(units, w2, kWarps, a0, a1);
                if (a0 >= own_u + G) break;
                if (a1 <= a0) continue;
                const float4 q0 = all[(w2 * 4 + 0) * 32 + lane], q1 = all[(w2 * 4 + 1) * 32 + lane];
                v0.x += q0.x;
                v0.y += q0.y;
                v0.z += q0.z;
                v0.w += q0.w;
                v1.x += q1.x;
                v1.y += q1.y;
                v1.z += q1.z;
                v1.w += q1.w;
            }
            const float vv[2][4] = {{v0.x, v0.y, v0.z, v0.w}, {v1.x, v1.y, v1.z, v1.w}};
            store_block(p.y, N, M, block, r, c, vv);
        }
    }
}

struct LaunchPlan {
    int mt, ctas, depth, smem_bytes;
};

// The deepest ring (2..kMaxDepth) whose layout fits in shared memory, or 0.
inline int fitting_depth(int G, int mt) {
    for (int d = kMaxDepth; d >= 2; --d)
        if (smem_layout(G, mt, d).total <= kSmemLimit) return d;
    return 0;
}

// Usable when the prepared x of the whole K range fits in shared memory (and
// the matrix has at least one full 32-row block, the height of a TMA box).
inline bool applicable(int M, int N, int K) {
    const int mt = decode::padded_batch(M);
    const int G = K / kGroup;
    return mt <= 4 && N >= kBlockRows && G * 8 * mt * 4 * 8 <= kXsBudgetBytes && fitting_depth(G, mt) > 0;
}

inline LaunchPlan plan(int M, int N, int K, int num_sms) {
    LaunchPlan P;
    P.mt = decode::padded_batch(M);
    const int G = K / kGroup;
    const int NB = (N + kBlockRows - 1) / kBlockRows;
    // at least ~4 groups per warp; at most one CTA per SM and per block
    const int64_t want = (static_cast<int64_t>(NB) * G + 4 * kWarps - 1) / (4 * kWarps);
    P.ctas = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms, std::min<int64_t>(want, NB))));
    P.depth = fitting_depth(G, P.mt);
    P.smem_bytes = smem_layout(G, P.mt, P.depth).total;
    return P;
}

}  // namespace decode_sk
}  // namespace w3
