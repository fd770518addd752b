// decode_split.cuh -- y = x * W^T for decode batches M <= 16, W in the
// exact-width uint3 / group-128 / bf16-scale format of the GSQ model card
// ("Storage layout" section), never materialised; the arithmetic of
// decode_gemv.cuh (register unpack into the bf16 mantissa, mma.sync with fp32
// accumulation, group scale applied in fp32).
//
// Work split.  The matrix is cut into 32-row blocks; a thread-block cluster of
// C CTAs (C = 1, 2, 4 or 8) owns a contiguous range of blocks, and its CTAs
// split K: CTA rank q takes the groups [G*q/C, G*(q+1)/C).  A CTA prepares x
// (pair order, 2^-e scaling, per-group corrections) for its K slice only, so
// the prepared x of a 16-row batch fits in shared memory whatever K is, and
// the block ranges of many clusters balance the work finer than whole blocks
// per SM would.  Inside a CTA the (block, group) units of the slice are cut
// into equal contiguous ranges, one per warp ("stream-K"): a warp's range is
// the end of one block, whole blocks and the start of another.  Blocks split
// between warps are added in warp order through shared memory.  With C > 1 the
// blocks of a cluster are shared out among its ranks; as a CTA finishes a
// block's sum over its slice it stores it into the shared memory of the rank
// that owns the block (distributed shared memory, during the main loop), and
// after one cluster barrier each rank adds the C slices of its blocks in rank
// order from its own shared memory.  Every sum has a fixed order: results are
// deterministic, and no global scratch or atomic is used.
//
// Loads: each warp streams its range through a private ring of tiled TMA
// copies, [32 rows x 36 words] (3 groups) or [32 rows x 12 words] boxes; with
// the kernel-native block order (NATIVE; see format_kernels.cuh) a stage is one
// 1-D bulk copy of a block's consecutive groups and a lane reads its 12 words
// of a group with three 16-byte shared-memory loads.  Batches of 9..16 rows use
// two n8 MMA tiles per k-step.
#pragma once

#include "decode_gemv.cuh"

namespace w3 {
namespace dsplit {

// Warps per CTA, and groups per full ring stage: 3 (a [32 rows][36 words] box), or 2
// for 16-row batches (two n8 tiles per k-step double the accumulators; the smaller stage
// keeps twelve warps within the registers and shared memory).
constexpr int kWarps = 12;
__host__ __device__ constexpr int stage_groups_for(int mt) { return mt > 8 ? 2 : 3; }
constexpr int kMaxDepth = 4;    // ring stages per warp; the launch picks 2..kMaxDepth
constexpr int kBlockRows = 32;  // rows per warp block (two 16-row MMA tiles)
constexpr int kMaxStageGroups = 3;
constexpr int kPitch1 = kWordsPerGroup;                       // 12 words: rows of a 1-group box
__host__ __device__ constexpr int stage_bytes(int mt) { return kBlockRows * stage_groups_for(mt) * kWordsPerGroup * 4; }
constexpr int kBox1Bytes = kBlockRows * kPitch1 * 4;          // 1536: one group of a block
constexpr int kNativeGroupWords = kBlockRows * kPitch1;       // 384
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMaxCluster = 8;
static_assert(kBlockRows * 2 * kWordsPerGroup * 4 % 128 == 0 && kBlockRows * 3 * kWordsPerGroup * 4 % 128 == 0 &&
                  kBox1Bytes % 128 == 0,
              "a tiled TMA destination in shared memory must be 128-byte aligned");

__host__ __device__ constexpr int n_tiles(int mt) { return mt > 8 ? 2 : 1; }

struct SmemLayout {
    int xs_off, corr_off, cpart_off, ncorr_off, bar_off, ring_off, slot_off, pb_off, total;
};

// Blocks a rank of a C-CTA cluster owns for the final sum, at most: rank q owns the cluster's
// blocks [nb*q/C, nb*(q+1)/C).
__host__ __device__ constexpr int share_blocks(int nb, int C) { return (nb + C - 1) / C; }

// gs: groups of the CTA's K slice (at most); nb: blocks of a cluster (at most).
__host__ __device__ inline SmemLayout smem_layout(int gs, int mt, int depth, int nb, int C) {
    const int nt = n_tiles(mt);
    SmemLayout L;
    L.xs_off = 0;                                                          // uint2 [gs][8][mt][4]
    L.corr_off = decode::align_up(L.xs_off + gs * 8 * mt * 4 * 8, 16);     // float [gs][8*nt]
    L.cpart_off = decode::align_up(L.corr_off + gs * 8 * nt * 4, 16);      // float [gs][mt][4]
    L.ncorr_off = decode::align_up(L.cpart_off + gs * mt * 4 * 4, 16);     // float4 [gs][nt][4]
    L.bar_off = decode::align_up(L.ncorr_off + gs * nt * 4 * 16, 16);      // u64 [warps][depth]
    L.ring_off = decode::align_up(L.bar_off + kWarps * depth * 8, 128);    // [warps][depth][stage bytes]
    L.slot_off = L.ring_off + kWarps * depth * stage_bytes(mt);            // float4 [warps][2 tiles][nt][32]
    L.pb_off = L.slot_off + kWarps * 2 * nt * 32 * 16;                     // float4 [C][share][2 tiles][nt][32] (C > 1)
    L.total = L.pb_off + (C > 1 ? C * share_blocks(nb, C) * 2 * nt * 32 * 16 : 0);
    return L;
}

struct Params {
    CUtensorMap tmapS;  // packed [N][3K/32] u32, box [32 rows][12 * stage groups words]
    CUtensorMap tmap1;  // same tensor, box [32 rows][12 words]
    const uint32_t *native;  // the same words in the native block order (NATIVE kernels)
    const uint16_t *x;
    const uint16_t *scales;
    uint16_t *y;
    int M, N, K, G;
    int C;      // CTAs per cluster (K split)
    int ncl;    // clusters; cluster i owns blocks [NB*i/ncl, NB*(i+1)/ncl)
    int depth;  // ring stages per warp
    int gs_max, nb_max;
    int hasS;   // the full-stage box fits in a row
};

// The unit range [u0, u1) of warp w among `nw` warps sharing `units` units.
__host__ __device__ __forceinline__ void warp_range(int64_t units, int w, int nw, int64_t &u0, int64_t &u1) {
    u0 = units * w / nw;
    u1 = units * (w + 1) / nw;
}

// One k-step of one 16-row tile for every n8 tile: the four A registers of the
// step (pairs 2K and 2K+1 of the lane's two rows), unpacked right before the MMAs.
template <int K, int NT>
__device__ __forceinline__ void tile_kstep(const uint32_t (&wa)[3], const uint32_t (&wb)[3], const uint2 (&b)[NT],
                                           float (&d)[NT][4], uint32_t magic) {
    const uint32_t a0 = decode::unpack_pair<2 * K>(wa[0], wa[1], wa[2], magic);
    const uint32_t a1 = decode::unpack_pair<2 * K>(wb[0], wb[1], wb[2], magic);
    const uint32_t a2 = decode::unpack_pair<2 * K + 1>(wa[0], wa[1], wa[2], magic);
    const uint32_t a3 = decode::unpack_pair<2 * K + 1>(wb[0], wb[1], wb[2], magic);
#pragma unroll
    for (int u = 0; u < NT; ++u) mma_bf16_m16n8k16(d[u], a0, a1, a2, a3, b[u].x, b[u].y, d[u]);
}

// k-steps K..7 of JN groups x 2 tiles: 2*JN*NT independent MMA chains interleaved k-step by k-step.
template <int K, int JN, int MT, int NT>
__device__ __forceinline__ void ksteps(const uint32_t (&w)[JN][4][3], const uint2 *xs_g, int jstride,
                                       float (&d)[JN][2][NT][4], uint32_t magic) {
    if constexpr (K < 8) {
#pragma unroll
        for (int j = 0; j < JN; ++j) {
            uint2 b[NT];
#pragma unroll
            for (int u = 0; u < NT; ++u) b[u] = xs_g[(j * jstride * 8 + K) * MT * 4 + u * 32];
            tile_kstep<K, NT>(w[j][0], w[j][1], b, d[j][0], magic);
            tile_kstep<K, NT>(w[j][2], w[j][3], b, d[j][1], magic);
        }
        ksteps<K + 1, JN, MT, NT>(w, xs_g, jstride, d, magic);
    }
}

// JN consecutive groups (1 or 3) of one 32-row block: group j of the stage is
// row i, word k at st[i*pitch + j*jstride_w + k]; xs_g points at the first
// group's prepared x; the group's scales multiply the fp32 results into acc.
template <int JN, int MT, int NT, bool NATIVE>
__device__ __forceinline__ void groups(const uint32_t *st, int pitch, int jstride_w, int grel, int gabs,
                                       const uint2 *xs_lane, const float4 *ncorr, const uint16_t *const (&sc)[4],
                                       int r, int c, float (&acc)[2][NT][4], uint32_t magic) {
    float s[JN][4];
#pragma unroll
    for (int j = 0; j < JN; ++j)
#pragma unroll
        for (int h = 0; h < 4; ++h) s[j][h] = bf16_bits_to_f32(__ldg(sc[h] + gabs + j));
    uint32_t w[JN][4][3];  // block c of group j in rows r, r+8, r+16, r+24
#pragma unroll
    for (int j = 0; j < JN; ++j) {
        if constexpr (NATIVE) {
            const uint4 *q = reinterpret_cast<const uint4 *>(st + j * kNativeGroupWords + (4 * r + c) * 12);
            const uint4 a = q[0], b = q[1], e = q[2];
            w[j][0][0] = a.x; w[j][0][1] = a.y; w[j][0][2] = a.z;
            w[j][1][0] = a.w; w[j][1][1] = b.x; w[j][1][2] = b.y;
            w[j][2][0] = b.z; w[j][2][1] = b.w; w[j][2][2] = e.x;
            w[j][3][0] = e.y; w[j][3][1] = e.z; w[j][3][2] = e.w;
        } else {
#pragma unroll
            for (int h = 0; h < 4; ++h)
#pragma unroll
                for (int i = 0; i < 3; ++i) w[j][h][i] = st[(8 * h + r) * pitch + j * jstride_w + 3 * c + i];
        }
    }
    float d[JN][2][NT][4];
#pragma unroll
    for (int j = 0; j < JN; ++j)
#pragma unroll
        for (int u = 0; u < NT; ++u) {
            const float4 nc = ncorr[((grel + j) * NT + u) * 4];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                d[j][t][u][0] = nc.x;
                d[j][t][u][1] = nc.y;
                d[j][t][u][2] = nc.z;
                d[j][t][u][3] = nc.w;
            }
        }
    ksteps<0, JN, MT, NT>(w, xs_lane + grel * 8 * MT * 4, 1, d, magic);
#pragma unroll
    for (int j = 0; j < JN; ++j)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                acc[t][u][0] = fmaf(s[j][2 * t], d[j][t][u][0], acc[t][u][0]);
                acc[t][u][1] = fmaf(s[j][2 * t], d[j][t][u][1], acc[t][u][1]);
                acc[t][u][2] = fmaf(s[j][2 * t + 1], d[j][t][u][2], acc[t][u][2]);
                acc[t][u][3] = fmaf(s[j][2 * t + 1], d[j][t][u][3], acc[t][u][3]);
            }
}

// Store a block's fragment (tile t, n8 tile u) of this lane: rows 16t + r (+8), batch columns 8u + 2c (+1).
__device__ __forceinline__ void store_frag(uint16_t *y, int N, int M, int block, int t, int u, int r, int c,
                                           const float4 &v) {
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = block * kBlockRows + 16 * t + r + ((i < 2) ? 0 : 8);
        const int m = 8 * u + 2 * c + (i & 1);
        if (row < N && m < M) y[static_cast<int64_t>(m) * N + row] = f32_to_bf16_rn(e[i]);
    }
}

template <int MT, bool NATIVE>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_split_kernel(const __grid_constant__ Params p) {
    static_assert(MT == 1 || MT == 2 || MT == 4 || MT == 8 || MT == 16, "batch rows padded to 1, 2, 4, 8, 16");
    constexpr int NT = n_tiles(MT);
    constexpr int kStageGroups = stage_groups_for(MT);
    constexpr int kPitchS = kStageGroups * kWordsPerGroup;
    constexpr int kStageBytes = stage_bytes(MT);
    extern __shared__ __align__(128) uint8_t smem[];
    const int M = p.M, N = p.N, G = p.G, C = p.C;
    const int depth = p.depth;
    const SmemLayout L = smem_layout(p.gs_max, MT, depth, p.nb_max, C);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int r = lane >> 2;
    const int c = lane & 3;
    pdl_trigger();  // the next kernel in the stream may start its own set-up

    // this CTA: cluster `cl`, rank q; its blocks and its K slice
    const int cl = blockIdx.x / C, q = blockIdx.x - cl * C;
    const int NB = (N + kBlockRows - 1) / kBlockRows;
    const int b_begin = static_cast<int>(static_cast<int64_t>(NB) * cl / p.ncl);
    const int b_end = static_cast<int>(static_cast<int64_t>(NB) * (cl + 1) / p.ncl);
    const int gq0 = G * q / C, Gs = G * (q + 1) / C - gq0;
    const int64_t units = static_cast<int64_t>(b_end - b_begin) * Gs;
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

    // The warp's range as a flat sequence of stages over [u0, u1) (a stage never crosses a
    // block boundary).  Two cursors (block index within the CTA's range, slice group) walk it:
    // one issues copies, one computes.
    const int64_t blk0 = Gs > 0 ? u0 / Gs : 0;
    const int g_first0 = static_cast<int>(u0 - blk0 * Gs);
    const int64_t last = u1 - 1;
    const int64_t blk_last = (u1 > u0) ? last / Gs : blk0;
    const int g_end_last = (u1 > u0) ? static_cast<int>(last - blk_last * Gs) + 1 : 0;
    auto stage_groups = [&](int64_t bl, int g) {
        const int end = (bl == blk_last) ? g_end_last : Gs;
        const int left = end - g;
        return left < kStageGroups ? left : kStageGroups;
    };
    auto advance = [&](int64_t &bl, int &g, int ng) {
        g += ng;
        const int end = (bl == blk_last) ? g_end_last : Gs;
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
                bulk_copy_g2s(dst,
                              p.native + (static_cast<int64_t>(row0 / kBlockRows) * G + gq0 + g) * kNativeGroupWords,
                              ng * kBox1Bytes, bar);
            } else if (ng == kStageGroups && p.hasS) {
                mbar_arrive_expect_tx(bar, kStageBytes);
                tma_load_2d(dst, &p.tmapS, (gq0 + g) * kWordsPerGroup, row0, bar);
            } else {
                mbar_arrive_expect_tx(bar, ng * kBox1Bytes);
                for (int j = 0; j < ng; ++j)
                    tma_load_2d(dst + j * kBox1Bytes, &p.tmap1, (gq0 + g + j) * kWordsPerGroup, row0, bar);
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
            const int end = (bl == blk_last) ? g_end_last : Gs;
            n += (end - g + kStageGroups - 1) / kStageGroups;
            ++bl;
            g = 0;
        }
        return n;
    }();

    int64_t ibl = blk0;
    int ig = g_first0;
    int issued = 0;
    int issue_slot = 0;  // == issued % depth
    // x (and, at the end, y) may belong to the previous kernel in the stream
    pdl_wait();
    decode::Params dp;  // prepare_x reads x, M and K only
    dp.x = p.x;
    dp.M = M;
    dp.K = p.K;
    decode::SmemLayout dl;
    dl.xs_off = L.xs_off;
    dl.corr_off = L.corr_off;
    dl.cpart_off = L.cpart_off;
    decode::prepare_x<MT>(dp, smem, dl, gq0, Gs);
    // each MMA chain starts from -corr: (-corr[8u+2c], -corr[8u+2c+1]) for rows r and r+8
    {
        const float *cf = reinterpret_cast<const float *>(smem + L.corr_off);
        float4 *nq = reinterpret_cast<float4 *>(smem + L.ncorr_off);
        for (int it = threadIdx.x; it < Gs * NT * 4; it += blockDim.x) {
            const int cc = it & 3, u = (it >> 2) % NT, g = it / (4 * NT);
            const float a = -cf[g * 8 * NT + 8 * u + 2 * cc], b = -cf[g * 8 * NT + 8 * u + 2 * cc + 1];
            nq[it] = make_float4(a, b, a, b);
        }
        __syncthreads();
    }
    // The first weight stages are issued only now.  Issued before x is prepared, their copies
    // slow the CTA's loads of x, the main loop starts later, and a call takes longer: 47.4 against
    // 45.1 us at M = 16 and 33.3 against 31.5 us at M = 8 on gate_proj.  (The stream-K decode,
    // whose x is a quarter of the size or less, gains from issuing them first.)
    for (; issued < depth - 1 && issued < nstages_total; ++issued) {
        advance(ibl, ig, issue(ibl, ig, issue_slot));
        issue_slot = (issue_slot + 1 == depth) ? 0 : issue_slot + 1;
    }

    // B fragments: lanes whose batch row is >= MT read words of other rows; the MMA keeps
    // columns apart and those columns are never stored.
    const uint2 *xs_lane = reinterpret_cast<const uint2 *>(smem + L.xs_off) + (r * 4 + c);
    const float4 *ncorr = reinterpret_cast<const float4 *>(smem + L.ncorr_off) + c;
    float4 *park = reinterpret_cast<float4 *>(smem + L.slot_off) + warp * 2 * NT * 32;
    float4 *pb = reinterpret_cast<float4 *>(smem + L.pb_off);

    // a block's sums over the CTA's slice: to y (C == 1), or into slot [q] of the block in the
    // shared memory of the rank that owns it
    const int nbc = b_end - b_begin;
    const int share = share_blocks(p.nb_max, C);
    auto emit = [&](int block, const float (&v)[2][NT][4]) {
        const int lb = block - b_begin;
        int qo = 0;  // owner rank: lb in [nbc*qo/C, nbc*(qo+1)/C)
        while (qo + 1 < C && lb >= nbc * (qo + 1) / C) ++qo;
        const int lo = lb - nbc * qo / C;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                const float4 f = make_float4(v[t][u][0], v[t][u][1], v[t][u][2], v[t][u][3]);
                if (C == 1) {
                    store_frag(p.y, N, M, block, t, u, r, c, f);
                } else {
                    const uint32_t local = smem_addr(pb + ((((q * share + lo) * 2 + t) * NT + u) * 32 + lane));
                    st_dsmem_f4(map_to_rank(local, qo), f);
                }
            }
    };

    bool ok = true;
    const uint32_t magic = decode::pinned_magic();
    uint32_t phase_bits = 0;
    float acc[2][NT][4] = {};
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
            if (ng == kStageGroups && (NATIVE || p.hasS)) {
                groups<kStageGroups, MT, NT, NATIVE>(st, kPitchS, kWordsPerGroup, cg, gq0 + cg, xs_lane, ncorr, sc, r,
                                                     c, acc, magic);
            } else {
                for (int j = 0; j < ng; ++j)
                    groups<1, MT, NT, NATIVE>(st + j * kBlockRows * kPitch1, kPitch1, 0, cg + j, gq0 + cg + j, xs_lane,
                                              ncorr, sc, r, c, acc, magic);
            }
        }
        // End of a segment.  A whole block is emitted.  A split block is either this warp's
        // first segment starting after the block's group 0 (a later part of a block owned by an
        // earlier warp: parked in the warp's slot), or the block's first part, which is this
        // warp's last segment (it owns the block and keeps the sums in acc until the end).
        const int g_stage = cg;
        const int64_t bl_stage = cbl;
        advance(cbl, cg, ng);
        if (cbl != bl_stage) {
            const int g_first = (bl_stage == blk0) ? g_first0 : 0;
            const bool whole = (g_first == 0) && (g_stage + ng == Gs);
            if (g_first == 0 && !whole) continue;  // owned: the range ends here, acc holds it
            if (whole) {
                if (ok) emit(block, acc);
            } else {
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int u = 0; u < NT; ++u)
                        park[(t * NT + u) * 32 + lane] = make_float4(acc[t][u][0], acc[t][u][1], acc[t][u][2], acc[t][u][3]);
            }
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int u = 0; u < NT; ++u)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[t][u][i] = 0.f;
        }
    }

    __syncthreads();
    // Owners: the warp holding group 0 of a split block adds the later warps' parts (each their
    // first segment, parked in their slot) to its own, in ascending warp (= ascending group) order.
    if (ok && u1 > u0) {
        // the last block starting inside [u0, u1): if it does not end inside the range it is
        // split, continues in later warps, and this warp owns it
        const int64_t own_u = ((u1 - 1) / Gs) * Gs;
        if (own_u >= u0 && own_u + Gs > u1) {
            const int block = b_begin + static_cast<int>(own_u / Gs);
            const float4 *all = reinterpret_cast<const float4 *>(smem + L.slot_off);
            // The later warps whose range starts inside the block, in warp order.  Warp starts
            // increase with the warp, so "starts before the block ends" selects a run of warps.
            // Four warps' parts are loaded before any is added (the loads overlap; the adds keep
            // warp order).  32-bit unit arithmetic: a CTA has fewer than 2^32 / kWarps units.
            const uint32_t units32 = static_cast<uint32_t>(units), own_end = static_cast<uint32_t>(own_u + Gs);
#pragma unroll
            for (int wc = 1; wc < kWarps; wc += 4) {
                float4 f[4][2][NT];
                bool use[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int w2 = wc + i;
                    const uint32_t a0 = units32 * static_cast<uint32_t>(w2) / kWarps;
                    const uint32_t a1 = units32 * static_cast<uint32_t>(w2 + 1) / kWarps;
                    use[i] = w2 < kWarps && w2 > warp && a0 < own_end && a1 > a0;
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int u = 0; u < NT; ++u)
                            f[i][t][u] = use[i] ? all[(w2 * 2 * NT + t * NT + u) * 32 + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (use[i]) {
#pragma unroll
                        for (int t = 0; t < 2; ++t)
#pragma unroll
                            for (int u = 0; u < NT; ++u) {
                                acc[t][u][0] += f[i][t][u].x;
                                acc[t][u][1] += f[i][t][u].y;
                                acc[t][u][2] += f[i][t][u].z;
                                acc[t][u][3] += f[i][t][u].w;
                            }
                    }
            }
            emit(block, acc);
        }
    }
    if (C == 1) return;

    // ---- the cluster: rank q adds the C slices of its blocks, in rank order ----
    // The barrier makes every rank's stores into this CTA's shared memory visible.  After it no
    // CTA touches another's shared memory, so a CTA may leave as soon as it is done.
    cluster_sync();
    const int sb0 = nbc * q / C, sb1 = nbc * (q + 1) / C;
    const int items = (sb1 - sb0) * 2 * NT * 32;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int ln = it & 31, u = (it >> 5) % NT, t = (it / (32 * NT)) & 1, lo = it / (64 * NT);
        float4 v = pb[((lo * 2 + t) * NT + u) * 32 + ln];
        for (int rk = 1; rk < C; ++rk) {
            const float4 f = pb[(((rk * share + lo) * 2 + t) * NT + u) * 32 + ln];
            v.x += f.x;
            v.y += f.y;
            v.z += f.z;
            v.w += f.w;
        }
        if (ok) store_frag(p.y, N, M, b_begin + sb0 + lo, t, u, ln >> 2, ln & 3, v);
    }
}

struct LaunchPlan {
    int mt, C, ncl, depth, gs_max, nb_max, smem_bytes;
    bool ok;
    int warps() const { return kWarps; }
};

// Ring stages that fit (2..kMaxDepth), or 0.
inline int fitting_depth(int gs, int mt, int nb, int C) {
    for (int d = kMaxDepth; d >= 2; --d)
        if (smem_layout(gs, mt, d, nb, C).total <= kSmemLimit) return d;
    return 0;
}

// Clusters of C CTAs that are resident at once; `active_clusters(C, smem)` asks the
// device (occupancy query) and returns 0 when it cannot say.  Whether a plan exists does
// not depend on that answer (the route query asks without a device): when fewer clusters
// are resident than SMs / C and their larger share of blocks would not fit in shared
// memory, the clusters run in waves instead.
template <class ActiveClusters>
inline LaunchPlan plan(int M, int N, int K, int num_sms, ActiveClusters active_clusters) {
    LaunchPlan best{};
    best.ok = false;
    const int mt = decode::padded_batch(M);
    best.mt = mt;
    const int G = K / kGroup;
    const int NB = (N + kBlockRows - 1) / kBlockRows;
    int64_t best_cost = -1;
    for (int C = 1; C <= kMaxCluster && C <= G; C *= 2) {
        const int gs = (G + C - 1) / C;
        int ncl = num_sms / C < NB ? num_sms / C : NB;
        if (ncl <= 0) break;
        int nb = (NB + ncl - 1) / ncl;
        int depth = fitting_depth(gs, mt, nb, C);
        if (depth == 0) continue;
        int waves = 1;
        for (int pass = 0; C > 1 && pass < 2; ++pass) {
            const int fit = active_clusters(C, smem_layout(gs, mt, depth, nb, C).total);
            if (fit <= 0 || fit >= ncl) break;
            const int nb_fit = (NB + fit - 1) / fit;
            const int depth_fit = fitting_depth(gs, mt, nb_fit, C);
            if (depth_fit == 0) {
                waves = (ncl + fit - 1) / fit;
                break;
            }
            ncl = fit;  // plan for the clusters that are resident at once
            nb = nb_fit;
            depth = depth_fit;
        }
        // The slowest CTA's (block, group) units, plus the cluster reduction.  The kernel streams
        // from HBM: CTAs with less work finish early and leave their bandwidth to the others, so
        // a finer split pays only when it gives many more SMs work (small N) or when x' of the
        // whole K range does not fit; a cluster costs about an eighth of the work.
        const int64_t cost = static_cast<int64_t>(waves) * nb * gs * 16 * (C > 1 ? 9 : 8) / 8;
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best.ok = true;
            best.mt = mt;
            best.C = C;
            best.ncl = ncl;
            best.depth = depth;
            best.gs_max = gs;
            best.nb_max = nb;
            best.smem_bytes = smem_layout(gs, mt, depth, nb, C).total;
        }
    }
    return best;
}

}  // namespace dsplit
}  // namespace w3
