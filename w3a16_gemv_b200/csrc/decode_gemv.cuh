// decode_gemv.cuh -- y = x * W^T for M <= 16 (decode), W in the exact-width
// uint3 / group-128 / bf16-scale format of the GSQ model card ("Storage
// layout" section), never materialised.
//
// The work is bound by HBM: each weight costs 3.125 bits of traffic and is
// used M times.  What the kernel has to make cheap is the unpack, which at
// M = 1 is the only arithmetic per weight.  Structure:
//
//  * A warp owns 32 weight rows (two 16-row MMA tiles) and streams its K range
//    through a private ring of shared-memory stages.  Each lane issues one
//    bulk copy (TMA engine, 1-D form) per stage for one row; completion is
//    counted on an mbarrier in transaction bytes.  A stage holds 3 groups
//    (144 bytes) of each row; the row pitch of 36 words keeps the per-lane
//    reads below free of shared-memory bank conflicts.
//  * Lane (r = lane/4, c = lane%4) unpacks 32-code block c of the current
//    group for rows r, r+8 of each tile.  A block becomes 16 bf16x2 registers
//    with one LOP3 per pair plus 9 shifts: each LOP3 drops two 3-bit codes into
//    the mantissa of bf16 128.0 at bit offsets e_lo, e_hi, giving the exact
//    values 128 + c*2^e.
//  * Those registers are the A operand (16 rows x 16 k) of mma.m16n8k16 with
//    fp32 accumulation; x (pre-scaled by 2^-e per slot and permuted to match
//    the pair order, prepared once per CTA in shared memory) is the B operand,
//    one column per batch row, shared by both tiles.  All 16 k of one MMA lie
//    in one 128-group, so the group scale is applied in fp32 after the 8 MMAs
//    of the group:  y += s[n,g] * (sum_k v_k x'_k - corr_g), where
//    corr_g = sum_k (128*2^-e_k + 4) x_k removes the 128 offset and the level
//    shift q = c - 4.  Nothing is rounded before the fp32 accumulation.
//  * The K range may be split over a thread-block cluster (split-K for short
//    or tall matrices); the partial sums are added in fixed rank order through
//    distributed shared memory, so results are deterministic.
#pragma once

#include <algorithm>

#include "common.cuh"

namespace w3 {
namespace decode {

constexpr int kTileRows = 16;                       // rows of one MMA tile
constexpr int kTilesPerWarp = 2;
constexpr int kRowsPerWarp = kTileRows * kTilesPerWarp;  // 32: one bulk copy per lane per stage
constexpr int kWarps = 2;                           // warps per CTA
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;  // 64
constexpr int kStageGroups = 3;                     // groups per stage (odd: conflict-free row pitch)
constexpr int kDepth = 4;                           // ring stages per warp
static_assert(kStageGroups % 2 == 1, "an odd number of groups per stage keeps the row pitch conflict-free");
constexpr int kRowPitchWords = kStageGroups * kWordsPerGroup;   // 36 for 3 groups
constexpr int kStageBytes = kRowsPerWarp * kRowPitchWords * 4;  // 4608 for 3 groups
static_assert(kStageBytes % 128 == 0, "a tiled TMA destination in shared memory must be 128-byte aligned");
constexpr int kXsBudgetBytes = 64 * 1024;                       // prepared-x budget per CTA
constexpr int kMaxCluster = 8;

// One extraction: codes `lo` and `hi` of a 32-code block land in the low and
// high bf16 halves with mantissa offsets e_lo, e_hi.
struct PairSpec {
    int lo, hi, elo, ehi;
};

// The 16 pairs of a block in the order they feed the MMA (pairs 2t and 2t+1
// form k-step t).  Chosen by an exhaustive search for the fewest shifts.
__host__ __device__ constexpr PairSpec pair_spec(int i) {
    constexpr PairSpec t[16] = {{0, 4, 4, 0},   {1, 7, 1, 3},   {2, 6, 4, 0},   {3, 9, 1, 3},
                                {5, 10, 4, 3},  {8, 12, 4, 0},  {11, 17, 1, 3}, {13, 18, 1, 0},
                                {14, 19, 4, 3}, {15, 21, 1, 3}, {16, 20, 4, 0}, {22, 27, 2, 1},
                                {23, 28, 1, 0}, {24, 29, 4, 3}, {25, 31, 1, 3}, {26, 30, 4, 0}};
    return t[i];
}

__host__ __device__ constexpr uint32_t pair_mask(int elo, int ehi) {
    return (7u << elo) | (7u << (16 + ehi));
}

// Mantissa offset of code j of a block under the schedule above.
__host__ __device__ constexpr int code_shift(int j) {
    int e = 0;
    for (int i = 0; i < 16; ++i) {
        if (pair_spec(i).lo == j) e = pair_spec(i).elo;
        if (pair_spec(i).hi == j) e = pair_spec(i).ehi;
    }
    return e;
}

constexpr uint32_t kMagic = 0x43004300u;  // bf16x2 (128.0, 128.0)

// kMagic in a register the compiler cannot rematerialise: kernels create it once
// and pass it to the unpack, which otherwise rebuilds the constant before many
// of its LOP3s.
__device__ __forceinline__ uint32_t pinned_magic() {
    uint32_t m;
    asm volatile("mov.b32 %0, %1;" : "=r"(m) : "n"(kMagic));
    return m;
}


// Unpack one 96-bit block (w0, w1, w2) into the 16 bf16x2 pair registers.
// Window s (a shift of the block by s bits) feeds the pairs whose codes sit at
// window bits e_lo and 16 + e_hi.
__device__ __forceinline__ void unpack_block(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t (&a)[16],
                                             uint32_t magic = kMagic) {
    const uint32_t wm4 = w0 << 4;                     // s = -4
    const uint32_t w_2 = w0 >> 2;                     // s = 2
    const uint32_t w_8 = w0 >> 8;                     // s = 8
    const uint32_t w11 = __funnelshift_r(w0, w1, 11); // s = 11
    const uint32_t w20 = __funnelshift_r(w0, w1, 20); // s = 20
    const uint32_t w38 = w1 >> 6;                     // s = 38
    const uint32_t w44 = __funnelshift_r(w1, w2, 12); // s = 44
    const uint32_t w68 = w2 >> 4;                     // s = 68
    const uint32_t w74 = w2 >> 10;                    // s = 74
    a[0] = and_or<pair_mask(4, 0)>(wm4, magic);
    a[1] = and_or<pair_mask(1, 3)>(w_2, magic);
    a[2] = and_or<pair_mask(4, 0)>(w_2, magic);
    a[3] = and_or<pair_mask(1, 3)>(w_8, magic);
    a[4] = and_or<pair_mask(4, 3)>(w11, magic);
    a[5] = and_or<pair_mask(4, 0)>(w20, magic);
    a[6] = and_or<pair_mask(1, 3)>(w1, magic);
    a[7] = and_or<pair_mask(1, 0)>(w38, magic);
    a[8] = and_or<pair_mask(4, 3)>(w38, magic);
    a[9] = and_or<pair_mask(1, 3)>(w44, magic);
    a[10] = and_or<pair_mask(4, 0)>(w44, magic);
    a[11] = and_or<pair_mask(2, 1)>(w2, magic);
    a[12] = and_or<pair_mask(1, 0)>(w68, magic);
    a[13] = and_or<pair_mask(4, 3)>(w68, magic);
    a[14] = and_or<pair_mask(1, 3)>(w74, magic);
    a[15] = and_or<pair_mask(4, 0)>(w74, magic);
}

// Pair I of a block (the I-th register of unpack_block), computed on its own so
// that callers can interleave the unpack with the MMAs; with the index known at
// compile time the windows shared by two pairs are computed once.
template <int I>
__device__ __forceinline__ uint32_t unpack_pair(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t magic = kMagic) {
    if constexpr (I == 0) return and_or<pair_mask(4, 0)>(w0 << 4, magic);
    if constexpr (I == 1) return and_or<pair_mask(1, 3)>(w0 >> 2, magic);
    if constexpr (I == 2) return and_or<pair_mask(4, 0)>(w0 >> 2, magic);
    if constexpr (I == 3) return and_or<pair_mask(1, 3)>(w0 >> 8, magic);
    if constexpr (I == 4) return and_or<pair_mask(4, 3)>(__funnelshift_r(w0, w1, 11), magic);
    if constexpr (I == 5) return and_or<pair_mask(4, 0)>(__funnelshift_r(w0, w1, 20), magic);
    if constexpr (I == 6) return and_or<pair_mask(1, 3)>(w1, magic);
    if constexpr (I == 7) return and_or<pair_mask(1, 0)>(w1 >> 6, magic);
    if constexpr (I == 8) return and_or<pair_mask(4, 3)>(w1 >> 6, magic);
    if constexpr (I == 9) return and_or<pair_mask(1, 3)>(__funnelshift_r(w1, w2, 12), magic);
    if constexpr (I == 10) return and_or<pair_mask(4, 0)>(__funnelshift_r(w1, w2, 12), magic);
    if constexpr (I == 11) return and_or<pair_mask(2, 1)>(w2, magic);
    if constexpr (I == 12) return and_or<pair_mask(1, 0)>(w2 >> 4, magic);
    if constexpr (I == 13) return and_or<pair_mask(4, 3)>(w2 >> 4, magic);
    if constexpr (I == 14) return and_or<pair_mask(1, 3)>(w2 >> 10, magic);
    return and_or<pair_mask(4, 0)>(w2 >> 10, magic);
}

// x * 2^-e as bf16 bits (exact: only the exponent changes).
__device__ __forceinline__ uint32_t scaled_bf16(uint16_t xb, int e) {
    const float f = bf16_bits_to_f32(xb) * __int_as_float((127 - e) << 23);
    return __float_as_uint(f) >> 16;
}

struct SmemLayout {
    int xs_off, corr_off, cpart_off, bar_off, ring_off, total;
};

__host__ __device__ inline int align_up(int v, int a) { return (v + a - 1) / a * a; }

// gchunk: groups of prepared x held at once; mt: batch rows padded to 1/2/4/8/16.
__host__ __device__ inline SmemLayout smem_layout(int gchunk, int mt) {
    const int nt = (mt + 7) / 8;
    SmemLayout L;
    L.xs_off = 0;                                                    // uint2 [gchunk][8][mt][4]
    L.corr_off = align_up(L.xs_off + gchunk * 8 * mt * 4 * 8, 16);   // float [gchunk][8*nt]
    L.cpart_off = align_up(L.corr_off + gchunk * 8 * nt * 4, 16);    // float [gchunk][mt][4]
    L.bar_off = align_up(L.cpart_off + gchunk * mt * 4 * 4, 16);     // u64 [kWarps][kDepth]
    L.ring_off = align_up(L.bar_off + kWarps * kDepth * 8, 128);     // [kWarps][kDepth][kStageBytes]
    L.total = L.ring_off + kWarps * kDepth * kStageBytes;
    return L;
}

struct Params {
    CUtensorMap tmap;    // packed [N][3K/32] u32, box [kRowsPerWarp][kRowPitchWords] (when use_tma2d)
    const uint16_t *x;
    const uint32_t *packed;
    const uint16_t *scales;
    uint16_t *y;
    int M, N, K;
    int groups_per_cta;  // K range of one cluster rank, in groups
    int gchunk;          // groups of prepared x per chunk
    int use_tma2d;       // 1: one tiled TMA copy per stage; 0: one 1-D bulk copy per row
};

// Prepare x' and the per-group corrections for groups [g0, g0 + ng) of the
// CTA's range.  Batch rows M..MT-1 are zero.
template <int MT>
__device__ __forceinline__ void prepare_x(const Params &p, uint8_t *smem, const SmemLayout &L, int g0, int ng) {
    constexpr int NT = (MT + 7) / 8;
    uint32_t *xs = reinterpret_cast<uint32_t *>(smem + L.xs_off);
    float *corr = reinterpret_cast<float *>(smem + L.corr_off);
    float *cpart = reinterpret_cast<float *>(smem + L.cpart_off);
    const int items = ng * MT * 4;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int c = it & 3;
        const int m = (it >> 2) % MT;
        const int g = it / (4 * MT);
        uint4 raw[4] = {};
        if (m < p.M) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.x + static_cast<int64_t>(m) * p.K +
                                                               static_cast<int64_t>(g0 + g) * kGroup + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i) raw[i] = __ldg(src + i);
        }
        const uint16_t *xv = reinterpret_cast<const uint16_t *>(raw);
        uint32_t *dst = xs + (((g * 8) * MT + m) * 4 + c) * 2;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const PairSpec ps = pair_spec(i);
            // uint2 index ((g*8 + t)*MT + m)*4 + c, component i&1, t = i/2
            dst[(i >> 1) * MT * 8 + (i & 1)] =
                scaled_bf16(xv[ps.lo], ps.elo) | (scaled_bf16(xv[ps.hi], ps.ehi) << 16);
        }
        // corr partial, positions in ascending order for a fixed summation order
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            part = fmaf(128.0f / static_cast<float>(1 << code_shift(j)) + 4.0f, bf16_bits_to_f32(xv[j]), part);
        cpart[(g * MT + m) * 4 + c] = part;
    }
    __syncthreads();
    for (int it = threadIdx.x; it < ng * 8 * NT; it += blockDim.x) {
        const int m = it % (8 * NT);
        const int g = it / (8 * NT);
        float v = 0.f;
        if (m < MT) {
            const float *q = cpart + (g * MT + m) * 4;
            v = ((q[0] + q[1]) + q[2]) + q[3];
        }
        corr[it] = v;
    }
    __syncthreads();
}

template <int MT>
__global__ void __launch_bounds__(kWarps * 32, 4) decode_kernel(const __grid_constant__ Params p) {
    constexpr int NT = (MT + 7) / 8;
    extern __shared__ __align__(128) uint8_t smem[];
    const int M = p.M, N = p.N;
    const int G = p.K / kGroup;
    const int words_per_row = G * kWordsPerGroup;
    const SmemLayout L = smem_layout(p.gchunk, MT);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int r = lane >> 2;  // fragment row group
    const int c = lane & 3;   // block within the group / thread in quad

    const int cta_g0 = blockIdx.y * p.groups_per_cta;
    const int cta_g1 = min(G, cta_g0 + p.groups_per_cta);

    const int n0 = blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
    const int nvalid = max(0, min(kRowsPerWarp, N - n0));

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off) + warp * kDepth;
    uint8_t *ring = smem + L.ring_off + warp * kDepth * kStageBytes;
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t ring0 = smem_addr(ring);
    if (lane == 0) {
        for (int s = 0; s < kDepth; ++s) mbar_init(bar0 + 8 * s, 1);
        mbar_init_fence();
    }
    __syncwarp();

    // B fragments of lane (r, c): batch row m = 8*nt + r; rows >= MT read nothing (stay 0)
    const uint2 *xs_lane = reinterpret_cast<const uint2 *>(smem + L.xs_off) + (r * 4 + c);
    const bool b_active = (MT >= 8) || (r < MT);
    const float *corr = reinterpret_cast<const float *>(smem + L.corr_off) + 2 * c;

    float yacc[kTilesPerWarp][NT][4];
#pragma unroll
    for (int t = 0; t < kTilesPerWarp; ++t)
#pragma unroll
        for (int u = 0; u < NT; ++u)
#pragma unroll
            for (int i = 0; i < 4; ++i) yacc[t][u][i] = 0.f;

    bool ok = true;
    uint32_t phase_bits = 0;  // parity of the next wait, one bit per ring slot

    // scale rows of this lane: tile t, half h -> row n0 + 16t + 8h + r (clamped)
    const uint16_t *sc[kTilesPerWarp][2];
#pragma unroll
    for (int t = 0; t < kTilesPerWarp; ++t)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            sc[t][h] = p.scales + static_cast<int64_t>(min(n0 + 16 * t + 8 * h + r, N - 1)) * G;

    for (int ch0 = cta_g0; ch0 < cta_g1; ch0 += p.gchunk) {
        const int ch1 = min(ch0 + p.gchunk, cta_g1);
        const int ng_chunk = ch1 - ch0;
        const int nstages = (ng_chunk + kStageGroups - 1) / kStageGroups;

        // stage s of this chunk -> ring slot s % kDepth; called by the whole warp
        auto issue = [&](int s) {
            const int slot = s % kDepth;
            const int gs = ch0 + s * kStageGroups;
            if (p.use_tma2d) {
                __syncwarp();  // every lane is done reading the slot being refilled
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar0 + 8 * slot, kStageBytes);
                    tma_load_2d(ring0 + slot * kStageBytes, &p.tmap, gs * kWordsPerGroup, n0, bar0 + 8 * slot);
                }
                return;
            }
            const uint32_t bytes = min(kStageGroups, ch1 - gs) * kBytesPerGroup;
            if (lane == 0) mbar_arrive_expect_tx(bar0 + 8 * slot, bytes * nvalid);
            __syncwarp();  // also: every lane is done reading the slot being refilled
            if (lane < nvalid) {
                const uint32_t *src = p.packed + static_cast<int64_t>(n0 + lane) * words_per_row +
                                      static_cast<int64_t>(gs) * kWordsPerGroup;
                bulk_copy_g2s(ring0 + slot * kStageBytes + lane * kRowPitchWords * 4, src, bytes, bar0 + 8 * slot);
            }
        };

        // start streaming weights before x' is prepared
        int issued = 0;
        if (nvalid > 0 && ok) {
            for (; issued < kDepth - 1 && issued < nstages; ++issued) issue(issued);
        }
        if (ch0 != cta_g0) __syncthreads();  // every warp is done with the previous chunk's x'
        prepare_x<MT>(p, smem, L, ch0, ng_chunk);

        if (nvalid == 0) continue;
        for (int s = 0; s < nstages; ++s) {
            if (ok && issued < nstages) issue(issued++);
            if (s >= issued) break;  // only after a timeout: nothing left in flight
            const int slot = s % kDepth;
            const int gs = s * kStageGroups;  // chunk-relative
            const int ng = min(kStageGroups, ng_chunk - gs);
            const uint32_t parity = (phase_bits >> slot) & 1u;
            phase_bits ^= 1u << slot;
            // warp-uniform: a timeout seen by any lane stops the whole warp
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar0 + 8 * slot, parity) && ok);
            if (!ok) continue;  // drain the copies still in flight, compute nothing
            const uint32_t *st = reinterpret_cast<const uint32_t *>(ring + slot * kStageBytes);
#pragma unroll
            for (int j = 0; j < kStageGroups; ++j) {
                if (j >= ng) break;
                const int g = gs + j;  // chunk-relative group
                const int gabs = ch0 + g;
                uint2 bfr[NT][8];
#pragma unroll
                for (int u = 0; u < NT; ++u)
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        bfr[u][k] = make_uint2(0u, 0u);
                        if (b_active) bfr[u][k] = xs_lane[(g * 8 + k) * MT * 4 + u * 32];
                    }
                float2 cr[NT];
#pragma unroll
                for (int u = 0; u < NT; ++u) cr[u] = *reinterpret_cast<const float2 *>(corr + g * 8 * NT + 8 * u);
#pragma unroll
                for (int t = 0; t < kTilesPerWarp; ++t) {
                    const float s_lo = bf16_bits_to_f32(__ldg(sc[t][0] + gabs));
                    const float s_hi = bf16_bits_to_f32(__ldg(sc[t][1] + gabs));
                    const uint32_t *pa = st + (16 * t + r) * kRowPitchWords + j * kWordsPerGroup + 3 * c;
                    const uint32_t *pb = pa + 8 * kRowPitchWords;
                    uint32_t A[16], B[16];
                    unpack_block(pa[0], pa[1], pa[2], A);
                    unpack_block(pb[0], pb[1], pb[2], B);
#pragma unroll
                    for (int u = 0; u < NT; ++u) {
                        float d[4] = {-cr[u].x, -cr[u].y, -cr[u].x, -cr[u].y};
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_bf16_m16n8k16(d, A[2 * k], B[2 * k], A[2 * k + 1], B[2 * k + 1], bfr[u][k].x,
                                              bfr[u][k].y, d);
                        yacc[t][u][0] = fmaf(s_lo, d[0], yacc[t][u][0]);
                        yacc[t][u][1] = fmaf(s_lo, d[1], yacc[t][u][1]);
                        yacc[t][u][2] = fmaf(s_hi, d[2], yacc[t][u][2]);
                        yacc[t][u][3] = fmaf(s_hi, d[3], yacc[t][u][3]);
                    }
                }
            }
        }
    }

    // split-K: add the cluster ranks' partials in rank order (rank 0 stores y)
    const uint32_t nranks = gridDim.y;
    bool store = true;
    if (nranks > 1) {
        __syncwarp();
        float4 *red = reinterpret_cast<float4 *>(ring);  // this warp's ring is idle now
#pragma unroll
        for (int t = 0; t < kTilesPerWarp; ++t)
#pragma unroll
            for (int u = 0; u < NT; ++u)
                red[(t * NT + u) * 32 + lane] = make_float4(yacc[t][u][0], yacc[t][u][1], yacc[t][u][2], yacc[t][u][3]);
        cluster_sync();
        const uint32_t rank = cluster_ctarank();
        if (rank == 0) {
            for (uint32_t q = 1; q < nranks; ++q) {
#pragma unroll
                for (int t = 0; t < kTilesPerWarp; ++t)
#pragma unroll
                    for (int u = 0; u < NT; ++u) {
                        const float4 v = ld_dsmem_f4(map_to_rank(smem_addr(red + (t * NT + u) * 32 + lane), q));
                        yacc[t][u][0] += v.x;
                        yacc[t][u][1] += v.y;
                        yacc[t][u][2] += v.z;
                        yacc[t][u][3] += v.w;
                    }
            }
        } else {
            store = false;
        }
        cluster_sync();
    }
    if (!store || !ok || nvalid == 0) return;
#pragma unroll
    for (int t = 0; t < kTilesPerWarp; ++t)
#pragma unroll
        for (int u = 0; u < NT; ++u)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = n0 + 16 * t + r + ((i < 2) ? 0 : 8);
                const int m = 8 * u + 2 * c + (i & 1);
                if (row < N && m < M) p.y[static_cast<int64_t>(m) * N + row] = f32_to_bf16_rn(yacc[t][u][i]);
            }
}

inline int padded_batch(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

struct LaunchPlan {
    int mt, cluster, groups_per_cta, gchunk, smem_bytes;
    dim3 grid;
};

// Split K over a cluster when there are too few row tiles to fill the GPU, or
// when the prepared x of the whole K range would not fit in shared memory.
inline LaunchPlan plan(int M, int N, int K, int num_sms) {
    LaunchPlan P;
    P.mt = padded_batch(M);
    const int G = K / kGroup;
    const int ctas_n = (N + kRowsPerCta - 1) / kRowsPerCta;
    const int warps_wanted = num_sms * 6;
    const int xs_per_group = 8 * P.mt * 4 * 8;
    int C = 1;
    while (C < kMaxCluster) {
        const int gpc = (G + C - 1) / C;
        const bool too_big = gpc * xs_per_group > kXsBudgetBytes;
        const bool too_few = ctas_n * C * kWarps < warps_wanted;
        const int gpc2 = (G + 2 * C - 1) / (2 * C);
        if ((too_big || too_few) && gpc2 >= 2) C *= 2;
        else break;
    }
    P.cluster = C;
    P.groups_per_cta = (G + C - 1) / C;
    // a chunk of prepared x is a whole number of stages unless it is the whole range
    int gchunk = std::min(P.groups_per_cta, kXsBudgetBytes / xs_per_group);
    if (gchunk < P.groups_per_cta) gchunk = std::max(kStageGroups, gchunk / kStageGroups * kStageGroups);
    P.gchunk = gchunk;
    P.smem_bytes = smem_layout(P.gchunk, P.mt).total;
    P.grid = dim3(ctas_n, C, 1);
    return P;
}

}  // namespace decode
}  // namespace w3
