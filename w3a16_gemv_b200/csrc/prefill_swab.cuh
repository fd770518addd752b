// prefill_swab.cuh -- y = x * W^T for large batches on the 5th-generation tensor
// cores with the operand roles swapped: the dequantized weights are the MMA's A
// operand, written by threads straight into tensor memory (tcgen05.st), and x is
// the B operand, copied into shared memory by TMA.  W is in the exact-width
// uint3 / group-128 / bf16-scale format of the GSQ model card ("Storage layout").
//
// Why: with the weights in shared memory (prefill_gemm.cuh) every stage stores
// the dequantized tile there and the tensor cores read it once per 128-row x
// tile, next to the x tiles and the TMA writes: the shared-memory pipe, not the
// tensor pipe, sets the pace.  With the weights in tensor memory, shared memory
// only carries x (written once by TMA, read once per MMA) and the packed words.
//
//  * CTA tile: 128 rows of W (one tensor-memory lane each, UMMA M = 128) x BN
//    rows of x (UMMA N, a multiple of 16 up to 256); K in stages of 64 for x
//    and of one 128-code group for W.  Tensor memory: the fp32 accumulator D
//    [128 lanes][BN columns] and a ring of 3 A stages of 64 columns.
//  * x: one tiled TMA copy per stage ([BN rows][64 k], 128-byte swizzle, the
//    K-major layout the UMMA descriptors describe), 6 stages deep.
//  * Packed W: a producer warp copies the CTA's 128 rows four stages at a time
//    ([128 rows][24 words] boxes), double-buffered.
//  * 8 dequantizing warps, two per tensor-memory lane quarter: each thread owns
//    one W row and half of each group's 128 codes, expands them to bf16(q * s)
//    (the same exact expansion as the shared-memory prefill: 12 code bits times
//    0x2001, one LOP3 per pair, a bf16x2 subtract of 132 and a bf16x2 multiply
//    by the group scale, rounded once) and stores 32 columns of the A stage.
//  * One elected lane issues 4 tcgen05.mma per x stage (A from tensor memory,
//    B = x from shared memory) and commits each x stage, and each group's A
//    stage, back to its producers.
//  * Epilogue: the dequantizing warps read D with tcgen05.ld (lane n = W row,
//    column m = x row), round to bf16 and store y[m][n]; a warp's 32 lanes
//    write 32 consecutive n of one y row (64 bytes) per store.
// CTAs that share a W tile are launched next to each other (x tile fastest),
// so its packed words come from DRAM once.  All waits are bounded.
#pragma once

#include "common.cuh"
#include "prefill_gemm.cuh"

namespace w3 {
namespace prefill_ab {

using prefill::desc_add;
using prefill::expand_half;
using prefill::fence_async_smem;
using prefill::make_idesc;
using prefill::mbar_arrive;
using prefill::sw128_kmajor_desc;
using prefill::tc_fence_after;
using prefill::tc_fence_before;
using prefill::tmem_ld32;
using prefill::umma_commit;

constexpr int kRowsW = 128;        // W rows per CTA: UMMA M, one tensor-memory lane each
constexpr int kMaxBN = 256;        // x rows per CTA at most: UMMA N
constexpr int kStageK = 64;        // k per stage: one 128-byte swizzle row of bf16
constexpr int kXStages = 6;        // x stages in shared memory
constexpr int kAStages = 3;        // A stages in tensor memory, one 128-code group each
constexpr int kChunkStages = 4;    // stages per packed-word copy
constexpr int kStageWords = kStageK * 3 / 32;            // 6 packed words per row and stage
constexpr int kChunkWords = kChunkStages * kStageWords;  // 24
constexpr int kDequantWarps = 8;   // two per lane quarter: W row x half of each stage's codes
constexpr int kFirstDequantWarp = 3;
constexpr int kThreads = (kFirstDequantWarp + kDequantWarps) * 32;  // x TMA, MMA, W TMA, dequant
constexpr int kXStageBytes = kMaxBN * kStageK * 2;        // 32 KB
constexpr int kWBufBytes = kRowsW * kChunkWords * 4;      // 12 KB
constexpr int kACols = kGroup / 2;                        // 64 columns per A stage (bf16 pairs)
constexpr int kACol0 = kMaxBN;                            // A ring after the accumulator
constexpr int kTmemCols = 512;
static_assert(kACol0 + kAStages * kACols <= kTmemCols, "tensor memory columns");
static_assert(kXStageBytes % 1024 == 0 && kWBufBytes % 128 == 0, "TMA destinations: 1024 / 128-byte alignment");

struct SmemLayout {
    static constexpr int x_off = 0;                                   // [kXStages][kMaxBN rows][128 B]
    static constexpr int w_off = x_off + kXStages * kXStageBytes;     // [2][kRowsW rows][24 words]
    static constexpr int sink_off = w_off + 2 * kWBufBytes;           // u32 per dequant thread
    static constexpr int bar_off = sink_off + kDequantWarps * 32 * 4;
    // x_full, x_empty [kXStages]; a_full, a_empty [kAStages]; w_full, w_empty [2]; acc
    static constexpr int nbars = 2 * kXStages + 2 * kAStages + 4 + 1;
    static constexpr int tmem_slot_off = bar_off + nbars * 8;
    static constexpr int total = tmem_slot_off + 16 + 1024;  // + slack to align the base to 1024
};
static_assert(SmemLayout::total <= 227 * 1024, "shared memory per CTA");

struct Params {
    CUtensorMap tmap_x;  // x [M][K] bf16, box [bn rows][64 k], 128-byte swizzle
    CUtensorMap tmap_w;  // packed [N][3K/32] u32, box [128 rows][24 words]
    const uint16_t *scales;
    uint16_t *y;
    int M, N, K;
    int bn;          // x rows per CTA (UMMA N), a multiple of 16 in [16, 256]
    int xtiles;      // x tiles per W tile
    uint32_t idesc;  // UMMA M = 128, N = bn, bf16 x bf16 -> fp32
};

// tcgen05.mma with A in tensor memory; called by every lane of a converged warp,
// issued by one elected lane.
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 consecutive 32-bit columns of this thread's lane from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) prefill_ab_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned, derived from the __shared__ array so that accesses stay shared-memory ones
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bars = sbase + SmemLayout::bar_off;
    const uint32_t bar_xfull = bars, bar_xempty = bars + 8 * kXStages;
    const uint32_t bar_afull = bars + 16 * kXStages, bar_aempty = bar_afull + 8 * kAStages;
    const uint32_t bar_wfull = bar_aempty + 8 * kAStages, bar_wempty = bar_wfull + 16;
    const uint32_t bar_acc = bar_wempty + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout::tmem_slot_off);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wt = static_cast<int>(blockIdx.x) / p.xtiles;  // x tile fastest in launch order
    const int xt = static_cast<int>(blockIdx.x) % p.xtiles;
    const int n0 = wt * kRowsW, m0 = xt * p.bn;
    const int nstages = p.K / kStageK;
    const int nchunks = (nstages + kChunkStages - 1) / kChunkStages;
    const int G = p.K / kGroup;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kXStages; ++s) {
            mbar_init(bar_xfull + 8 * s, 1);
            mbar_init(bar_xempty + 8 * s, 1);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(bar_afull + 8 * s, kDequantWarps);  // one arrival per dequantizing warp
            mbar_init(bar_aempty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_wfull + 8 * b, 1);
            mbar_init(bar_wempty + 8 * b, kDequantWarps);
        }
        mbar_init(bar_acc, 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ---- x tiles by TMA ----
        if (lane == 0) {
            for (int s = 0; s < nstages && ok; ++s) {
                const int slot = s % kXStages;
                ok = mbar_wait_bounded(bar_xempty + 8 * slot, ((s / kXStages) & 1) ^ 1);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_xfull + 8 * slot, p.bn * kStageK * 2);
                tma_load_2d(sbase + SmemLayout::x_off + slot * kXStageBytes, &p.tmap_x, s * kStageK, m0,
                            bar_xfull + 8 * slot);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue: the whole warp runs the loop, one elected lane issues ----
        const uint64_t xdesc0 = sw128_kmajor_desc(sbase + SmemLayout::x_off);
        for (int s = 0; s < nstages && ok; ++s) {
            const int xs = s % kXStages;
            const int g = s >> 1, as = g % kAStages;  // two x stages per group of W
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_xfull + 8 * xs, (s / kXStages) & 1) &&
                                             ((s & 1) || mbar_wait_bounded(bar_afull + 8 * as, (g / kAStages) & 1)));
            if (!ok) break;
            tc_fence_after();
            const uint64_t xd = desc_add(xdesc0, xs * kXStageBytes);
            const uint32_t ta = tmem + kACol0 + as * kACols + (s & 1) * (kStageK / 2);
#pragma unroll
            for (int kk = 0; kk < kStageK / 16; ++kk)
                umma_ts(tmem, ta + kk * 8, desc_add(xd, kk * 32), p.idesc, (s > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar_xempty + 8 * xs);  // the x stage is free once these MMAs are done
            if (s & 1) umma_commit(bar_aempty + 8 * as);  // and the group's A stage after its second x stage
        }
        if (ok) umma_commit(bar_acc);
    } else if (warp == 2) {
        // ---- packed words of the CTA's rows, four stages per copy, two buffers ----
        if (lane == 0) {
            for (int c = 0; c < nchunks && ok; ++c) {
                const int b = c & 1;
                ok = mbar_wait_bounded(bar_wempty + 8 * b, ((c >> 1) & 1) ^ 1);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_wfull + 8 * b, kWBufBytes);
                tma_load_2d(sbase + SmemLayout::w_off + b * kWBufBytes, &p.tmap_w, c * kChunkWords, n0,
                            bar_wfull + 8 * b);
            }
        }
    } else {
        // ---- dequantizing warps: row r of the tile (lane quarter warp % 4), half h of each group ----
        const int dw = warp - kFirstDequantWarp;  // 0 .. 7
        const int q = warp & 3;                   // a warp reaches tensor-memory lanes 32*(warp % 4) .. +31
        const int h = dw >> 2;                    // codes 64h .. 64h+63 of each group
        const int r = 32 * q + lane;
        const int n = n0 + r;
        const bool row_ok = n < p.N;
        const uint32_t tlane = tmem + (static_cast<uint32_t>(32 * q) << 16);
        const uint16_t *srow = p.scales + static_cast<int64_t>(row_ok ? n : 0) * G;
        uint32_t magic, sub;  // expansion constants, created once
        asm volatile("mov.b32 %0, %1;" : "=r"(magic) : "n"(0x43004300u));  // bf16x2 (128, 128)
        asm volatile("mov.b32 %0, %1;" : "=r"(sub) : "n"(0x43044304u));    // bf16x2 (132, 132)
        constexpr int kChunkGroups = kChunkStages / 2;
        uint32_t sc_cur[kChunkGroups] = {}, sc_next[kChunkGroups] = {};
        auto load_scales = [&](int c, uint32_t (&dst)[kChunkGroups]) {
#pragma unroll
            for (int i = 0; i < kChunkGroups; ++i) {
                const int g = kChunkGroups * c + i;
                const uint32_t hs = (row_ok && g < G) ? __ldg(srow + g) : 0u;
                dst[i] = hs | (hs << 16);
            }
        };
        load_scales(0, sc_cur);
        for (int c = 0; c < nchunks && ok; ++c) {
            load_scales(c + 1, sc_next);
            const int b = c & 1;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_wfull + 8 * b, (c >> 1) & 1));
            if (!ok) break;
            uint32_t words[kChunkWords];
            const uint4 *src = reinterpret_cast<const uint4 *>(smem + SmemLayout::w_off + b * kWBufBytes +
                                                                r * kChunkWords * 4);
#pragma unroll
            for (int i = 0; i < kChunkWords / 4; ++i) {
                const uint4 v = src[i];
                words[4 * i] = v.x;
                words[4 * i + 1] = v.y;
                words[4 * i + 2] = v.z;
                words[4 * i + 3] = v.w;
            }
            // The next copy into this buffer is an async-proxy write, and an arrive orders memory
            // operations, not the arrival of load results in registers: a store that depends on
            // every loaded register precedes the warp's arrival.
            uint32_t landed = 0;
#pragma unroll
            for (int i = 0; i < kChunkWords; i += 4) landed ^= words[i];
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(sbase + SmemLayout::sink_off +
                                                          4 * (threadIdx.x - kFirstDequantWarp * 32)),
                         "r"(landed)
                         : "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_wempty + 8 * b);
#pragma unroll
            for (int gi = 0; gi < kChunkGroups; ++gi) {
                const int g = c * kChunkGroups + gi;
                if (g >= G || !ok) break;
                uint32_t out[32];  // codes 64h .. 64h+63 of the group: words 12*gi + 6h .. +5
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t cur[3];
#pragma unroll
                    for (int i = 0; i < 3; ++i)
                        cur[i] = h ? words[kWordsPerGroup * gi + 6 + 3 * part + i]
                                   : words[kWordsPerGroup * gi + 3 * part + i];
                    uint32_t o16[16];
                    expand_half<0>(cur, sc_cur[gi], magic, sub, o16);
#pragma unroll
                    for (int i = 0; i < 16; ++i) out[16 * part + i] = o16[i];
                }
                const int as = g % kAStages;
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_aempty + 8 * as, ((g / kAStages) & 1) ^ 1));
                if (!ok) break;
                tc_fence_after();
                tmem_st32(tlane + kACol0 + as * kACols + 32 * h, out);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_afull + 8 * as);
            }
#pragma unroll
            for (int i = 0; i < kChunkGroups; ++i) sc_cur[i] = sc_next[i];
        }

        // ---- epilogue: D [lane = W row][column = x row] -> y[m][n]; half h takes columns 128h .. ----
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_acc, 0));
        tc_fence_after();
        if (ok) {
            const int c_end = min(p.bn, 128 * h + 128);
            for (int c0 = 128 * h; c0 < c_end; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tlane + c0, v);
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int m = m0 + c0 + i;
                        if (c0 + i < p.bn && m < p.M)
                            p.y[static_cast<int64_t>(m) * p.N + n] = f32_to_bf16_rn(__uint_as_float(v[i]));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

struct LaunchPlan {
    int bn, xtiles;
    dim3 grid;
};

// x rows per CTA: all of M up to 256 (a multiple of 16), else 256.
inline LaunchPlan plan(int M, int N) {
    LaunchPlan P;
    P.bn = M >= kMaxBN ? kMaxBN : (M + 15) / 16 * 16;
    P.xtiles = (M + P.bn - 1) / P.bn;
    const int wtiles = (N + kRowsW - 1) / kRowsW;
    P.grid = dim3(static_cast<unsigned>(wtiles * P.xtiles), 1, 1);
    return P;
}

}  // namespace prefill_ab
}  // namespace w3
