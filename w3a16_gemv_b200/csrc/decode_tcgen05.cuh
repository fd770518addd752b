// decode_tcgen05.cuh -- y = x * W^T for M <= 16 on the 5th-generation tensor
// cores, W in the exact-width uint3 / group-128 / bf16-scale format of the GSQ
// model card ("Storage layout" section), never materialised in memory.
//
// The roles of the operands are swapped with respect to a GEMM over the batch:
// the weights are the MMA's M dimension (128 rows per CTA) and the batch is
// its N dimension (16 columns, rows of x beyond M read as zeros).
//
//  * Loads: one warp issues, per stage of 3 groups, one tiled TMA copy of the
//    packed words of the CTA's 128 rows ([128 rows][36 words]) and six copies
//    of x ([16 rows][64 k], 128-byte swizzle, the UMMA B-operand layout).
//  * Row warps (4 x 32 threads, one weight row per thread): for each group the
//    thread reads its row's 12 words, expands the 128 codes in natural k order
//    to the exact levels q = c - 4 in bf16 (12 bits of two code pairs times
//    0x2001 put each pair's second code 13 bits above its first; one LOP3 per
//    pair into the mantissa of bf16 128.0, then a bf16x2 subtract of 132), and
//    writes the 64 bf16x2 words into its tensor-memory lane with one
//    tcgen05.st -- the A operand, double-buffered.
//  * One thread issues 8 tcgen05.mma (A from tensor memory, B = x from shared
//    memory, fp32 accumulation in tensor memory) per group into a fresh
//    per-group accumulator of 16 columns.
//  * The row threads read each group's 16 results back (tcgen05.ld) and add
//    s[n,g] * D to fp32 registers: the group scale is applied in fp32 and
//    nothing is rounded before the final bf16 store.
#pragma once

#include "common.cuh"
#include "prefill_gemm.cuh"

namespace w3 {
namespace decode_tc {

using prefill::fence_async_smem;
using prefill::mbar_arrive;
using prefill::sw128_kmajor_desc;
using prefill::tc_fence_after;
using prefill::tc_fence_before;
using prefill::umma_commit;

constexpr int kRows = 128;             // weight rows per CTA = UMMA M
constexpr int kBatch = 16;             // UMMA N: batch rows (x rows >= M are zero)
constexpr int kStageGroups = 3;
constexpr int kStages = 3;
constexpr int kPitch = kStageGroups * kWordsPerGroup;       // 36 words per row and stage
constexpr int kPackedBytes = kRows * kPitch * 4;            // 18432
constexpr int kXBox = kBatch * 64 * 2;                      // 2 KB: [16 rows][64 k] bf16
constexpr int kXBytes = kStageGroups * 2 * kXBox;           // 12 KB per stage
constexpr int kABuffers = 2, kDBuffers = 2;
constexpr int kAColsPerGroup = kGroup / 2;                  // 64 columns: two bf16 per column
constexpr int kTmemCols = 256;
constexpr int kThreads = 6 * 32;                            // TMA warp, MMA warp, 4 row warps
static_assert(kPackedBytes % 1024 == 0 && kXBytes % 1024 == 0, "stage buffers keep 1024-byte alignment");

struct SmemLayout {
    static constexpr int x_off = 0;                                    // [kStages][kXBytes], 1024-aligned
    static constexpr int packed_off = x_off + kStages * kXBytes;       // [kStages][kPackedBytes]
    static constexpr int bar_off = packed_off + kStages * kPackedBytes;
    // stage_full, stage_empty [kStages]; a_full, a_free [kABuffers]; d_full, d_free [kDBuffers]
    static constexpr int nbars = 2 * kStages + 2 * kABuffers + 2 * kDBuffers;
    static constexpr int tmem_slot_off = bar_off + nbars * 8;
    static constexpr int total = tmem_slot_off + 16 + 1024;
};

struct Params {
    CUtensorMap tmap_w;  // packed [N][3K/32] u32, box [128 rows][36 words]
    CUtensorMap tmap_x;  // x [M][K] bf16, box [16 rows][64 k], 128-byte swizzle
    const uint16_t *scales;
    uint16_t *y;
    int M, N, K;
    uint32_t idesc;      // UMMA M=128, N=16, bf16 x bf16 -> f32
};

__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 64 consecutive 32-bit columns of this thread's TMEM lane from registers.
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&v)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,"
        "%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]), "r"(v[32]), "r"(v[33]), "r"(v[34]), "r"(v[35]),
        "r"(v[36]), "r"(v[37]), "r"(v[38]), "r"(v[39]), "r"(v[40]), "r"(v[41]), "r"(v[42]), "r"(v[43]), "r"(v[44]),
        "r"(v[45]), "r"(v[46]), "r"(v[47]), "r"(v[48]), "r"(v[49]), "r"(v[50]), "r"(v[51]), "r"(v[52]), "r"(v[53]),
        "r"(v[54]), "r"(v[55]), "r"(v[56]), "r"(v[57]), "r"(v[58]), "r"(v[59]), "r"(v[60]), "r"(v[61]), "r"(v[62]),
        "r"(v[63])
        : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Bits [12q, 12q+12) of a group's 384-bit stream w[0..11]: codes 4q..4q+3.
template <int Q>
__device__ __forceinline__ uint32_t quad12(const uint32_t (&w)[12]) {
    constexpr int b = 12 * Q, i = b / 32, s = b % 32;
    if constexpr (s + 12 <= 32) return (w[i] >> s) & 0xFFFu;
    else return __funnelshift_r(w[i], w[i + 1], s) & 0xFFFu;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t v, uint32_t sub) {
    uint32_t q;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(v), "r"(sub));
    return q;
}

// The group's 128 codes as 64 bf16x2 words of exact levels q = c - 4, natural k order.
template <int Q>
__device__ __forceinline__ void expand_levels(const uint32_t (&w)[12], uint32_t (&out)[64]) {
    if constexpr (Q < 32) {
        constexpr uint32_t kMagic2 = 0x43004300u;  // bf16x2 (128, 128)
        constexpr uint32_t kSub = 0x43044304u;     // bf16x2 (132, 132)
        const uint32_t x = quad12<Q>(w) * 0x2001u;
        out[2 * Q] = bf16x2_sub(and_or<0x00070007u>(x, kMagic2), kSub);
        out[2 * Q + 1] = bf16x2_sub(and_or<0x00070007u>(x >> 6, kMagic2), kSub);
        expand_levels<Q + 1>(w, out);
    }
}

__global__ void __launch_bounds__(kThreads, 2) decode_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t x_base = sbase + SmemLayout::x_off;
    const uint32_t w_base = sbase + SmemLayout::packed_off;
    const uint32_t bars = sbase + SmemLayout::bar_off;
    const uint32_t stage_full = bars, stage_empty = bars + 8 * kStages;
    const uint32_t a_full = bars + 16 * kStages, a_free = a_full + 8 * kABuffers;
    const uint32_t d_full = a_free + 8 * kABuffers, d_free = d_full + 8 * kDBuffers;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout::tmem_slot_off);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kRows;
    const int G = p.K / kGroup;
    const int nstages = (G + kStageGroups - 1) / kStageGroups;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(stage_full + 8 * s, 1);
            mbar_init(stage_empty + 8 * s, kRows + 1);  // row threads read the words, the MMAs read x
        }
        for (int b = 0; b < kABuffers; ++b) {
            mbar_init(a_full + 8 * b, kRows);
            mbar_init(a_free + 8 * b, 1);
        }
        for (int b = 0; b < kDBuffers; ++b) {
            mbar_init(d_full + 8 * b, 1);
            mbar_init(d_free + 8 * b, kRows);
        }
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
    const uint32_t tmem_a = tmem;                                   // [kABuffers][64 columns]
    const uint32_t tmem_d = tmem + kABuffers * kAColsPerGroup;      // [kDBuffers][16 columns]
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {  // ---- loads ----
            for (int s = 0; s < nstages && ok; ++s) {
                const int slot = s % kStages;
                ok = mbar_wait_bounded(stage_empty + 8 * slot, ((s / kStages) & 1) ^ 1);
                if (!ok) break;
                const uint32_t bar = stage_full + 8 * slot;
                mbar_arrive_expect_tx(bar, kPackedBytes + kXBytes);
                tma_load_2d(w_base + slot * kPackedBytes, &p.tmap_w, s * kPitch, n0, bar);
                const uint32_t xs = x_base + slot * kXBytes;
#pragma unroll
                for (int h = 0; h < 2 * kStageGroups; ++h)
                    tma_load_2d(xs + h * kXBox, &p.tmap_x, (s * kStageGroups * 2 + h) * 64, 0, bar);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ---- MMA issue ----
            for (int j = 0; j < G && ok; ++j) {
                const int s = j / kStageGroups, gi = j % kStageGroups, slot = s % kStages;
                const int ab = j % kABuffers, db = j % kDBuffers;
                if (gi == 0) ok = mbar_wait_bounded(stage_full + 8 * slot, (s / kStages) & 1);
                ok = ok && mbar_wait_bounded(a_full + 8 * ab, (j / kABuffers) & 1) &&
                     mbar_wait_bounded(d_free + 8 * db, ((j / kDBuffers) & 1) ^ 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t xg = x_base + slot * kXBytes + gi * 2 * kXBox;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tmem_d + db * kBatch, tmem_a + ab * kAColsPerGroup + kk * 8,
                            sw128_kmajor_desc(xg + (kk / 4) * kXBox + (kk % 4) * 32), p.idesc, kk > 0 ? 1u : 0u);
                umma_commit(a_free + 8 * ab);
                umma_commit(d_full + 8 * db);
                if (gi == kStageGroups - 1 || j == G - 1) umma_commit(stage_empty + 8 * slot);
            }
        }
    } else {
        // ---- row warps: one weight row per thread ----
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;
        const int n = n0 + r;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint16_t *srow = p.scales + static_cast<int64_t>(min(n, p.N - 1)) * G;
        float acc[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) acc[b] = 0.f;
        float s_prev = 0.f;

        // fold group j's result (tensor-memory buffer j % kDBuffers) into acc
        auto readback = [&](int j, float sg) {
            const int db = j % kDBuffers;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(d_full + 8 * db, (j / kDBuffers) & 1) && ok);
            tc_fence_after();
            uint32_t v[kBatch];
            tmem_ld16(tmem_d + db * kBatch + lane_off, v);
            tc_fence_before();
            mbar_arrive(d_free + 8 * db);
#pragma unroll
            for (int b = 0; b < kBatch; ++b) acc[b] = fmaf(sg, __uint_as_float(v[b]), acc[b]);
        };

        for (int j = 0; j < G && ok; ++j) {
            const int s = j / kStageGroups, gi = j % kStageGroups, slot = s % kStages;
            const int ab = j % kABuffers;
            const float sg = bf16_bits_to_f32(__ldg(srow + j));
            if (gi == 0) ok = __all_sync(0xffffffffu, mbar_wait_bounded(stage_full + 8 * slot, (s / kStages) & 1));
            if (!ok) break;
            uint32_t w[12];
            const uint4 *src = reinterpret_cast<const uint4 *>(smem + SmemLayout::packed_off + slot * kPackedBytes +
                                                               r * kPitch * 4 + gi * kBytesPerGroup);
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const uint4 q = src[i];
                w[4 * i] = q.x;
                w[4 * i + 1] = q.y;
                w[4 * i + 2] = q.z;
                w[4 * i + 3] = q.w;
            }
            if (gi == kStageGroups - 1 || j == G - 1) mbar_arrive(stage_empty + 8 * slot);
            uint32_t out[64];
            expand_levels<0>(w, out);
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(a_free + 8 * ab, ((j / kABuffers) & 1) ^ 1));
            if (!ok) break;
            tc_fence_after();
            tmem_st64(tmem_a + ab * kAColsPerGroup + lane_off, out);
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            mbar_arrive(a_full + 8 * ab);
            if (j > 0) readback(j - 1, s_prev);
            s_prev = sg;
        }
        if (ok && G > 0) readback(G - 1, s_prev);
        if (ok && n < p.N) {
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
                if (b < p.M) p.y[static_cast<int64_t>(b) * p.N + n] = f32_to_bf16_rn(acc[b]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace decode_tc
}  // namespace w3
