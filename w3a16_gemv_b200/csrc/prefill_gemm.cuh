// prefill_gemm.cuh -- y = x * W^T for batches M > 16 on the 5th-generation
// tensor cores (tcgen05), W in the exact-width uint3 / group-128 / bf16-scale
// format of the GSQ model card ("Storage layout" section).
//
// A prefill batch makes the product a real dense contraction (2*M*N*K flops
// over (3/8)*N*K bytes of weights), so it runs as a GEMM whose B operand is
// produced on the fly:
//
//  * CTA tile: 256 rows of x (two 128-row UMMA tiles) x BN rows of W (BN a
//    multiple of 32, at most 256, chosen per shape to fill the last wave),
//    over K in stages of 64.  The fp32 accumulators live in tensor memory:
//    2 x BN columns of the 512 the CTA allocates.
//  * A (x): one tiled TMA copy per 128-row tile and stage, 128-byte swizzle,
//    the canonical K-major layout the UMMA descriptors describe.
//  * Packed W: one producer warp copies the CTA's rows, 24 words (four stages)
//    per row and copy, into shared memory by TMA.
//  * B (W): 8 dequantizing warps, one thread per W row (kDequantWarps = 16,
//    two threads per row each expanding half of a stage's 64 codes, is built
//    too and was slower).  Codes are expanded in natural k order four at a
//    time: the 12 bits of two code pairs times 0x2001 place each pair's second
//    code 13 bits above its first, so one LOP3 (mask | bf16 128.0) per pair
//    gives (128 + c_k, 128 + c_k+1) exactly; a bf16x2 subtract of 132 gives the
//    levels q = c - 4, and a bf16x2 multiply by the group scale gives
//    bf16(q * s), rounded once.  The rows are stored into the stage's B buffer
//    in the 128-byte-swizzled K-major layout, then made visible to the tensor
//    cores' async proxy; one arrival per warp hands the stage over.
//  * One elected lane issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) for
//    both 128-row tiles (only the first when the batch tile holds <= 128 rows)
//    and commits each stage back to the producers.
//  * Launch order: the batch tile varies fastest, so the CTAs sharing a W tile
//    run side by side and its packed words come from DRAM once.
//  * Epilogue: the dequantizing warps read the accumulators with tcgen05.ld,
//    round to bf16 and store y.
// All waits are bounded; a timeout is recorded and the CTA winds down.
#pragma once

#include "common.cuh"

namespace w3 {
namespace prefill {

constexpr int kTileM = 256;          // rows of x per CTA (two UMMA M=128 tiles)
constexpr int kUmmaM = 128;
constexpr int kMaxTileN = 256;       // rows of W per CTA at most
constexpr int kStageK = 64;          // k per pipeline stage = one 128-byte swizzle atom of bf16
constexpr int kStages = 3;
constexpr int kDequantWarps = 8;     // 8: one thread per W row, 16: two (BN <= 256)
constexpr int kHalves = 16 / kDequantWarps;  // 32-code halves of a stage per thread
constexpr int kChunkStages = 4;      // stages per packed-word copy (an even number: whole groups)
constexpr int kChunkGroups = kChunkStages / 2;
constexpr int kThreads = (2 + kDequantWarps + 1) * 32;  // x TMA, MMA, dequant warps, packed-word TMA
constexpr int kTmemCols = 512;
constexpr int kABytes = kUmmaM * kStageK * 2;     // 16 KB per 128-row tile and stage
constexpr int kBBytes = kMaxTileN * kStageK * 2;  // 32 KB per stage (BN rows used)
constexpr int kStageWords = kStageK * 3 / 32;     // 6 packed words per row and stage

struct SmemLayout {
    // all operand buffers are 1024-byte aligned (the 128-byte swizzle period)
    static constexpr int a_off = 0;                                  // [kStages][2][kABytes]
    static constexpr int b_off = a_off + kStages * 2 * kABytes;      // [kStages][kBBytes]
    static constexpr int w_off = b_off + kStages * kBBytes;          // [BN rows][6 * kChunkStages words] packed
    static constexpr int sink_off = w_off + kMaxTileN * kChunkStages * 6 * 4;  // u32 per dequant thread: see the release below
    static constexpr int bar_off = sink_off + kDequantWarps * 32 * 4;  // full_a, full_b, empty [kStages], acc, w_full, w_empty
    static constexpr int tmem_slot_off = bar_off + (3 * kStages + 3) * 8;
    static constexpr int total = tmem_slot_off + 16 + 1024;          // + slack to align the base to 1024
};

struct Params {
    CUtensorMap tmap_x;  // x [M][K] bf16, box [128 rows][64 k], 128-byte swizzle
    CUtensorMap tmap_w;  // packed [N][3K/32] u32, box [BN rows][24 words]
    const uint16_t *scales;
    uint16_t *y;
    int M, N, K;
    int tile_n;      // BN, a multiple of 32
    uint32_t idesc;  // UMMA instruction descriptor for M=128, N=BN
};

// K-major operand tile with 128-byte rows, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address (16-byte units)
    d |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (unused for swizzled K-major)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride byte offset: next 8-row group
    d |= static_cast<uint64_t>(1) << 46;                  // descriptor version (Blackwell)
    d |= static_cast<uint64_t>(2) << 61;                  // layout: 128-byte swizzle
    return d;
}

// bf16 x bf16 -> fp32, both operands K-major, D in tensor memory.
__host__ __device__ constexpr uint32_t make_idesc(int m, int n) {
    return (1u << 4)       // D format: f32
           | (1u << 7)     // A format: bf16
           | (1u << 10)    // B format: bf16
           | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// The descriptor of the same tile `bytes` further on (the start address field
// counts 16-byte units and never carries out for shared-memory addresses).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// tcgen05.mma and tcgen05.commit are single-thread instructions.  These
// wrappers are called by every lane of a converged warp and issue from one
// lane chosen by elect.sync: with warp-uniform operands the issuing loop costs
// a few instructions per MMA (issued from one thread inside a branch it costs
// several times more and, at small N, limits the tensor pipe).
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t bf16x2_sub_mul(uint32_t v, uint32_t sub, uint32_t mul) {
    uint32_t q, r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(v), "r"(sub));  // exact: c - 4
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(q), "r"(mul));  // bf16(q * s), one rounding
    return r;
}

// Expand codes 4I .. 31 of a 96-bit half stage w[0..2] (32 codes) into bf16x2
// words out[2I ..] of bf16(q*s), natural k order.
template <int I>
__device__ __forceinline__ void expand_half(const uint32_t (&w)[3], uint32_t s2, uint32_t magic, uint32_t sub,
                                            uint32_t (&out)[16]) {
    if constexpr (I < 8) {
        constexpr int b = 12 * I, i = b / 32, sh = b % 32;
        uint32_t bits;
        if constexpr (sh + 12 <= 32) bits = (w[i] >> sh) & 0xFFFu;
        else bits = __funnelshift_r(w[i], w[i + 1], sh) & 0xFFFu;
        const uint32_t x = bits * 0x2001u;  // second code of each pair 13 bits above the first
        out[2 * I] = bf16x2_sub_mul(and_or<0x00070007u>(x, magic), sub, s2);
        out[2 * I + 1] = bf16x2_sub_mul(and_or<0x00070007u>(x >> 6, magic), sub, s2);
        expand_half<I + 1>(w, s2, magic, sub, out);
    }
}

__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned, derived from the __shared__ array so that accesses stay shared-memory ones
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(smem);
    const uint32_t a_base = sbase + SmemLayout::a_off;
    const uint32_t b_base = sbase + SmemLayout::b_off;
    const uint32_t bar_full_a = sbase + SmemLayout::bar_off;
    const uint32_t bar_full_b = bar_full_a + 8 * kStages;
    const uint32_t bar_empty = bar_full_b + 8 * kStages;
    const uint32_t bar_acc = bar_empty + 8 * kStages;
    const uint32_t bar_wfull = bar_acc + 8, bar_wempty = bar_acc + 16;
    constexpr int kChunkWords = kChunkStages * kStageWords;  // words per row and copy
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout::tmem_slot_off);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // CTAs that share a W tile are adjacent in launch order, so they run together and the
    // tile's packed words come from DRAM once and from L2 for the other batch tiles
    const int mtiles = (p.M + kTileM - 1) / kTileM;
    const int m0 = static_cast<int>(blockIdx.x % mtiles) * kTileM;
    const int n0 = static_cast<int>(blockIdx.x / mtiles) * p.tile_n;
    const int nstages = p.K / kStageK;
    const int G = p.K / kGroup;
    // a batch tile of at most 128 rows needs only the first UMMA tile (mid-sized batches)
    const bool two_tiles = m0 + kUmmaM < p.M;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full_a + 8 * s, 1);
            mbar_init(bar_full_b + 8 * s, kDequantWarps);  // one arrival per dequant warp
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_acc, 1);
        mbar_init(bar_wfull, 1);
        mbar_init(bar_wempty, kDequantWarps);
        mbar_init_fence();
    }
    if (warp == 1) {  // allocate the accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
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
        // ---- A producer: x tiles by TMA ----
        if (lane == 0) {
            for (int s = 0; s < nstages && ok; ++s) {
                const int slot = s % kStages;
                const uint32_t round = static_cast<uint32_t>(s / kStages);
                ok = mbar_wait_bounded(bar_empty + 8 * slot, (round & 1u) ^ 1u);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_full_a + 8 * slot, (two_tiles ? 2 : 1) * kABytes);
                const uint32_t dst = a_base + slot * 2 * kABytes;
                tma_load_2d(dst, &p.tmap_x, s * kStageK, m0, bar_full_a + 8 * slot);
                if (two_tiles) tma_load_2d(dst + kABytes, &p.tmap_x, s * kStageK, m0 + kUmmaM, bar_full_a + 8 * slot);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer: the whole warp runs the loop, one elected lane issues ----
        const uint64_t adesc0 = sw128_kmajor_desc(a_base), bdesc0 = sw128_kmajor_desc(b_base);
        const uint32_t d1 = tmem + static_cast<uint32_t>(p.tile_n);
        for (int s = 0; s < nstages && ok; ++s) {
            const int slot = s % kStages;
            const uint32_t par = static_cast<uint32_t>(s / kStages) & 1u;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_full_a + 8 * slot, par) &&
                                             mbar_wait_bounded(bar_full_b + 8 * slot, par));
            if (!ok) break;
            tc_fence_after();
            const uint64_t ad = desc_add(adesc0, slot * 2 * kABytes);
            const uint64_t bd0 = desc_add(bdesc0, slot * kBBytes);
#pragma unroll
            for (int kk = 0; kk < kStageK / 16; ++kk) {
                const uint64_t bd = desc_add(bd0, kk * 32);
                const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                umma_bf16(tmem, desc_add(ad, kk * 32), bd, p.idesc, acc);
                if (two_tiles) umma_bf16(d1, desc_add(ad, kABytes + kk * 32), bd, p.idesc, acc);
            }
            umma_commit(bar_empty + 8 * slot);  // frees the stage once these MMAs have read it
        }
        if (ok) umma_commit(bar_acc);  // all accumulation done
    } else if (warp == 2 + kDequantWarps) {
        // ---- packed words of the CTA's rows, four stages per TMA copy ----
        if (lane == 0) {
            const int nchunks = (nstages + kChunkStages - 1) / kChunkStages;
            for (int c = 0; c < nchunks && ok; ++c) {
                ok = mbar_wait_bounded(bar_wempty, (c & 1) ^ 1);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_wfull, p.tile_n * kChunkWords * 4);
                tma_load_2d(sbase + SmemLayout::w_off, &p.tmap_w, c * kChunkWords, n0, bar_wfull);
            }
        }
    } else {
        // ---- B producers: row r of the tile; with 16 warps, half dw/8 of each stage's 64 codes ----
        const int dw = warp - 2;             // 0 .. kDequantWarps-1
        const int hsel = dw >> 3;            // the half this thread expands when kHalves == 1
        const int r = (dw & 7) * 32 + lane;  // row of the tile
        const int n = n0 + r;
        const bool row_ok = (r < p.tile_n) && (n < p.N);
        const uint16_t *srow = p.scales + static_cast<int64_t>(row_ok ? n : 0) * G;
        const uint32_t *wsm = reinterpret_cast<const uint32_t *>(smem + SmemLayout::w_off);
        uint32_t magic, sub;  // expansion constants, created once (opaque: not rebuilt before each use)
        asm volatile("mov.b32 %0, %1;" : "=r"(magic) : "n"(0x43004300u));  // bf16x2 (128, 128)
        asm volatile("mov.b32 %0, %1;" : "=r"(sub) : "n"(0x43044304u));    // bf16x2 (132, 132)
        // the row's 24 words of a 4-stage chunk come from the shared-memory copy; the chunk's two
        // group scales are loaded one chunk ahead
        const int nchunks = (nstages + kChunkStages - 1) / kChunkStages;
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
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_wfull, c & 1));
            if (!ok) break;
            uint32_t words[kChunkWords];
            if (r < p.tile_n) {
                const uint4 *src = reinterpret_cast<const uint4 *>(wsm + r * kChunkWords);
#pragma unroll
                for (int i = 0; i < kChunkWords / 4; ++i) {
                    const uint4 q = src[i];
                    words[4 * i] = q.x;
                    words[4 * i + 1] = q.y;
                    words[4 * i + 2] = q.z;
                    words[4 * i + 3] = q.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < kChunkWords; ++i) words[i] = 0u;
            }
            // The next copy into the buffer is an async-proxy write, and an arrive orders memory
            // operations, not the arrival of load results in registers.  A store that depends on
            // every loaded register therefore precedes the warp's arrival: the buffer is released
            // only once every lane's loads have completed.
            uint32_t landed = 0;
#pragma unroll
            for (int i = 0; i < kChunkWords; i += 4) landed ^= words[i];
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(sbase + SmemLayout::sink_off + 4 * (threadIdx.x - 64)),
                         "r"(landed)
                         : "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_wempty);
#pragma unroll
            for (int u = 0; u < kChunkStages; ++u) {
                const int s = c * kChunkStages + u;
                if (s >= nstages || !ok) break;
                const uint32_t s2 = sc_cur[u >> 1];  // one scale per 128 codes = two stages
                uint32_t out[kHalves][16];
#pragma unroll
                for (int hh = 0; hh < kHalves; ++hh) {
                    uint32_t cur[3];  // half h of the stage: words 3h .. 3h+2
#pragma unroll
                    for (int i = 0; i < 3; ++i)
                        cur[i] = (kHalves == 2) ? words[kStageWords * u + 3 * hh + i]
                                                : (hsel ? words[kStageWords * u + 3 + i] : words[kStageWords * u + i]);
                    expand_half<0>(cur, s2, magic, sub, out[hh]);
                }
                const int slot = s % kStages;
                const uint32_t round = static_cast<uint32_t>(s / kStages);
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_empty + 8 * slot, (round & 1u) ^ 1u));
                if (!ok) break;
                if (r < p.tile_n) {
                    const uint32_t row = b_base + slot * kBBytes + r * 128;
#pragma unroll
                    for (int hh = 0; hh < kHalves; ++hh) {
                        const int h = (kHalves == 2) ? hh : hsel;
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const uint32_t dst = row + (((4 * h + jj) ^ (r & 7)) << 4);
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                                         "r"(out[hh][4 * jj]), "r"(out[hh][4 * jj + 1]), "r"(out[hh][4 * jj + 2]),
                                         "r"(out[hh][4 * jj + 3])
                                         : "memory");
                        }
                    }
                }
                fence_async_smem();
                __syncwarp();  // the warp's stores are ordered before lane 0's arrival
                if (lane == 0) mbar_arrive(bar_full_b + 8 * slot);
            }
#pragma unroll
            for (int i = 0; i < kChunkGroups; ++i) sc_cur[i] = sc_next[i];
        }

        // ---- epilogue: TMEM -> bf16 -> y; per TMEM lane quarter, kDequantWarps/4 warps share the tiles ----
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_acc, 0));
        tc_fence_after();
        if (ok) {
            const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
            const int tsub = (dw >> 2) & 1;  // accumulator tile
            const int ch = dw >> 3;          // with 16 warps: every other 32-column chunk
            const int m = m0 + tsub * kUmmaM + quarter * 32 + lane;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(tsub * p.tile_n);
            const int cols = (tsub == 0 || two_tiles) ? p.tile_n : 0;  // tile 1 holds nothing when unused
            for (int c0 = 32 * ch; c0 < cols; c0 += 32 * (kDequantWarps / 8)) {
                uint32_t v[32];
                tmem_ld32(tbase + c0, v);
                if (m < p.M) {
                    uint16_t *yrow = p.y + static_cast<int64_t>(m) * p.N;
                    const int nb = n0 + c0;
                    if (nb + 32 <= p.N && (p.N % 8) == 0) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = static_cast<uint32_t>(f32_to_bf16_rn(__uint_as_float(v[2 * i]))) |
                                    (static_cast<uint32_t>(f32_to_bf16_rn(__uint_as_float(v[2 * i + 1]))) << 16);
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + nb);
#pragma unroll
                        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    } else {
                        for (int i = 0; i < 32; ++i)
                            if (nb + i < p.N) yrow[nb + i] = f32_to_bf16_rn(__uint_as_float(v[i]));
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
    int tile_n;
    dim3 grid;
};

// BN: a multiple of 32 in [128, 256] that leaves the last wave fullest (a
// multiple of 32 so that the epilogue's 32-column TMEM reads never cross into
// the next tile's columns).
inline LaunchPlan plan(int M, int N, int num_sms) {
    LaunchPlan P;
    const int mt = (M + kTileM - 1) / kTileM;
    int best = kMaxTileN;
    double best_eff = -1.0;
    for (int bn = kMaxTileN; bn >= 128; bn -= 32) {
        const int tiles = mt * ((N + bn - 1) / bn);
        const int waves = (tiles + num_sms - 1) / num_sms;
        // useful work over scheduled work, counting padding of the last N tile
        const double eff = static_cast<double>(M) * N / (static_cast<double>(waves) * num_sms * kTileM * bn);
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = bn;
        }
    }
    if (N < 128) best = (N + 31) / 32 * 32;
    P.tile_n = best;
    P.grid = dim3(mt * ((N + best - 1) / best), 1, 1);  // batch tile fastest
    return P;
}

}  // namespace prefill
}  // namespace w3
