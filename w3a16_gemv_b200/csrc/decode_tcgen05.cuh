// decode_tcgen05.cuh -- y = x * W^T for 17 <= M <= 32 on the 5th-generation tensor
// cores, W in the exact-width uint3 / group-128 / bf16-scale format of the GSQ
// model card ("Storage layout" section), never materialised in memory.
//
// The roles of the operands are swapped with respect to a GEMM over the batch:
// the weights are the MMA's M dimension (two 128-row tiles per CTA) and the
// batch is its N dimension (W3_TC_BATCH columns; rows of x beyond M read as zeros and
// their columns of the result are never stored).  The unpack of a weight is
// done once whatever M is, and the tensor cores do all of the multiply-adds.
//
//  * Work: the (256-row tile, group) units of the matrix are split into equal
//    contiguous ranges, one per CTA and one CTA per SM (stream-K).  A range
//    covers the end of one tile, whole tiles and the start of another; a tile
//    that several CTAs share is finished by a small second kernel that adds
//    their fp32 partial sums in CTA order, so the result does not depend on
//    timing.
//  * Loads (one warp): per stage of up to 3 groups, one tiled TMA copy of the
//    packed words of the CTA's 256 rows ([256 rows][36 words], or one
//    [256 rows][12 words] copy per group) and two copies of x per group
//    ([W3_TC_BATCH rows][64 k], 128-byte swizzle: the UMMA B operand).  The same
//    warp then permutes each 32-k block of x in place into the order of the
//    unpack below (byte permutes, no arithmetic).  A second warp copies the
//    stage's group scales (256 rows x up to 3) into a shared-memory ring, so
//    no row thread ever waits on a global load.
//  * Row warps (8 x 32 threads, one weight row per thread): a 32-code block
//    (3 words) becomes 16 bf16x2 words with 16 LOP3s and 9 shifts -- the same
//    pair schedule as the mma.sync decode: each LOP3 drops two codes into the
//    mantissa of bf16 128.0 at bit offsets e_lo, e_hi, the exact value
//    128 + c*2^e -- and one bf16x2 FMA per pair, v*2^-e - (128*2^-e + 4),
//    turns each into the exact level q = c - 4 (the ten FMA constants are
//    pinned in registers).  The group's 64 words go to the thread's
//    tensor-memory lane (two tcgen05.st): the A operand.
//  * One warp per tile, on different SM sub-partitions, issues 8 tcgen05.mma
//    per group from an elected lane (A from tensor memory, B = permuted x from
//    shared memory) into a fresh per-group fp32 accumulator of W3_TC_BATCH columns (four
//    buffers per tile).  The issue of these short MMAs shares its sub-partition
//    with two row warps and is what paces the kernel, hence one warp per tile.
//  * The row threads read each group's results back two groups later
//    (tcgen05.ld) and add s[n,g] * D to fp32 registers: the group scale is
//    applied in fp32 and nothing is rounded before the bf16 store.
// The file is compiled in its own namespace: W3_TC_NS names the instance and
// W3_TC_BATCH is its UMMA N (the library builds decode_tc32, 32 columns, for
// batches of 17..32 rows; up to 16 rows the mma.sync decodes are faster).
#ifndef W3_TC_NS
#define W3_TC_NS decode_tc32
#endif
#ifndef W3_TC_BATCH
#define W3_TC_BATCH 32
#endif

#include "common.cuh"
#include "decode_gemv.cuh"
#include "prefill_gemm.cuh"

namespace w3 {
namespace W3_TC_NS {

using decode::pair_spec;
using prefill::desc_add;
using prefill::fence_async_smem;
using prefill::mbar_arrive;
using prefill::sw128_kmajor_desc;
using prefill::tc_fence_after;
using prefill::tc_fence_before;
using prefill::umma_commit;

constexpr int kTileRows = 128;                    // UMMA M: one tensor-memory lane per row
constexpr int kTiles = 2;                         // row tiles per CTA, sharing x
constexpr int kRows = kTiles * kTileRows;         // 256 rows per CTA (one TMA box)
constexpr int kBatch = W3_TC_BATCH;               // UMMA N
static_assert(kBatch == 16 || kBatch == 32, "batch widths 16 and 32");
constexpr int kStageGroups = 3;
// One resident CTA per SM: it takes the shared and tensor memory budgets below.
constexpr int kCtasPerSm = 1;
constexpr int kStages = kBatch == 32 ? 3 : 4;
constexpr int kPitch3 = kStageGroups * kWordsPerGroup;        // 36 words: rows of a 3-group box
constexpr int kPitch1 = kWordsPerGroup;                       // 12 words: rows of a 1-group box
constexpr int kBox1Bytes = kRows * kPitch1 * 4;               // 12 KB
constexpr int kXBox = kBatch * 64 * 2;                        // 2 or 4 KB: [batch rows][64 k] bf16
constexpr int kXGroupBytes = 2 * kXBox;                       // 4 KB
constexpr int kXBytes = kStageGroups * kXGroupBytes;          // 12 KB
constexpr int kStageBytes = kXBytes + kStageGroups * kBox1Bytes;  // 48 KB
constexpr int kABuf = kBatch == 32 ? 2 : 3;                   // A buffers (one group each) per tile
constexpr int kDBuf = 4;                                      // accumulators per tile
constexpr int kLag = 2;                                       // groups between MMA and read-back
constexpr int kACols = 64;                                    // 128 codes, two bf16 per column
constexpr int kDCol0 = kABuf * kACols;                        // 192
constexpr int kTileCols = kDCol0 + kDBuf * kBatch;            // 256 columns per tile
constexpr int kTmemCols = kTiles * kTileCols;                 // 512 or 256 (two CTAs per SM)
static_assert(kTmemCols * kCtasPerSm <= 512, "tensor memory per SM");
constexpr int kRowWarps = kTiles * 4;
constexpr int kScaleWarp = 2 + kRowWarps;                     // warp 10
constexpr int kMmaWarp1 = 3 + kRowWarps;                      // warp 11: the MMAs of tile 1 (warp 1: tile 0)
constexpr int kThreads = (4 + kRowWarps) * 32;                // load, MMA x 2, row warps, scale warp
constexpr int kScaleSlotBytes = kStageGroups * kRows * 2;     // [3 groups][256 rows] bf16

constexpr int kMinUnitsPerCta = 6;  // (tile, group) units per CTA at least
static_assert(kXGroupBytes % 1024 == 0 && kXBytes % 1024 == 0 && kStageBytes % 1024 == 0,
              "swizzled x boxes need 1024-byte alignment");
static_assert(kBox1Bytes % 128 == 0, "tiled TMA destinations need 128-byte alignment");
static_assert(kStageGroups * kBox1Bytes == kRows * kPitch3 * 4, "a 3-group box fills the same bytes");
// The row threads read group j - kDBuf back (iteration j - kDBuf + kLag) before they
// hand over the A operand of group j, so "A of group j is full" also means "the
// accumulator of group j is free" and the MMA side needs no separate barrier.
static_assert(kDBuf >= kLag + 1, "read-back must finish before the accumulator is reused");

struct SmemLayout {
    static constexpr int stage_off = 0;  // [kStages]{x: [3][2 boxes], packed}
    static constexpr int scale_off = stage_off + kStages * kStageBytes;  // [kStages][3][256] bf16
    static constexpr int bar_off = scale_off + kStages * kScaleSlotBytes;
    // full, empty, bready [kStages]; a_full [kTiles][kABuf]; done [kTiles][kDBuf] (the MMAs of a group and tile)
    static constexpr int nbars = 3 * kStages + kTiles * kABuf + kTiles * kDBuf;
    static constexpr int tmem_slot_off = bar_off + nbars * 8;
    static constexpr int total = tmem_slot_off + 16 + 1024;  // + slack for 1024-byte alignment
};
static_assert(SmemLayout::total <= 227 * 1024, "shared memory per CTA");

struct Params {
    CUtensorMap tmap_w3;  // packed [N][3K/32] u32, box [256 rows][36 words] (valid when has_w3)
    CUtensorMap tmap_w1;  // packed, box [256 rows][12 words]
    CUtensorMap tmap_x;   // x [M][K] bf16, box [16 rows][64 k], 128-byte swizzle
    const uint16_t *scales;
    uint16_t *y;
    float *partial;       // [P][2][16][256] fp32 partial sums of shared tiles
    int M, N, K;
    int G;                // groups per row
    int P;                // CTAs
    int has_w3;
    int64_t U;            // units: 256-row tiles x groups
    uint32_t idesc;       // UMMA M=128, N=16, bf16 x bf16 -> f32
};

struct FixupParams {
    const float *partial;
    uint16_t *y;
    int M, N, G, P;
    int64_t U;
};

// First unit of CTA c: the ranges [unit_begin(c), unit_begin(c + 1)) tile the units.
__host__ __device__ inline int64_t unit_begin(int c, int64_t U, int P) { return static_cast<int64_t>(c) * U / P; }

// A tile that several CTAs' ranges share is left as fp32 partial sums, two slots per CTA: slot 0
// holds the first tile of CTA c's range, slot 1 its last (a range is contiguous, so no other
// tile of it can be shared).
__host__ __device__ inline int partial_slot(int c, int64_t t, int64_t U, int P, int G) {
    return unit_begin(c, U, P) / G == t ? 0 : 1;
}

// The shared tile that fix-up block b finishes, or -1: the tile that the boundary
// unit_begin(b + 1) cuts, unless that boundary is a tile boundary or an earlier boundary cuts
// the same tile (an earlier block finishes it then).
__host__ __device__ inline int64_t fixup_tile(int b, int64_t U, int P, int G) {
    const int64_t u = unit_begin(b + 1, U, P);
    const int64_t t0 = (u / G) * G;
    if (u == t0 || unit_begin(b, U, P) > t0) return -1;
    return u / G;
}

// Whether CTA c holds a part of tile t, for c at or after the block that finishes t: the CTAs
// b, b + 1, ... up to the first one whose range starts after the tile.
__host__ __device__ inline bool holds_part(int c, int64_t t, int64_t U, int P, int G) {
    return c < P && unit_begin(c, U, P) < (t + 1) * G;
}

// ---- compile-time constants of the pair schedule ----------------------------------

// bf16x2 (2^-e_lo, 2^-e_hi) for pair i: the scaling of x' in the pair's two slots.
__host__ __device__ constexpr uint32_t pair_mul(int i) {
    return static_cast<uint32_t>((127 - pair_spec(i).elo) << 7) | (static_cast<uint32_t>(127 - pair_spec(i).ehi) << 23);
}
// bf16 bits of a positive integer v < 256 with at most 8 significant bits.
__host__ __device__ constexpr uint32_t bf16_of_int(int v) {
    int e = 0;
    while ((v >> (e + 1)) != 0) ++e;
    return static_cast<uint32_t>(((127 + e) << 7) | (((v - (1 << e)) << 7) >> e));
}
// bf16x2 (-(128*2^-e_lo + 4), -(128*2^-e_hi + 4)) for pair i.
__host__ __device__ constexpr uint32_t pair_add(int i) {
    return (0x8000u | bf16_of_int((128 >> pair_spec(i).elo) + 4)) |
           ((0x8000u | bf16_of_int((128 >> pair_spec(i).ehi) + 4)) << 16);
}
static_assert(bf16_of_int(132) == 0x4304u && bf16_of_int(12) == 0x4140u && bf16_of_int(68) == 0x4288u,
              "bf16 encoding of the level offsets");
// The (e_lo, e_hi) combinations of the pair schedule, and the combination of pair i.
constexpr int kOffsetKinds = 5;
__host__ __device__ constexpr int offset_kind(int elo, int ehi) {
    return elo == 4 && ehi == 0 ? 0 : elo == 1 && ehi == 3 ? 1 : elo == 4 && ehi == 3 ? 2 : elo == 1 && ehi == 0 ? 3 : 4;
}
__host__ __device__ constexpr int pair_kind(int i) { return offset_kind(pair_spec(i).elo, pair_spec(i).ehi); }
__host__ __device__ constexpr bool pair_kinds_complete() {
    for (int i = 0; i < 16; ++i) {
        const int k = pair_kind(i);
        const int elo = k == 0 ? 4 : k == 1 ? 1 : k == 2 ? 4 : k == 3 ? 1 : 2;
        const int ehi = k == 0 ? 0 : k == 1 ? 3 : k == 2 ? 3 : k == 3 ? 0 : 1;
        if (elo != pair_spec(i).elo || ehi != pair_spec(i).ehi) return false;
    }
    return true;
}
static_assert(pair_kinds_complete(), "every pair's offsets are one of the five kinds");

// The FMA constants of the five kinds, held in registers.  Written through
// opaque moves so that the compiler keeps them instead of re-creating them
// before every use.
struct LevelConsts {
    uint32_t mul[kOffsetKinds], add[kOffsetKinds];
    uint32_t magic = decode::pinned_magic();
    __device__ __forceinline__ LevelConsts() {
#pragma unroll
        for (int k = 0; k < kOffsetKinds; ++k) {
            const int elo = k == 0 ? 4 : k == 1 ? 1 : k == 2 ? 4 : k == 3 ? 1 : 2;
            const int ehi = k == 0 ? 0 : k == 1 ? 3 : k == 2 ? 3 : k == 3 ? 0 : 1;
            const uint32_t m = static_cast<uint32_t>((127 - elo) << 7) | (static_cast<uint32_t>(127 - ehi) << 23);
            const uint32_t a = (0x8000u | bf16_of_int((128 >> elo) + 4)) | ((0x8000u | bf16_of_int((128 >> ehi) + 4)) << 16);
            asm volatile("mov.b32 %0, %1;" : "=r"(mul[k]) : "r"(m));
            asm volatile("mov.b32 %0, %1;" : "=r"(add[k]) : "r"(a));
        }
    }
};
// __byte_perm selector taking element lo of word a and element hi of word b.
__host__ __device__ constexpr uint32_t pair_sel(int i) {
    const uint32_t b0 = 2u * (pair_spec(i).lo & 1), b2 = 4u + 2u * (pair_spec(i).hi & 1);
    return b0 | ((b0 + 1) << 4) | (b2 << 8) | ((b2 + 1) << 12);
}

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// tcgen05.mma with A in tensor memory, called by every lane of a converged
// warp and issued by one elected lane (see umma_bf16).  ACC: add to D.
template <bool ACC>
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, %4;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "n"(ACC ? 1 : 0)
        : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane from registers.
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

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// kBatch (16 or 32) consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld_batch(uint32_t taddr, uint32_t (&v)[kBatch]) {
#if W3_TC_BATCH == 16
    tmem_ld16(taddr, v);
#else
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#endif
}

// Half H of a group's 128 codes (blocks 2H, 2H+1; 6 of the 12 words) as 32
// bf16x2 words of exact levels in pair order: word 16*b + i holds codes
// (lo_i, hi_i) of block 2H + b.
template <int H>
__device__ __forceinline__ void half_levels(const uint32_t (&w)[kWordsPerGroup], const LevelConsts &lc,
                                            uint32_t (&a)[32]) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const int bb = 2 * H + b;
        uint32_t blk[16];
        decode::unpack_block(w[3 * bb], w[3 * bb + 1], w[3 * bb + 2], blk, lc.magic);
#pragma unroll
        for (int i = 0; i < 16; ++i) a[16 * b + i] = bf16x2_fma(blk[i], lc.mul[pair_kind(i)], lc.add[pair_kind(i)]);
    }
}

// Permute x of one stage in place: each 32-k block of each batch row is put in
// pair order (word i of the block = elements lo_i, hi_i).  The boxes are in the
// 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8), so a
// block's four chunks stay together.
__device__ __forceinline__ void permute_x(uint8_t *xs, int ns, int lane) {
    for (int jj = 0; jj < ns; ++jj) {
#pragma unroll
        for (int it = 0; it < kBatch / 8; ++it) {
            const int item = lane + 32 * it;  // kBatch rows x 4 blocks
            const int r = item % kBatch, bl = item / kBatch;
            uint8_t *row = xs + jj * kXGroupBytes + (bl >> 1) * kXBox + r * 128;
            const int h = bl & 1, sw = r & 7;
            uint32_t src[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 q = *reinterpret_cast<const uint4 *>(row + (((4 * h + c) ^ sw) << 4));
                src[4 * c] = q.x;
                src[4 * c + 1] = q.y;
                src[4 * c + 2] = q.z;
                src[4 * c + 3] = q.w;
            }
            uint32_t out[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                out[i] = __byte_perm(src[pair_spec(i).lo >> 1], src[pair_spec(i).hi >> 1], pair_sel(i));
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4 *>(row + (((4 * h + c) ^ sw) << 4)) =
                    make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
        }
    }
}

// Walks a CTA's unit range as segments (one per 256-row tile touched); every
// role walks the same segments and splits them into the same stages.
struct Walk {
    int64_t u, end;
    int G;
    __host__ __device__ Walk(int c, int64_t U, int P, int G_)
        : u(unit_begin(c, U, P)), end(unit_begin(c + 1, U, P)), G(G_) {}
    __device__ explicit Walk(const Params &p) : Walk(blockIdx.x, p.U, p.P, p.G) {}
    // next segment: tile t, first group g0, length len; false when done
    __host__ __device__ bool next(int64_t &t, int &g0, int &len) {
        if (u >= end) return false;
        t = u / G;
        g0 = static_cast<int>(u - t * G);
        const int64_t se = (t + 1) * G < end ? (t + 1) * G : end;
        len = static_cast<int>(se - u);
        u = se;
        return true;
    }
};

__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned, derived from the __shared__ array so that accesses stay shared-memory ones
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bars = sbase + SmemLayout::bar_off;
    const uint32_t bar_full = bars, bar_empty = bars + 8 * kStages, bar_bready = bars + 16 * kStages;
    const uint32_t bar_afull = bars + 24 * kStages;                // [kTiles][kABuf]
    const uint32_t bar_done = bar_afull + 8 * kTiles * kABuf;      // [kTiles][kDBuf]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout::tmem_slot_off);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // the partial-sum fix-up grid may start now; it waits for this grid to finish
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1 + 32);  // the TMA bytes and the 32 lanes of the scale warp
            mbar_init(bar_empty + 8 * s, kRows + kTiles);  // row threads read the words, each tile's MMAs read x
            mbar_init(bar_bready + 8 * s, 1);
        }
        for (int b = 0; b < kTiles * kABuf; ++b) mbar_init(bar_afull + 8 * b, kTileRows);
        for (int b = 0; b < kTiles * kDBuf; ++b) mbar_init(bar_done + 8 * b, 1);
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
    // x, y and the scratch may belong to the previous kernel in the stream
    pdl_wait();

    if (warp == 0) {
        // ---- loads, then the in-place permutation of x one stage behind ----
        Walk walk(p);
        int64_t t;
        int g0, len, stage = 0, prev_ns = 0;
        auto prep = [&](int st, int ns) {
            const int slot = st % kStages;
            ok = ok && __all_sync(0xffffffffu, mbar_wait_bounded(bar_full + 8 * slot, (st / kStages) & 1));
            if (!ok) return;
            permute_x(smem + SmemLayout::stage_off + slot * kStageBytes, ns, lane);
            fence_async_smem();  // generic writes -> read by the tensor cores (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_bready + 8 * slot);
        };
        while (ok && walk.next(t, g0, len)) {
            for (int gs = 0; gs < len && ok; gs += kStageGroups) {
                const int ns = min(kStageGroups, len - gs);
                const int slot = stage % kStages;
                if (lane == 0) {
                    ok = mbar_wait_bounded(bar_empty + 8 * slot, ((stage / kStages) & 1) ^ 1);
                    if (ok) {
                        const uint32_t bar = bar_full + 8 * slot;
                        const uint32_t st = sbase + SmemLayout::stage_off + slot * kStageBytes;
                        const int g = g0 + gs;
                        const int row0 = static_cast<int>(t * kRows);
                        mbar_arrive_expect_tx(bar, ns * (kXGroupBytes + kBox1Bytes));
                        for (int jj = 0; jj < ns; ++jj) {
                            tma_load_2d(st + jj * kXGroupBytes, &p.tmap_x, (g + jj) * kGroup, 0, bar);
                            tma_load_2d(st + jj * kXGroupBytes + kXBox, &p.tmap_x, (g + jj) * kGroup + 64, 0, bar);
                        }
                        if (ns == kStageGroups && p.has_w3) {
                            tma_load_2d(st + kXBytes, &p.tmap_w3, g * kWordsPerGroup, row0, bar);
                        } else {
                            for (int jj = 0; jj < ns; ++jj)
                                tma_load_2d(st + kXBytes + jj * kBox1Bytes, &p.tmap_w1, (g + jj) * kWordsPerGroup,
                                            row0, bar);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (stage > 0) prep(stage - 1, prev_ns);
                prev_ns = ns;
                ++stage;
            }
        }
        if (ok && stage > 0) prep(stage - 1, prev_ns);
    } else if (warp == 1 || warp == kMmaWarp1) {
        // ---- MMA issue, one warp per tile (on different SM sub-partitions): per group, 8 MMAs
        //      into a fresh accumulator; the whole warp runs the loop and one elected lane issues ----
        const int tile = warp == 1 ? 0 : 1;
        const uint32_t tt = tmem + tile * kTileCols;
        const uint32_t afull = bar_afull + 8 * tile * kABuf, done = bar_done + 8 * tile * kDBuf;
        const uint64_t xdesc0 = sw128_kmajor_desc(sbase + SmemLayout::stage_off);
        Walk walk(p);
        int64_t t;
        int g0, len, slot = 0, ab = 0, db = 0;
        uint32_t sph = 0, aph = 0;  // phases of the stage ring and of the A-buffer ring
        while (ok && walk.next(t, g0, len)) {
            for (int gs = 0; gs < len && ok; gs += kStageGroups) {
                const int ns = min(kStageGroups, len - gs);
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_bready + 8 * slot, sph));
                const uint64_t xd = desc_add(xdesc0, slot * kStageBytes);
                for (int jj = 0; jj < ns && ok; ++jj) {
                    ok = __all_sync(0xffffffffu, mbar_wait_bounded(afull + 8 * ab, aph));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t dcol = tt + kDCol0 + db * kBatch, acol = tt + ab * kACols;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t bd = desc_add(xd, jj * kXGroupBytes + (kk >> 2) * kXBox + (kk & 3) * 32);
                        if (kk == 0) umma_ts<false>(dcol, acol, bd, p.idesc);
                        else umma_ts<true>(dcol, acol + kk * 8, bd, p.idesc);
                    }
                    umma_commit(done + 8 * db);  // this tile: A read, D written
                    if (++ab == kABuf) {
                        ab = 0;
                        aph ^= 1u;
                    }
                    db = (db + 1) % kDBuf;
                }
                if (!ok) break;
                umma_commit(bar_empty + 8 * slot);
                if (++slot == kStages) {
                    slot = 0;
                    sph ^= 1u;
                }
            }
        }
    } else if (warp == kScaleWarp) {
        // ---- group scales of each stage into the shared-memory ring ----
        Walk walk(p);
        int64_t t;
        int g0, len, stage = 0;
        while (ok && walk.next(t, g0, len)) {
            for (int gs = 0; gs < len && ok; gs += kStageGroups) {
                const int ns = min(kStageGroups, len - gs);
                const int slot = stage % kStages;
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_empty + 8 * slot, ((stage / kStages) & 1) ^ 1));
                if (!ok) break;
                uint16_t *dst = reinterpret_cast<uint16_t *>(smem + SmemLayout::scale_off + slot * kScaleSlotBytes);
                uint16_t v[kRows / 32][kStageGroups];
#pragma unroll
                for (int q = 0; q < kRows / 32; ++q) {
                    const int64_t n = t * kRows + lane + 32 * q;
                    const uint16_t *src = p.scales + (n < p.N ? n : p.N - 1) * static_cast<int64_t>(p.G) + g0 + gs;
#pragma unroll
                    for (int jj = 0; jj < kStageGroups; ++jj) v[q][jj] = jj < ns ? __ldg(src + jj) : uint16_t(0);
                }
#pragma unroll
                for (int q = 0; q < kRows / 32; ++q)
#pragma unroll
                    for (int jj = 0; jj < kStageGroups; ++jj) dst[jj * kRows + lane + 32 * q] = v[q][jj];
                mbar_arrive(bar_full + 8 * slot);  // release: the stores above are visible to the waiters
                ++stage;
            }
        }
    } else {
        // ---- row warps: one weight row per thread ----
        const int tile = (warp - 2) >> 2;
        const int quarter = warp & 3;  // a warp reaches TMEM lanes 32*(warp % 4) .. +31
        const int r = tile * kTileRows + quarter * 32 + lane;
        const uint32_t tt = tmem + tile * kTileCols + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t afull = bar_afull + 8 * tile * kABuf, done = bar_done + 8 * tile * kDBuf;
        float acc[kBatch];
        float s0 = 0.f, s1 = 0.f;  // scales of the (at most kLag = 2) groups awaiting read-back
        static_assert(kLag == 2, "the read-back queue below holds two groups");

        const LevelConsts lc;
        auto readback = [&](int jr, float sg) {
            const int db = jr % kDBuf;
            ok = ok && __all_sync(0xffffffffu, mbar_wait_bounded(done + 8 * db, (jr / kDBuf) & 1));
            if (!ok) return;
            tc_fence_after();
            uint32_t v[kBatch];
            tmem_ld_batch(tt + kDCol0 + db * kBatch, v);
#pragma unroll
            for (int b = 0; b < kBatch; ++b) acc[b] = fmaf(sg, __uint_as_float(v[b]), acc[b]);
        };

        Walk walk(p);
        int64_t t;
        int g0, len, stage = 0, j = 0;
        while (ok && walk.next(t, g0, len)) {
#pragma unroll
            for (int b = 0; b < kBatch; ++b) acc[b] = 0.f;
            int pend = 0;
            const int64_t n = t * kRows + r;
            for (int gs = 0; gs < len && ok; gs += kStageGroups) {
                const int ns = min(kStageGroups, len - gs);
                const int slot = stage % kStages;
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_full + 8 * slot, (stage / kStages) & 1));
                if (!ok) break;
                const uint8_t *pk = smem + SmemLayout::stage_off + slot * kStageBytes + kXBytes;
                const uint16_t *sc = reinterpret_cast<const uint16_t *>(smem + SmemLayout::scale_off +
                                                                        slot * kScaleSlotBytes) + r;
                const bool box3 = ns == kStageGroups && p.has_w3;
                for (int jj = 0; jj < ns; ++jj, ++j) {
                    const float sg = bf16_bits_to_f32(sc[jj * kRows]);
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        box3 ? pk + r * (kPitch3 * 4) + jj * kBytesPerGroup : pk + jj * kBox1Bytes + r * kBytesPerGroup);
                    uint32_t w[kWordsPerGroup];
#pragma unroll
                    for (int i = 0; i < 3; ++i) {
                        const uint4 q = src[i];
                        w[4 * i] = q.x;
                        w[4 * i + 1] = q.y;
                        w[4 * i + 2] = q.z;
                        w[4 * i + 3] = q.w;
                    }
                    if (jj == ns - 1) mbar_arrive(bar_empty + 8 * slot);
                    // the group's levels, one half (blocks 0-1, then 2-3) at a time
                    uint32_t a[32];
                    half_levels<0>(w, lc, a);
                    const int ab = j % kABuf;
                    if (j >= kABuf) {  // the MMAs of group j - kABuf have read this A buffer
                        const int jp = j - kABuf;
                        ok = __all_sync(0xffffffffu, mbar_wait_bounded(done + 8 * (jp % kDBuf), (jp / kDBuf) & 1));
                        if (!ok) break;
                    }
                    tc_fence_after();
                    tmem_st32(tt + ab * kACols, a);
                    half_levels<1>(w, lc, a);
                    tmem_st32(tt + ab * kACols + 32, a);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    mbar_arrive(afull + 8 * ab);
                    if (pend == 2) {
                        readback(j - 2, s0);
                        s0 = s1;
                        pend = 1;
                    }
                    if (pend == 0) s0 = sg;
                    else s1 = sg;
                    ++pend;
                }
                ++stage;
            }
            if (pend >= 1) readback(j - pend, s0);
            if (pend == 2) readback(j - 1, s1);
            if (len == p.G) {  // the whole tile is this CTA's: store y
                if (n < p.N) {
#pragma unroll
                    for (int b = 0; b < kBatch; ++b)
                        if (b < p.M) p.y[static_cast<int64_t>(b) * p.N + n] = f32_to_bf16_rn(acc[b]);
                }
            } else {  // shared tile: fp32 partial sums for the fix-up kernel
                float *dst = p.partial +
                             (static_cast<int64_t>(blockIdx.x) * 2 + partial_slot(blockIdx.x, t, p.U, p.P, p.G)) *
                                 kBatch * kRows +
                             r;
#pragma unroll
                for (int b = 0; b < kBatch; ++b)
                    if (b < p.M) dst[b * kRows] = acc[b];
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

// Tiles shared by several CTAs: block i-1 handles the tile that unit_begin(i)
// falls inside (when it is the first such boundary of that tile) and adds the
// partial sums of the CTAs that cover it, in CTA order.
__global__ void __launch_bounds__(kRows) decode_tc_fixup_kernel(const __grid_constant__ FixupParams p) {
    pdl_wait();
    const int64_t t = fixup_tile(blockIdx.x, p.U, p.P, p.G);
    if (t < 0) return;
    const int r = threadIdx.x;
    const int64_t n = t * kRows + r;
    if (n >= p.N) return;
    float acc[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) acc[b] = 0.f;
    // contributors in rounds of 4 whose loads are all issued before the adds
    constexpr int kRound = 4;
    for (int c = blockIdx.x; c < p.P;) {
        const float *src[kRound];
        int cnt = 0;
        for (; cnt < kRound && holds_part(c, t, p.U, p.P, p.G); ++c)
            src[cnt++] = p.partial + (static_cast<int64_t>(c) * 2 + partial_slot(c, t, p.U, p.P, p.G)) * kBatch * kRows + r;
        float v[kRound][kBatch];
#pragma unroll
        for (int q = 0; q < kRound; ++q)
#pragma unroll
            for (int b = 0; b < kBatch; ++b) v[q][b] = (q < cnt && b < p.M) ? __ldcg(src[q] + b * kRows) : 0.f;
#pragma unroll
        for (int q = 0; q < kRound; ++q)
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
                if (q < cnt) acc[b] += v[q][b];
        if (cnt < kRound) break;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
        if (b < p.M) p.y[static_cast<int64_t>(b) * p.N + n] = f32_to_bf16_rn(acc[b]);
}

struct LaunchPlan {
    int P;              // CTAs (one per SM at most)
    int64_t U;          // units
    int64_t ws_floats;  // partial-sum workspace (0 when one CTA does everything)
};

inline LaunchPlan plan(int64_t N, int64_t K, int num_sms) {
    LaunchPlan L;
    const int64_t T = (N + kRows - 1) / kRows;
    L.U = T * (K / kGroup);
    int64_t P = L.U / kMinUnitsPerCta;
    if (P > static_cast<int64_t>(num_sms) * kCtasPerSm) P = static_cast<int64_t>(num_sms) * kCtasPerSm;
    if (P < 1) P = 1;
    L.P = static_cast<int>(P);
    L.ws_floats = L.P > 1 ? static_cast<int64_t>(L.P) * 2 * kBatch * kRows : 0;
    return L;
}

// What the host launcher needs of this instance.
struct Instance {
    static constexpr int batch = kBatch, rows = kRows, tile_rows = kTileRows, threads = kThreads;
    static constexpr int pitch1 = kPitch1, pitch3 = kPitch3, smem_bytes = SmemLayout::total;
    using ParamsT = Params;
    using FixupT = FixupParams;
    using PlanT = LaunchPlan;
    static PlanT make_plan(int64_t N, int64_t K, int sms) { return plan(N, K, sms); }
    static cudaError_t set_smem() {
        return cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemLayout::total);
    }
    static cudaError_t launch(const cudaLaunchConfig_t &cfg, const Params &prm) {
        return cudaLaunchKernelEx(&cfg, decode_tc_kernel, prm);
    }
    static cudaError_t launch_fixup(const cudaLaunchConfig_t &cfg, const FixupParams &fp) {
        return cudaLaunchKernelEx(&cfg, decode_tc_fixup_kernel, fp);
    }
};

}  // namespace W3_TC_NS
}  // namespace w3
