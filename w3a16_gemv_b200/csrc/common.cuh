// common.cuh -- device helpers shared by the kernels of libw3a16.so (sm_100a only).
//
// Inline PTX wrappers for the Blackwell features the kernels use: mbarriers,
// bulk (TMA engine) copies, thread-block-cluster distributed shared memory,
// warp-level bf16 MMA, and a bounded wait that records a timeout instead of
// hanging.
#pragma once

#include <cstdint>
#include <cuda.h>  // CUtensorMap (type only; the encoder is fetched at run time)
#include <cuda_runtime.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libw3a16 is written for sm_100a (B200) only"
#endif

namespace w3 {

constexpr int kGroup = 128;          // weights per bf16 scale (card: weight_scale_group_size)
constexpr int kWordsPerBlock = 3;    // 32 codes x 3 bits = 96 bits
constexpr int kWordsPerGroup = 12;   // 128 codes x 3 bits / 32
constexpr int kBytesPerGroup = 48;

// Device error flag bits (read and cleared by w3_check_device_error).
constexpr unsigned kDevErrTimeout = 1u;
// A bounded wait gives up after this many SM clock cycles (about 2 s at the
// B200's 1.965 GHz maximum; the SM cycle counter is cheap to read, unlike the
// global timer).
// (The test variant of the library shortens it to make a wait run out quickly.)
#ifndef W3_WAIT_LIMIT_CYCLES
#define W3_WAIT_LIMIT_CYCLES 4000000000ll
#endif
constexpr long long kWaitLimitCycles = W3_WAIT_LIMIT_CYCLES;

// Set by kernels, read and cleared by w3_check_device_error (the library is one
// translation unit, so this is its only definition).
__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_error(unsigned bits) { atomicOr(&g_device_error, bits); }

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier --------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async proxy and the cluster.
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the barrier to complete; give up after
// kWaitLimitCycles, record kDevErrTimeout and return false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitLimitCycles) {
            record_error(kDevErrTimeout);
            return false;
        }
    }
}

// ---- bulk copy global -> shared (TMA engine, non-tensor form) ----------------------
// dst, src 16-byte aligned, bytes a multiple of 16.  Completion is signalled on `bar`
// as transaction bytes.

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---- tiled tensor copy global -> shared (TMA) ------------------------------------------
// Box origin (x = innermost element index, y = row); x * element size must be a
// multiple of 16 bytes.  Out-of-range elements are filled with zeros and still
// count toward the transaction bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// ---- programmatic dependent launch ---------------------------------------------------
// A kernel launched with programmatic stream serialization may start while the
// previous kernel in the stream is still running.  It signals its own dependents
// early (pdl_trigger) and waits for its predecessor's completion and memory
// (pdl_wait) before it reads anything the predecessor may write (x) or writes
// anything it may read (y, scratch).  Both are no-ops for a normal launch.

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---- thread-block clusters ---------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_dsmem_f4(uint32_t addr, const float4 &v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// ---- bit manipulation ----------------------------------------------------------------

// (a & MASK) | c in exactly one LOP3: the mask is the instruction's immediate
// and c stays in a register.  (Written as C, the two constants would not both
// fit a single LOP3 and the compiler splits it in two.)
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "r"(c));
    return d;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// fp32 -> bf16 bits, round to nearest even (NaN kept quiet).
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
    uint16_t r;
    asm("{ .reg .b16 t; cvt.rn.bf16.f32 t, %1; mov.b16 %0, t; }" : "=h"(r) : "f"(f));
    return r;
}

// ---- warp-level tensor-core product ------------------------------------------------------
// D = A (16x16 bf16, row) * B (16x8 bf16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_m16n8k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                  uint32_t a3, uint32_t b0, uint32_t b1, const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

}  // namespace w3
