// api.cu -- the extern "C" entry points of libw3a16.so (declared in include/w3a16.h).
//
// Host side only: argument checks, per-device set-up, kernel selection and
// launch.  All arithmetic runs in the kernels included below (one translation
// unit, so the device error flag needs no relocatable device code).
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "../../include/w3a16.h"
#include "common.cuh"
#include "decode_gemv.cuh"
#include "decode_split.cuh"
#include "decode_streamk.cuh"
// the tensor-core decode for 17 <= M <= 32 (32 batch columns)
#define W3_TC_NS decode_tc32
#define W3_TC_BATCH 32
#include "decode_tcgen05.cuh"
#include "format_kernels.cuh"
#include "prefill_gemm.cuh"
#include "prefill_swab.cuh"

namespace w3 {
namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxElems = int64_t(1) << 40;
constexpr int64_t kMaxDim = int64_t(1) << 30;

struct DeviceState {
    std::once_flag once;
    w3_status status = W3_OK;
    int num_sms = 0;
    cudaMemPool_t pool = nullptr;  // stream-ordered scratch of w3a16_gemm (kept, never trimmed)
};
DeviceState g_dev[kMaxDevices];

// Once per device: check that it is an sm_100 part and raise the kernels'
// dynamic shared-memory limits.
w3_status device_setup(int *num_sms, cudaMemPool_t *pool = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W3_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return W3_ERR_UNSUPPORTED;
    DeviceState &st = g_dev[dev];
    std::call_once(st.once, [&] {
        int major = 0, minor = 0, sms = 0, optin = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
            st.status = W3_ERR_CUDA;
            return;
        }
        if (major != 10 || minor != 0) {
            st.status = W3_ERR_UNSUPPORTED;
            return;
        }
        st.num_sms = sms;
        const void *kernels[] = {
            reinterpret_cast<const void *>(decode::decode_kernel<1>),
            reinterpret_cast<const void *>(decode::decode_kernel<2>),
            reinterpret_cast<const void *>(decode::decode_kernel<4>),
            reinterpret_cast<const void *>(decode::decode_kernel<8>),
            reinterpret_cast<const void *>(decode::decode_kernel<16>),
        };
        const void *split_kernels[] = {
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<1, false>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<2, false>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<4, false>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<8, false>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<16, false>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<1, true>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<2, true>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<4, true>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<8, true>),
            reinterpret_cast<const void *>(dsplit::decode_split_kernel<16, true>),
        };
        for (const void *k : split_kernels) {
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess ||
                cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
                st.status = W3_ERR_CUDA;
                return;
            }
        }
        const void *sk_kernels[] = {
            reinterpret_cast<const void *>(decode_sk::decode_sk_kernel<1, false>),
            reinterpret_cast<const void *>(decode_sk::decode_sk_kernel<2, false>),
            reinterpret_cast<const void *>(decode_sk::decode_sk_kernel<4, false>),
            reinterpret_cast<const void *>(decode_sk::decode_sk_kernel<1, true>),
            reinterpret_cast<const void *>(decode_sk::decode_sk_kernel<2, true>),
            reinterpret_cast<const void *>(decode_sk::decode_sk_kernel<4, true>),
        };
        for (const void *k : sk_kernels) {
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess) {
                st.status = W3_ERR_CUDA;
                return;
            }
        }
        if (decode_tc32::Instance::set_smem() != cudaSuccess) {
            st.status = W3_ERR_CUDA;
            return;
        }
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        uint64_t keep = UINT64_MAX;
        if (cudaMemPoolCreate(&st.pool, &props) != cudaSuccess ||
            cudaMemPoolSetAttribute(st.pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
            st.status = W3_ERR_CUDA;
            return;
        }
        if (cudaFuncSetAttribute(prefill_ab::prefill_ab_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 prefill_ab::SmemLayout::total) != cudaSuccess) {
            st.status = W3_ERR_CUDA;
            return;
        }
        if (cudaFuncSetAttribute(prefill::prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 prefill::SmemLayout::total) != cudaSuccess) {
            st.status = W3_ERR_CUDA;
            return;
        }
        for (const void *k : kernels) {
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess) {
                st.status = W3_ERR_CUDA;
                return;
            }
        }
        st.status = W3_OK;
    });
    *num_sms = st.num_sms;
    if (pool) *pool = st.pool;
    return st.status;
}

// cuTensorMapEncodeTiled from the driver, fetched once through the runtime.
PFN_cuTensorMapEncodeTiled tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
    });
    return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Programmatic dependent launch: the kernel may start before the previous kernel in
// the stream ends; it waits for it (griddepcontrol.wait) before touching x, y or
// scratch.  Weights and scales are read before that wait, so a kernel that writes
// them must not precede the call with an early trigger of its own (this library's
// kernels that write weights -- pack, repack -- never trigger early).
void set_pdl(cudaLaunchAttribute &a) {
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
}

bool overlaps(const void *a, int64_t abytes, const void *b, int64_t bbytes) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

w3_status check_nk(int64_t N, int64_t K) {
    if (N < 1 || K < kGroup || K % kGroup != 0) return W3_ERR_SHAPE;
    if (N > kMaxDim || K > kMaxDim || N * K > kMaxElems) return W3_ERR_SHAPE;
    return W3_OK;
}

w3_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? W3_OK : W3_ERR_CUDA;
}

// A [rows][box_words] box over the packed matrix [N][3K/32] u32.
w3_status encode_packed_map(CUtensorMap *map, const int32_t *packed, int64_t N, int64_t words, uint32_t box_words,
                            uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
    if (!enc) return W3_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(words), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(words * 4)};
    cuuint32_t box[2] = {box_words, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<int32_t *>(packed), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? W3_OK
               : W3_ERR_CUDA;
}

// The stream-K decode on the row-major words (`packed`) or, when `native` is given, on the
// same words in the native block order.
w3_status launch_decode_sk(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int M,
                           int N, int K, int num_sms, cudaStream_t stream, const int32_t *native = nullptr) {
    const decode_sk::LaunchPlan P = decode_sk::plan(M, N, K, num_sms);
    decode_sk::Params prm;
    const int64_t words = static_cast<int64_t>(K) * 3 / 32;
    prm.native = reinterpret_cast<const uint32_t *>(native);
    if (!native) {
        if (w3_status s = encode_packed_map(&prm.tmap1, packed, N, words, decode_sk::kPitch1, decode_sk::kBlockRows))
            return s;
        prm.tmap3 = prm.tmap1;  // only used when a segment has 3 groups left, which needs K >= 384
        if (words >= decode_sk::kPitch3) {
            if (w3_status s =
                    encode_packed_map(&prm.tmap3, packed, N, words, decode_sk::kPitch3, decode_sk::kBlockRows))
                return s;
        }
    }
    prm.x = x;
    prm.scales = scales;
    prm.y = y;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.ctas = P.ctas;
    prm.depth = P.depth;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.ctas, 1, 1);
    cfg.blockDim = dim3(decode_sk::kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = P.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);  // overlaps the set-up with the previous kernel's tail
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (native) {
        switch (P.mt) {
            case 1: e = cudaLaunchKernelEx(&cfg, decode_sk::decode_sk_kernel<1, true>, prm); break;
            case 2: e = cudaLaunchKernelEx(&cfg, decode_sk::decode_sk_kernel<2, true>, prm); break;
            default: e = cudaLaunchKernelEx(&cfg, decode_sk::decode_sk_kernel<4, true>, prm); break;
        }
    } else {
        switch (P.mt) {
            case 1: e = cudaLaunchKernelEx(&cfg, decode_sk::decode_sk_kernel<1, false>, prm); break;
            case 2: e = cudaLaunchKernelEx(&cfg, decode_sk::decode_sk_kernel<2, false>, prm); break;
            default: e = cudaLaunchKernelEx(&cfg, decode_sk::decode_sk_kernel<4, false>, prm); break;
        }
    }
    return e == cudaSuccess ? W3_OK : W3_ERR_CUDA;
}

// Tensor-core decode (tcgen05, weights as the MMA's M dimension), M <= I::batch.
// Shared tiles are finished by the fix-up kernel, launched behind it with
// programmatic dependent launch; their fp32 partial sums live in `partial`
// (I::make_plan(...).ws_floats floats, unused when that is 0).  Returns
// W3_ERR_UNSUPPORTED, without launching, for shapes it does not take (N < 256).
template <class I>
w3_status launch_decode_tc(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int M,
                           int N, int K, const typename I::PlanT &P, float *partial, cudaStream_t stream) {
    if (N < I::rows || M > I::batch) return W3_ERR_UNSUPPORTED;
    typename I::ParamsT prm;
    const int64_t words = static_cast<int64_t>(K) * 3 / 32;
    if (encode_packed_map(&prm.tmap_w1, packed, N, words, I::pitch1, I::rows) != W3_OK) return W3_ERR_CUDA;
    prm.has_w3 = words >= I::pitch3;
    prm.tmap_w3 = prm.tmap_w1;
    if (prm.has_w3 && encode_packed_map(&prm.tmap_w3, packed, N, words, I::pitch3, I::rows) != W3_OK)
        return W3_ERR_CUDA;
    PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
    if (!enc) return W3_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(I::batch)};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&prm.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return W3_ERR_CUDA;
    prm.scales = scales;
    prm.y = y;
    prm.partial = partial;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.G = K / kGroup;
    prm.P = P.P;
    prm.U = P.U;
    prm.idesc = prefill::make_idesc(I::tile_rows, I::batch);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.P, 1, 1);
    cfg.blockDim = dim3(I::threads, 1, 1);
    cfg.dynamicSmemBytes = I::smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute mattr[1];
    set_pdl(mattr[0]);
    cfg.attrs = mattr;
    cfg.numAttrs = 1;
    if (I::launch(cfg, prm) != cudaSuccess) return W3_ERR_CUDA;
    if (P.P == 1) return W3_OK;
    typename I::FixupT fp;
    fp.partial = partial;
    fp.y = y;
    fp.M = M;
    fp.N = N;
    fp.G = prm.G;
    fp.P = P.P;
    fp.U = P.U;
    cudaLaunchConfig_t fcfg = {};
    fcfg.gridDim = dim3(P.P - 1, 1, 1);
    fcfg.blockDim = dim3(I::rows, 1, 1);
    fcfg.stream = stream;
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);
    fcfg.attrs = attr;
    fcfg.numAttrs = 1;
    return I::launch_fixup(fcfg, fp) == cudaSuccess ? W3_OK : W3_ERR_CUDA;
}

w3_status launch_prefill(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int M,
                         int N, int K, int num_sms, cudaStream_t stream) {
    const prefill::LaunchPlan P = prefill::plan(M, N, num_sms);
    prefill::Params prm;
    PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
    if (!enc) return W3_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {prefill::kStageK, prefill::kUmmaM};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&prm.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return W3_ERR_CUDA;
    // [BN rows][24 words] boxes over the packed matrix: four stages of the CTA's rows per copy
    if (encode_packed_map(&prm.tmap_w, packed, N, static_cast<int64_t>(K) * 3 / 32,
                          prefill::kChunkStages * prefill::kStageWords, static_cast<uint32_t>(P.tile_n)) != W3_OK)
        return W3_ERR_CUDA;
    prm.scales = scales;
    prm.y = y;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.tile_n = P.tile_n;
    prm.idesc = prefill::make_idesc(prefill::kUmmaM, P.tile_n);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = P.grid;
    cfg.blockDim = dim3(prefill::kThreads, 1, 1);
    cfg.dynamicSmemBytes = prefill::SmemLayout::total;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, prefill::prefill_kernel, prm) == cudaSuccess ? W3_OK : W3_ERR_CUDA;
}

// Which prefill kernel.  Both run one CTA per SM and stream K in 64-wide stages, so each takes
// (waves of CTAs) x (K / 64 stages) x (time of one stage of a wave), and only the stage times
// differ.  Measured on B200 over 55 shapes (M 17..4096, N 300..57344, K 1152..28672; each
// kernel timed alone), a wave's stage takes about
//   prefill_kernel:    441 ns + 1.82 ns x BN x h   (BN rows of W per CTA; h = the share of its
//                      two 128-row MMA tiles that hold rows of x; its dequantizing producers
//                      set the fixed part, the MMAs' shared-memory operand reads the rest)
//   prefill_ab_kernel: 313 ns + 0.51 ns x bn       (bn rows of x per CTA, 128 rows of W)
// The K / 64 factor is common, so the choice holds for every K.  Those times were taken with
// the calls back to back, where the clocks settle under the power cap; in short runs at full
// clock the shared-memory kernel gains a few per cent at large M (2048 x 28672 x 8192: 707 us
// against 727), so the tensor-memory kernel is taken only when it is predicted 3 % faster.  On
// the 55 shapes the rule then picks the faster kernel to within 1.2 %, and it is within 0.6 %
// on 19 shapes timed on another box.
bool prefer_prefill_ab(int M, int N, int sms) {
    const prefill::LaunchPlan po = prefill::plan(M, N, sms);
    const prefill_ab::LaunchPlan pa = prefill_ab::plan(M, N);
    const int mt = (M + prefill::kTileM - 1) / prefill::kTileM;
    const double h = static_cast<double>((M + prefill::kUmmaM - 1) / prefill::kUmmaM) / (2.0 * mt);
    const double waves_o = std::ceil(static_cast<double>(po.grid.x) / sms);
    const double waves_a = std::ceil(static_cast<double>(pa.grid.x) / sms);
    const double stage_o = 441.0 + 1.82 * po.tile_n * h;
    const double stage_a = 313.0 + 0.51 * pa.bn;
    return waves_a * stage_a < 0.97 * waves_o * stage_o;
}

// Prefill with the weights in tensor memory (prefill_swab.cuh).
w3_status launch_prefill_ab(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int M,
                            int N, int K, cudaStream_t stream) {
    const prefill_ab::LaunchPlan P = prefill_ab::plan(M, N);
    prefill_ab::Params prm;
    PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
    if (!enc) return W3_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {prefill_ab::kStageK, static_cast<cuuint32_t>(P.bn)};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&prm.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return W3_ERR_CUDA;
    // [128 rows][24 words] boxes over the packed matrix: four stages of the CTA's rows per copy
    if (encode_packed_map(&prm.tmap_w, packed, N, static_cast<int64_t>(K) * 3 / 32, prefill_ab::kChunkWords,
                          prefill_ab::kRowsW) != W3_OK)
        return W3_ERR_CUDA;
    prm.scales = scales;
    prm.y = y;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.bn = P.bn;
    prm.xtiles = P.xtiles;
    prm.idesc = prefill::make_idesc(prefill_ab::kRowsW, P.bn);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = P.grid;
    cfg.blockDim = dim3(prefill_ab::kThreads, 1, 1);
    cfg.dynamicSmemBytes = prefill_ab::SmemLayout::total;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, prefill_ab::prefill_ab_kernel, prm) == cudaSuccess ? W3_OK : W3_ERR_CUDA;
}

w3_status launch_decode(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int M,
                        int N, int K, int num_sms, cudaStream_t stream) {
    const decode::LaunchPlan P = decode::plan(M, N, K, num_sms);
    decode::Params prm;
    prm.x = x;
    prm.packed = reinterpret_cast<const uint32_t *>(packed);
    prm.scales = scales;
    prm.y = y;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.groups_per_cta = P.groups_per_cta;
    prm.gchunk = P.gchunk;
    // one tiled TMA copy per stage when the box fits inside the matrix, else per-row bulk copies
    prm.use_tma2d = 0;
    const int64_t words = static_cast<int64_t>(K) * 3 / 32;
    if (N >= decode::kRowsPerWarp && words >= decode::kRowPitchWords) {
        PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
        if (!enc) return W3_ERR_CUDA;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(words), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(words * 4)};
        cuuint32_t box[2] = {decode::kRowPitchWords, decode::kRowsPerWarp};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&prm.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<int32_t *>(packed), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W3_ERR_CUDA;
        prm.use_tma2d = 1;
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = P.grid;
    cfg.blockDim = dim3(decode::kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = P.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (P.cluster > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = P.cluster;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaError_t e;
    switch (P.mt) {
        case 1: e = cudaLaunchKernelEx(&cfg, decode::decode_kernel<1>, prm); break;
        case 2: e = cudaLaunchKernelEx(&cfg, decode::decode_kernel<2>, prm); break;
        case 4: e = cudaLaunchKernelEx(&cfg, decode::decode_kernel<4>, prm); break;
        case 8: e = cudaLaunchKernelEx(&cfg, decode::decode_kernel<8>, prm); break;
        default: e = cudaLaunchKernelEx(&cfg, decode::decode_kernel<16>, prm); break;
    }
    return e == cudaSuccess ? W3_OK : W3_ERR_CUDA;
}

const void *split_kernel(int mt) {
    switch (mt) {
        case 1: return reinterpret_cast<const void *>(dsplit::decode_split_kernel<1, false>);
        case 2: return reinterpret_cast<const void *>(dsplit::decode_split_kernel<2, false>);
        case 4: return reinterpret_cast<const void *>(dsplit::decode_split_kernel<4, false>);
        case 8: return reinterpret_cast<const void *>(dsplit::decode_split_kernel<8, false>);
        default: return reinterpret_cast<const void *>(dsplit::decode_split_kernel<16, false>);
    }
}

// Clusters of C CTAs of the split decode (batch padded to mt) with `smem` bytes each that
// the current device keeps resident at once (0 if the query fails).  Cached per device.
int split_active_clusters(int mt, int C, int smem) {
    struct Key {
        int dev, mt, C, smem, n;
    };
    static std::mutex mu;
    static Key cache[256];
    static int ncache = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    {
        std::lock_guard<std::mutex> g(mu);
        for (int i = 0; i < ncache; ++i)
            if (cache[i].dev == dev && cache[i].mt == mt && cache[i].C == C && cache[i].smem == smem) return cache[i].n;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, 1, 1);
    cfg.blockDim = dim3(dsplit::kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, split_kernel(mt), &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> g(mu);
    if (ncache < 256) cache[ncache++] = {dev, mt, C, smem, n};
    return n;
}

dsplit::LaunchPlan split_plan(int M, int N, int K, int sms) {
    const int mt = decode::padded_batch(M);
    return dsplit::plan(M, N, K, sms, [&](int C, int smem) { return split_active_clusters(mt, C, smem); });
}

// The split decode (decode_split.cuh), M <= 16, N >= 32, on the row-major words (`packed`)
// or, when `native` is given, on the native block order.
w3_status launch_decode_split(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int M,
                              int N, int K, const dsplit::LaunchPlan &P, cudaStream_t stream,
                              const int32_t *native = nullptr) {
    dsplit::Params prm;
    const int64_t words = static_cast<int64_t>(K) * 3 / 32;
    prm.native = reinterpret_cast<const uint32_t *>(native);
    const int pitch_s = dsplit::stage_groups_for(P.mt) * kWordsPerGroup;
    prm.hasS = words >= pitch_s;
    if (!native) {
        if (w3_status s = encode_packed_map(&prm.tmap1, packed, N, words, dsplit::kPitch1, dsplit::kBlockRows))
            return s;
        prm.tmapS = prm.tmap1;
        if (prm.hasS) {
            if (w3_status s = encode_packed_map(&prm.tmapS, packed, N, words, pitch_s, dsplit::kBlockRows)) return s;
        }
    }
    prm.x = x;
    prm.scales = scales;
    prm.y = y;
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.G = K / kGroup;
    prm.C = P.C;
    prm.ncl = P.ncl;
    prm.depth = P.depth;
    prm.gs_max = P.gs_max;
    prm.nb_max = P.nb_max;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.ncl * P.C, 1, 1);
    cfg.blockDim = dim3(P.warps() * 32, 1, 1);
    cfg.dynamicSmemBytes = P.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    set_pdl(attr[0]);  // overlaps the set-up with the previous kernel's tail
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (P.C > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = P.C;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    cudaError_t e;
    if (native) {
        switch (P.mt) {
            case 1: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<1, true>, prm); break;
            case 2: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<2, true>, prm); break;
            case 4: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<4, true>, prm); break;
            case 8: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<8, true>, prm); break;
            default: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<16, true>, prm); break;
        }
    } else {
        switch (P.mt) {
            case 1: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<1, false>, prm); break;
            case 2: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<2, false>, prm); break;
            case 4: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<4, false>, prm); break;
            case 8: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<8, false>, prm); break;
            default: e = cudaLaunchKernelEx(&cfg, dsplit::decode_split_kernel<16, false>, prm); break;
        }
    }
    return e == cudaSuccess ? W3_OK : W3_ERR_CUDA;
}

// ---- kernel selection (host logic only: depends on the shape and the SM count) --------

// Smallest batch of the split decode (below it, on many rows, the stream-K decode).
constexpr int kSplitMinBatch = 5;

enum class Route {
    DecodeSplit,    // decode_split_kernel: M <= 16, N >= 32 where a plan fits (cluster split-K, mma.sync)
    DecodeStreamK,  // decode_sk_kernel: M <= 4, at least one 32-row block per SM, x of all of K fits
    Decode,         // decode_kernel: the remaining shapes of M <= 16 (N < 32, or no split plan)
    DecodeTc32,     // decode_tc32 decode_tc_kernel (+ fix-up): 17 <= M <= 32, N >= 256
    Prefill,        // prefill_kernel: M > 16 (not on the 32-wide decode), K >= 256
    PrefillAb,      // prefill_ab_kernel: chosen over prefill_kernel per shape
    Passes,         // no prefill kernel fits (K < 256): 16-row passes of the decode routes
};

// Whether the split decode has a launch plan (shared memory for the prepared x of a K slice,
// a ring and the cluster's partial sums); the answer does not depend on the device's occupancy.
bool split_fits(int64_t mb, int64_t N, int64_t K, int sms) {
    return dsplit::plan(static_cast<int>(mb), static_cast<int>(N), static_cast<int>(K), sms,
                        [](int, int) { return 0; })
        .ok;
}

// The route of one pass of at most 16 batch rows.
Route decode_route(int64_t mb, int64_t N, int64_t K, int sms) {
    if (N >= dsplit::kBlockRows && mb >= kSplitMinBatch && split_fits(mb, N, K, sms)) return Route::DecodeSplit;
    if (N >= static_cast<int64_t>(decode_sk::kBlockRows) * sms &&
        decode_sk::applicable(static_cast<int>(mb), static_cast<int>(N), static_cast<int>(K)))
        return Route::DecodeStreamK;
    // fewer 32-row blocks than SMs, or x of the whole K range too large for the stream-K decode:
    // the split decode (each CTA prepares x for its K slice only; 1x4096x4096 in 5.5 us against
    // 6.9 on the older cluster decode, 1x1024x28672 in 8.5 against 14.8)
    if (N >= dsplit::kBlockRows && split_fits(mb, N, K, sms)) return Route::DecodeSplit;
    return Route::Decode;
}

Route choose_route(int64_t M, int64_t N, int64_t K, int sms) {
    if (M <= 16) return decode_route(M, N, K, sms);
    if (M <= decode_tc32::kBatch && N >= decode_tc32::kRows) return Route::DecodeTc32;
    // the prefill kernels' packed-word copies are 24 words wide: rows of at least 256 codes
    if (K >= 256)
        return prefer_prefill_ab(static_cast<int>(M), static_cast<int>(N), sms) ? Route::PrefillAb : Route::Prefill;
    return Route::Passes;
}

// Kernels one w3a16_gemm call launches for M x N x K: the route's main kernel, plus the
// fix-up kernel where the tensor-core decode splits a tile between CTAs; the passes route
// adds up its 16-row passes (one kernel each).
int64_t launches_for(int64_t M, int64_t N, int64_t K, int sms) {
    switch (choose_route(M, N, K, sms)) {
        case Route::DecodeTc32: return decode_tc32::plan(N, K, sms).P > 1 ? 2 : 1;
        case Route::Passes: return (M + 15) / 16;
        default: return 1;
    }
}

const char *route_name(Route r) {
    switch (r) {
        case Route::DecodeSplit: return "decode_split";
        case Route::DecodeStreamK: return "decode_sk";
        case Route::Decode: return "decode";
        case Route::DecodeTc32: return "decode_tc32";
        case Route::Prefill: return "prefill";
        case Route::PrefillAb: return "prefill_ab";
        case Route::Passes: return "passes";
    }
    return "";
}

// Fixed scratch of w3a16_gemm_noalloc: the fp32 partial sums of the tensor-core
// decode for up to kNoAllocMaxCtas CTAs (one per SM).  Every slot the fix-up
// kernel reads is written by the main kernel of the same call, so nothing in
// it has to start at zero.
constexpr int kNoAllocMaxCtas = 160 * decode_tc32::kCtasPerSm;
constexpr int64_t kNoAllocScratchFloats = int64_t(kNoAllocMaxCtas) * 2 * decode_tc32::kBatch * decode_tc32::kRows;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

struct NoAllocState {
    std::once_flag once;
    float *scratch = nullptr;
};
NoAllocState g_noalloc[kMaxDevices];

// Address of the scratch on the current device (looked up once per device, with
// that device current).
float *noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    NoAllocState &st = g_noalloc[dev];
    std::call_once(st.once, [&] {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) == cudaSuccess) st.scratch = static_cast<float *>(ptr);
    });
    return st.scratch;
}

// Where the tensor-core decode keeps its partial sums: a stream-ordered allocation
// from `pool` (w3a16_gemm), or the fixed array `fixed` of `fixed_floats` floats
// (w3a16_gemm_noalloc, which must never allocate).
struct ScratchSource {
    cudaMemPool_t pool = nullptr;
    float *fixed = nullptr;
    int64_t fixed_floats = 0;

    w3_status acquire(int64_t floats, cudaStream_t st, float **out) const {
        *out = nullptr;
        if (floats <= 0) return W3_OK;
        if (!pool) {
            if (!fixed) return W3_ERR_CUDA;
            if (floats > fixed_floats) return W3_ERR_UNSUPPORTED;
            *out = fixed;
            return W3_OK;
        }
        return cudaMallocFromPoolAsync(reinterpret_cast<void **>(out), floats * sizeof(float), pool, st) ==
                       cudaSuccess
                   ? W3_OK
                   : W3_ERR_CUDA;
    }
    w3_status release(float *p, cudaStream_t st) const {
        if (!p || !pool) return W3_OK;
        return cudaFreeAsync(p, st) == cudaSuccess ? W3_OK : W3_ERR_CUDA;
    }
};

// y = x W^T for validated arguments: the route's kernels, in stream order.
w3_status run_gemm(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int64_t M,
                   int64_t N, int64_t K, int sms, cudaStream_t st, const ScratchSource &scratch) {
    const int n = static_cast<int>(N), k = static_cast<int>(K);
    const Route route = choose_route(M, N, K, sms);
    if (route == Route::Prefill) return launch_prefill(x, packed, scales, y, static_cast<int>(M), n, k, sms, st);
    if (route == Route::PrefillAb) return launch_prefill_ab(x, packed, scales, y, static_cast<int>(M), n, k, st);
    if (route == Route::DecodeTc32) {
        const decode_tc32::LaunchPlan plan32 = decode_tc32::plan(N, K, sms);
        float *partial = nullptr;
        if (w3_status s = scratch.acquire(plan32.ws_floats, st, &partial)) return s;
        w3_status status = launch_decode_tc<decode_tc32::Instance>(x, packed, scales, y, static_cast<int>(M), n, k,
                                                                   plan32, partial, st);
        if (w3_status s = scratch.release(partial, st); s && status == W3_OK) status = s;
        return status;
    }
    // Decode routes, in passes of at most 16 batch rows (one pass unless M > 16 with K < 256,
    // where no prefill kernel fits).
    w3_status status = W3_OK;
    for (int64_t m0 = 0; m0 < M && status == W3_OK; m0 += 16) {
        const int mb = static_cast<int>(std::min<int64_t>(16, M - m0));
        const uint16_t *xp = x + m0 * K;
        uint16_t *yp = y + m0 * N;
        switch (decode_route(mb, N, K, sms)) {
            case Route::DecodeSplit: {
                // the route was chosen because a plan exists, with or without the occupancy answer
                const dsplit::LaunchPlan sp = split_plan(mb, n, k, sms);
                status = sp.ok ? launch_decode_split(xp, packed, scales, yp, mb, n, k, sp, st) : W3_ERR_UNSUPPORTED;
                break;
            }
            case Route::DecodeStreamK: status = launch_decode_sk(xp, packed, scales, yp, mb, n, k, sms, st); break;
            default: status = launch_decode(xp, packed, scales, yp, mb, n, k, sms, st); break;
        }
    }
    return status;
}

// The checks every product entry point makes before anything is launched.
w3_status check_gemm_args(const uint16_t *x, const int32_t *packed, const uint16_t *scales, const uint16_t *y,
                          int64_t M, int64_t N, int64_t K) {
    if (!x || !packed || !scales || !y) return W3_ERR_NULL;
    if (w3_status s = check_nk(N, K)) return s;
    if (M < 1 || M > kMaxDim || M * K > kMaxElems || M * N > kMaxElems) return W3_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y)) return W3_ERR_ALIGN;
    const int64_t ybytes = M * N * 2;
    if (overlaps(y, ybytes, x, M * K * 2) || overlaps(y, ybytes, packed, N * K * 3 / 8) ||
        overlaps(y, ybytes, scales, N * (K / kGroup) * 2))
        return W3_ERR_ALIAS;
    return W3_OK;
}

// y = x W^T on the native block order (validated arguments): M <= 16, N >= 32.
w3_status run_gemm_native(const uint16_t *x, const int32_t *native, const uint16_t *scales, uint16_t *y,
                          int64_t M, int64_t N, int64_t K, int sms, cudaStream_t st) {
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    if (M <= 4 && N >= static_cast<int64_t>(decode_sk::kBlockRows) * sms && decode_sk::applicable(m, n, k))
        return launch_decode_sk(x, nullptr, scales, y, m, n, k, sms, st, native);
    const dsplit::LaunchPlan sp = split_plan(m, n, k, sms);
    if (!sp.ok) return W3_ERR_UNSUPPORTED;
    return launch_decode_split(x, nullptr, scales, y, m, n, k, sp, st, native);
}

int64_t native_words(int64_t N, int64_t K) { return (N + 31) / 32 * 32 * (K * 3 / 32); }

#ifdef W3_TEST_HOOKS
// Test-only: one thread waits, with the bounded wait every kernel uses, on an
// mbarrier phase that nothing completes, so the wait runs out and records the
// timeout flag.  Built only into the test variant of the library (which also
// shortens the wait limit).
__global__ void wait_timeout_kernel() {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        mbar_init_fence();
        (void)mbar_wait_bounded(smem_addr(&bar), 0);
    }
}
#endif

}  // namespace
}  // namespace w3

using namespace w3;

extern "C" {

const char *w3_status_string(w3_status s) {
    switch (s) {
        case W3_OK: return "ok";
        case W3_ERR_NULL: return "a required pointer is NULL";
        case W3_ERR_SHAPE: return "a size is out of range (M, N >= 1; K a positive multiple of 128)";
        case W3_ERR_ALIGN: return "an array pointer is not 16-byte aligned";
        case W3_ERR_CUDA: return "the CUDA runtime reported an error";
        case W3_ERR_UNSUPPORTED: return "the current device is not an sm_100 (B200) GPU";
        case W3_ERR_TIMEOUT: return "a device-side wait timed out";
        case W3_ERR_ALIAS: return "the output overlaps an input";
    }
    return "unknown status";
}

int32_t w3_abi_version(void) { return 1; }

int64_t w3_packed_words_per_row(int64_t K) {
    return (K >= kGroup && K % kGroup == 0) ? K * 3 / 32 : -1;
}

int64_t w3_groups_per_row(int64_t K) { return (K >= kGroup && K % kGroup == 0) ? K / kGroup : -1; }

w3_status w3_pack(const uint8_t *codes, int32_t *packed, int64_t N, int64_t K, w3_stream_t stream) {
    if (!codes || !packed) return W3_ERR_NULL;
    if (w3_status s = check_nk(N, K)) return s;
    if (!aligned16(codes) || !aligned16(packed)) return W3_ERR_ALIGN;
    if (overlaps(codes, N * K, packed, N * K * 3 / 8)) return W3_ERR_ALIAS;
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    const int64_t nblocks = N * K / 32;
    pack_kernel<<<grid_for(nblocks, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        codes, reinterpret_cast<uint32_t *>(packed), nblocks);
    return launch_status();
}

w3_status w3_unpack(const int32_t *packed, uint8_t *codes, int64_t N, int64_t K, w3_stream_t stream) {
    if (!codes || !packed) return W3_ERR_NULL;
    if (w3_status s = check_nk(N, K)) return s;
    if (!aligned16(codes) || !aligned16(packed)) return W3_ERR_ALIGN;
    if (overlaps(codes, N * K, packed, N * K * 3 / 8)) return W3_ERR_ALIAS;
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    const int64_t nblocks = N * K / 32;
    unpack_kernel<<<grid_for(nblocks, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint32_t *>(packed), codes, nblocks);
    return launch_status();
}

w3_status w3_repack_ct4(const int32_t *ct4, int32_t *packed, int64_t N, int64_t K, int64_t *out_of_range,
                        w3_stream_t stream) {
    if (!ct4 || !packed) return W3_ERR_NULL;
    if (w3_status s = check_nk(N, K)) return s;
    if (!aligned16(ct4) || !aligned16(packed) || (out_of_range && (reinterpret_cast<uintptr_t>(out_of_range) & 7u)))
        return W3_ERR_ALIGN;
    if (overlaps(ct4, N * K / 2, packed, N * K * 3 / 8) ||
        (out_of_range && (overlaps(out_of_range, 8, ct4, N * K / 2) || overlaps(out_of_range, 8, packed, N * K * 3 / 8))))
        return W3_ERR_ALIAS;
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (out_of_range && cudaMemsetAsync(out_of_range, 0, sizeof(int64_t), st) != cudaSuccess) return W3_ERR_CUDA;
    const int64_t nblocks = N * K / 32;
    repack_ct4_kernel<<<grid_for(nblocks, 256), 256, 0, st>>>(reinterpret_cast<const uint4 *>(ct4),
                                                             reinterpret_cast<uint32_t *>(packed), nblocks,
                                                             reinterpret_cast<unsigned long long *>(out_of_range));
    return launch_status();
}

w3_status w3_dequant_f32(const int32_t *packed, const uint16_t *scales, float *w, int64_t N, int64_t K,
                         w3_stream_t stream) {
    if (!packed || !scales || !w) return W3_ERR_NULL;
    if (w3_status s = check_nk(N, K)) return s;
    if (!aligned16(packed) || !aligned16(scales) || !aligned16(w)) return W3_ERR_ALIGN;
    if (overlaps(w, N * K * 4, packed, N * K * 3 / 8) || overlaps(w, N * K * 4, scales, N * (K / kGroup) * 2))
        return W3_ERR_ALIAS;
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    const int64_t nblocks = N * K / 32;
    dequant_f32_kernel<<<grid_for(nblocks, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint32_t *>(packed), scales, w, nblocks, K / 32, K / kGroup);
    return launch_status();
}

w3_status w3a16_gemm(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y, int64_t M,
                     int64_t N, int64_t K, w3_stream_t stream) {
    if (w3_status s = check_gemm_args(x, packed, scales, y, M, N, K)) return s;
    int sms;
    cudaMemPool_t pool;
    if (w3_status s = device_setup(&sms, &pool)) return s;
    ScratchSource scratch;
    scratch.pool = pool;
    return run_gemm(x, packed, scales, y, M, N, K, sms, reinterpret_cast<cudaStream_t>(stream), scratch);
}

w3_status w3a16_gemm_noalloc(const uint16_t *x, const int32_t *packed, const uint16_t *scales, uint16_t *y,
                             int64_t M, int64_t N, int64_t K, w3_stream_t stream) {
    if (w3_status s = check_gemm_args(x, packed, scales, y, M, N, K)) return s;
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    ScratchSource scratch;  // no pool: every route that needs scratch gets the fixed array
    scratch.fixed = noalloc_scratch();
    scratch.fixed_floats = kNoAllocScratchFloats;
    if (!scratch.fixed) return W3_ERR_CUDA;
    return run_gemm(x, packed, scales, y, M, N, K, sms, reinterpret_cast<cudaStream_t>(stream), scratch);
}

int64_t w3_native_words(int64_t N, int64_t K) { return check_nk(N, K) == W3_OK ? native_words(N, K) : -1; }

// The three conversions of the native block order: one thread per 3-word block.
static w3_status native_convert(int kind, const void *src, void *dst, int64_t N, int64_t K, w3_stream_t stream) {
    if (!src || !dst) return W3_ERR_NULL;
    if (w3_status s = check_nk(N, K)) return s;
    if (!aligned16(src) || !aligned16(dst)) return W3_ERR_ALIGN;
    const int64_t nwords = native_words(N, K), rwords = N * K * 3 / 32;
    const int64_t src_bytes = kind == 0 ? N * K : kind == 1 ? rwords * 4 : nwords * 4;
    const int64_t dst_bytes = kind == 2 ? rwords * 4 : nwords * 4;
    if (overlaps(src, src_bytes, dst, dst_bytes)) return W3_ERR_ALIAS;
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    const int64_t nthreads = nwords / 3;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (kind == 0)
        pack_native_kernel<<<grid_for(nthreads, 256), 256, 0, st>>>(static_cast<const uint8_t *>(src),
                                                                    static_cast<uint32_t *>(dst), N, K, nthreads);
    else if (kind == 1)
        native_from_packed_kernel<<<grid_for(nthreads, 256), 256, 0, st>>>(static_cast<const uint32_t *>(src),
                                                                           static_cast<uint32_t *>(dst), N, K,
                                                                           nthreads);
    else
        packed_from_native_kernel<<<grid_for(nthreads, 256), 256, 0, st>>>(static_cast<const uint32_t *>(src),
                                                                           static_cast<uint32_t *>(dst), N, K,
                                                                           nthreads);
    return launch_status();
}

w3_status w3_pack_native(const uint8_t *codes, int32_t *native, int64_t N, int64_t K, w3_stream_t stream) {
    return native_convert(0, codes, native, N, K, stream);
}

w3_status w3_native_from_packed(const int32_t *packed, int32_t *native, int64_t N, int64_t K, w3_stream_t stream) {
    return native_convert(1, packed, native, N, K, stream);
}

w3_status w3_packed_from_native(const int32_t *native, int32_t *packed, int64_t N, int64_t K, w3_stream_t stream) {
    return native_convert(2, native, packed, N, K, stream);
}

w3_status w3a16_gemm_native(const uint16_t *x, const int32_t *native, const uint16_t *scales, uint16_t *y, int64_t M,
                            int64_t N, int64_t K, w3_stream_t stream) {
    if (!x || !native || !scales || !y) return W3_ERR_NULL;
    if (w3_status s = check_nk(N, K)) return s;
    if (M < 1 || M > 16 || N < 32) return M < 1 ? W3_ERR_SHAPE : W3_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(native) || !aligned16(scales) || !aligned16(y)) return W3_ERR_ALIGN;
    const int64_t ybytes = M * N * 2;
    if (overlaps(y, ybytes, x, M * K * 2) || overlaps(y, ybytes, native, native_words(N, K) * 4) ||
        overlaps(y, ybytes, scales, N * (K / kGroup) * 2))
        return W3_ERR_ALIAS;
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    return run_gemm_native(x, native, scales, y, M, N, K, sms, reinterpret_cast<cudaStream_t>(stream));
}

const char *w3a16_gemm_route(int64_t M, int64_t N, int64_t K, int32_t num_sms) {
    if (M < 1 || check_nk(N, K) != W3_OK || M > kMaxDim || num_sms < 1) return nullptr;
    return route_name(choose_route(M, N, K, num_sms));
}

int32_t w3a16_gemm_launches(int64_t M, int64_t N, int64_t K, int32_t num_sms) {
    if (M < 1 || check_nk(N, K) != W3_OK || M > kMaxDim || num_sms < 1) return -1;
    const int64_t n = launches_for(M, N, K, num_sms);
    return n > INT32_MAX ? INT32_MAX : static_cast<int32_t>(n);
}

#ifdef W3_TEST_HOOKS
w3_status w3_test_wait_timeout(w3_stream_t stream) {
    int sms;
    if (w3_status s = device_setup(&sms)) return s;
    wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    return launch_status();
}
#endif

w3_status w3_check_device_error(w3_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return W3_ERR_CUDA;
    unsigned int flag = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&flag, g_device_error, sizeof flag) != cudaSuccess) return W3_ERR_CUDA;
    if (flag == 0) return W3_OK;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) return W3_ERR_CUDA;
    return W3_ERR_TIMEOUT;
}

}  // extern "C"
