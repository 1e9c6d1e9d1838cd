// Activation pre-pass of the TMA-fed tensor-core kernels, and the TMA map
// encoder they share.
//
// The pre-pass rounds X (fp32 [M, K]) once to fp16 and stores it in the chunk
// order the MMA operands use (pairs (k + t, k + t + 4), t = 0..3, within
// every 8 elements k .. k+7, see dequant.cuh).  The GEMM kernels then load activation tiles
// with TMA straight into the 128-byte-swizzled operand layout, with no
// conversion work and at half the bytes of fp32.  It is a pure streaming
// kernel: 4 bytes read and 2 written per element.  An activation that is not
// a finite fp16 value after rounding latches kStatusRange.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "kernels.cuh"
#include "tmapipe.cuh"

namespace rtq {
namespace {

__global__ void __launch_bounds__(256)
    cvt_x16_kernel(const float4 *__restrict__ X, uint4 *__restrict__ Xh, int64_t n_chunks,
                   DevCtl *ctl) {
    // the next kernel may be scheduled now: it reads this one's output only
    // after its own wait for this grid's completion
    pdl_launch_dependents();
    pdl_wait_prior_grid();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    uint32_t bad = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_chunks;
         i += stride) {
        const float4 a = __ldcs(X + 2 * i), b = __ldcs(X + 2 * i + 1);
        const uint4 c = x8_f16(a, b);
        bad |= f16x2_nonfinite(make_uint2(c.x, c.y)) | f16x2_nonfinite(make_uint2(c.z, c.w));
        Xh[i] = c;
    }
    if (__any_sync(0xffffffffu, bad != 0) && (threadIdx.x & 31) == 0)
        atomicOr(&ctl->status, 1u << kStatusRange);
}

// The same rounding in a shape that fits on each SM beside a persistent GEMM
// CTA of another launch, for an input rounded on a second stream while that
// launch computes.  Registers are split between an SM's four sub-partitions
// (16384 each) and a block's warps are spread over them, so the block is one
// warp per sub-partition: 128 threads of at most 64 registers (2048 a
// sub-partition), which fits beside the activation-resident kernel's 5 warps
// of 88 registers (14080) per sub-partition, with no shared memory; four
// chunks in flight per thread.
constexpr int kLeanThreads = 128;
constexpr int kLeanDepth = 4;
__global__ void __launch_bounds__(kLeanThreads, 8)
    cvt_x16_lean_kernel(const float4 *__restrict__ X, uint4 *__restrict__ Xh, int64_t n_chunks,
                        DevCtl *ctl) {
    const uint32_t stride = gridDim.x * blockDim.x;       // chunks between a thread's chunks
    uint32_t bad = 0;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const float4 *x = X + 2 * i;
    uint4 *h = Xh + i;
    for (; i + (kLeanDepth - 1) * static_cast<int64_t>(stride) < n_chunks;
         i += kLeanDepth * stride, x += 2 * kLeanDepth * stride, h += kLeanDepth * stride) {
        float4 a[kLeanDepth], b[kLeanDepth];
#pragma unroll
        for (int d = 0; d < kLeanDepth; ++d) {
            a[d] = __ldcs(x + 2 * d * stride);
            b[d] = __ldcs(x + 2 * d * stride + 1);
        }
#pragma unroll
        for (int d = 0; d < kLeanDepth; ++d) {
            const uint4 c = x8_f16(a[d], b[d]);
            h[d * stride] = c;
            bad |= f16x2_nonfinite(make_uint2(c.x, c.y)) | f16x2_nonfinite(make_uint2(c.z, c.w));
        }
    }
    for (; i < n_chunks; i += stride, x += 2 * stride, h += stride) {
        const uint4 c = x8_f16(__ldcs(x), __ldcs(x + 1));
        h[0] = c;
        bad |= f16x2_nonfinite(make_uint2(c.x, c.y)) | f16x2_nonfinite(make_uint2(c.z, c.w));
    }
    if (__any_sync(0xffffffffu, bad != 0) && (threadIdx.x & 31) == 0)
        atomicOr(&ctl->status, 1u << kStatusRange);
}

// The same rounding over up to kMaxGroup tensors, one grid-stride walk over
// their concatenated 8-element chunks (end[i]: running chunk totals).
struct CvtGroup {
    const float4 *X[kMaxGroup];
    uint4 *Xh[kMaxGroup];
    int64_t end[kMaxGroup];
    int count;
};

__global__ void __launch_bounds__(256) cvt_x16_group_kernel(const __grid_constant__ CvtGroup g,
                                                            DevCtl *ctl) {
    pdl_launch_dependents();
    pdl_wait_prior_grid();
    const int64_t total = g.end[g.count - 1];
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    uint32_t bad = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += stride) {
        int t = 0;
        while (i >= g.end[t]) ++t;
        const int64_t c = i - (t > 0 ? g.end[t - 1] : 0);
        const float4 a = __ldcs(g.X[t] + 2 * c), b = __ldcs(g.X[t] + 2 * c + 1);
        const uint4 v = x8_f16(a, b);
        bad |= f16x2_nonfinite(make_uint2(v.x, v.y)) | f16x2_nonfinite(make_uint2(v.z, v.w));
        g.Xh[t][c] = v;
    }
    if (__any_sync(0xffffffffu, bad != 0) && (threadIdx.x & 31) == 0)
        atomicOr(&ctl->status, 1u << kStatusRange);
}

// Launch shape of a pre-pass over n_chunks chunks: 256 threads a block, at
// most 8 blocks per SM, programmatic dependent launch.
cudaLaunchConfig_t cvt_config(int64_t n_chunks, cudaStream_t s, cudaLaunchAttribute *attr) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (n_chunks + 255) / 256;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, 8LL * sms))), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

}  // namespace

cudaError_t launch_cvt_x16(const float *X, void *Xh, int64_t M, int64_t K, DevCtl *ctl,
                           cudaStream_t s) {
    const int64_t n_chunks = M * K / 8;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = cvt_config(n_chunks, s, attr);
    const float4 *x4 = reinterpret_cast<const float4 *>(X);
    uint4 *h = static_cast<uint4 *>(Xh);
    return cudaLaunchKernelEx(&cfg, cvt_x16_kernel, x4, h, n_chunks, ctl);
}

cudaError_t launch_cvt_x16_lean(const float *X, void *Xh, int64_t M, int64_t K, DevCtl *ctl,
                                cudaStream_t s) {
    const int64_t n_chunks = M * K / 8;
    if (n_chunks == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = std::min<int64_t>(sms, (n_chunks + kLeanThreads - 1) / kLeanThreads);
    cvt_x16_lean_kernel<<<static_cast<unsigned>(blocks), kLeanThreads, 0, s>>>(
        reinterpret_cast<const float4 *>(X), static_cast<uint4 *>(Xh), n_chunks, ctl);
    return cudaGetLastError();
}

bool cvt_x16_lean_shape(int *threads, int *regs) {
    static std::atomic<int> regs_cache{0};   // looked up once
    int r = regs_cache.load(std::memory_order_acquire);
    if (r == 0) {
        cudaFuncAttributes fa = {};
        if (cudaFuncGetAttributes(&fa, cvt_x16_lean_kernel) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        r = fa.numRegs;
        regs_cache.store(r, std::memory_order_release);
    }
    *threads = kLeanThreads;
    *regs = r;
    return true;
}

cudaError_t launch_cvt_x16_group(const float *const *X, void *const *Xh, const int64_t *K,
                                 int count, int64_t M, DevCtl *ctl, cudaStream_t s) {
    if (count < 1 || count > kMaxGroup) return cudaErrorInvalidValue;
    CvtGroup g = {};
    g.count = count;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        g.X[i] = reinterpret_cast<const float4 *>(X[i]);
        g.Xh[i] = static_cast<uint4 *>(Xh[i]);
        total += M * K[i] / 8;
        g.end[i] = total;
    }
    if (total == 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = cvt_config(total, s, attr);
    return cudaLaunchKernelEx(&cfg, cvt_x16_group_kernel, g, ctl);
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}
}  // namespace

bool encode_tma_2d(CUtensorMap *map, CUtensorMapDataType dt, int esize, const void *ptr,
                   uint64_t cols, uint64_t rows, uint32_t bcols, CUtensorMapSwizzle swizzle,
                   uint32_t brows) {
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
    cuuint32_t box[2] = {bcols, brows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace rtq
