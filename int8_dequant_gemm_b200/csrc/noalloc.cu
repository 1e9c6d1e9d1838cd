// rt_qgemm_noalloc: the quantized GEMM without any device allocation.
//
// The TMA-fed tensor-core kernels that stage the activations rounded to the
// 16-bit operand type (activation-resident below 16384 rows, weight-streamed)
// need scratch for them (M * K * 2 bytes).  rt_qgemm_q4/q8 take it from
// a per-stream workspace that grows with cudaMalloc and, when it grows,
// synchronizes the stream and frees the old buffer.  Some callers cannot do
// that: a serving process whose pool allocator already owns nearly all of
// HBM (so a late cudaMalloc fails), or a latency-bound loop that cannot take
// the stall of a growth sync or of cudaFree.  This entry point runs the same
// kernels on scratch that lives in a fixed file-scope device array instead,
// and rejects problems that do not fit in it.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/rtq.h"
#include "kernels.cuh"

// One array per device, loaded with this module.  Every rt_qgemm_noalloc call
// on a device shares it; nothing in it has to start at zero, because each
// call's pre-pass writes every byte the call's GEMM kernel then reads.
static __device__ __align__(256) unsigned char g_rtq_noalloc_scratch[RT_NOALLOC_SCRATCH_BYTES];

namespace {

using rtq::kMaxDevices;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Set-up, once per device, with that device current: the device address of
// the array.  This may load the module, so the first call on a device should
// come before any stream capture.
rt_status scratch_ptr(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RT_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RT_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_rtq_noalloc_scratch) != cudaSuccess) return RT_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return RT_OK;
}

inline rt_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RT_OK : RT_ERR_CUDA; }

}  // namespace

extern "C" rt_status rt_qgemm_noalloc(int fmt, const float *X, const void *Wq, const void *scales,
                                      float *Y, int64_t M, int64_t N, int64_t K, int path,
                                      void *stream) {
    if (fmt != 4 && fmt != 8) return RT_ERR_INVALID_ARG;
    rt_status st = rtq::check_gemm_args(fmt, X, Wq, scales, Y, M, N, K);
    if (st != RT_OK) return st;
    if (path < RT_PATH_AUTO || path > RT_PATH_TC) return RT_ERR_INVALID_ARG;
    const int kern = rtq::plan_with_scales(fmt, M, N, K, path, scales);
    if (kern < 0) return RT_ERR_UNSUPPORTED_SHAPE;
    const bool staged = kern == RT_KERNEL_TC_X_RESIDENT || kern == RT_KERNEL_TC_W_STREAMED;
    if (staged && M * K * 2 > static_cast<int64_t>(RT_NOALLOC_SCRATCH_BYTES))
        return RT_ERR_SCRATCH_LIMIT;
    void *xh = nullptr;
    if ((st = scratch_ptr(&xh)) != RT_OK) return st;
    if (M == 0) return RT_OK;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    if (kern == RT_KERNEL_SIMT)
        return from_cuda(rtq::launch_simt(fmt, X, Wq, scales, nullptr, Y, m, n, k, s));
    rtq::DevCtl *ctl = nullptr;
    if ((st = rtq::device_ctl(&ctl)) != RT_OK) return st;
    if (kern == RT_KERNEL_TC_W_STATIONARY)
        return from_cuda(rtq::launch_tc(fmt, X, Wq, scales, nullptr, Y, m, n, k, ctl, s));
    if (kern == RT_KERNEL_TC_X_RESIDENT_PAIR)
        return from_cuda(rtq::launch_xp(fmt, X, Wq, scales, nullptr, Y, m, n, k, ctl, s));
    if (rtq::launch_cvt_x16(X, xh, M, K, ctl, s) != cudaSuccess) return RT_ERR_CUDA;
    if (kern == RT_KERNEL_TC_X_RESIDENT)
        return from_cuda(rtq::launch_xs(fmt, xh, Wq, scales, nullptr, Y, m, n, k, ctl, s));
    return from_cuda(rtq::launch_ws(fmt, xh, Wq, scales, nullptr, Y, m, n, k, ctl, s));
}
