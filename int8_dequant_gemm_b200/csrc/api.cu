// C ABI of the library (declared in include/rtq.h): argument validation, the
// M-based choice between the SIMT and tensor-core kernels, the per-block
// projection driver and the device status word.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/rtq.h"
#include "kernels.cuh"

// Latched by kernels whose bounded waits gave up (bit RT_ERR_DEVICE_TIMEOUT).
__device__ unsigned int g_rtq_device_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
unsigned *g_status_ptr[kMaxDevices] = {nullptr};

// Device address of the status word on the current device (looked up once).
rt_status status_word(unsigned **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_status_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_rtq_device_status) != cudaSuccess) return RT_ERR_CUDA;
        g_status_ptr[dev] = static_cast<unsigned *>(p);
    }
    *out = g_status_ptr[dev];
    return RT_OK;
}

inline bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline bool overlap(const void *a, int64_t abytes, const void *b, int64_t bbytes) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

// Validation shared by both formats.  wbytes/sbytes: sizes of the payload and
// the scale tensor; walign/salign: their required alignment.
rt_status validate(const float *X, const void *Wq, const void *S, const float *Y, int64_t M,
                   int64_t N, int64_t K, int64_t wbytes, int64_t sbytes, uintptr_t salign,
                   int64_t k_granule) {
    if (M < 0 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
        return RT_ERR_INVALID_ARG;
    if (K % k_granule != 0) return RT_ERR_UNSUPPORTED_SHAPE;
    if (!Wq || !S) return RT_ERR_INVALID_ARG;
    if (M > 0 && (!X || !Y)) return RT_ERR_INVALID_ARG;
    if (!aligned(Wq, 16) || !aligned(S, salign)) return RT_ERR_ALIGNMENT;
    if (M > 0 && (!aligned(X, 16) || !aligned(Y, 16))) return RT_ERR_ALIGNMENT;
    if (M > 0) {
        const int64_t ybytes = M * N * 4;
        if (overlap(Y, ybytes, X, M * K * 4) || overlap(Y, ybytes, Wq, wbytes) ||
            overlap(Y, ybytes, S, sbytes))
            return RT_ERR_INVALID_ARG;
    }
    return RT_OK;
}

int pick_path(int64_t M, int64_t K, int path) {
    const bool tc_ok = (K % 64) == 0;
    if (path == RT_PATH_TC || path == RT_PATH_TC_BF16) return tc_ok ? path : -1;
    if (path == RT_PATH_SIMT) return RT_PATH_SIMT;
    if (path != RT_PATH_AUTO) return -2;
    return (M <= rtq::kAutoSimtMaxM || !tc_ok) ? RT_PATH_SIMT : RT_PATH_TC;
}

inline rt_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RT_OK : RT_ERR_CUDA; }

}  // namespace

extern "C" {

const char *rt_status_string(int status) {
    switch (status) {
        case RT_OK: return "ok";
        case RT_ERR_INVALID_ARG: return "invalid argument";
        case RT_ERR_ALIGNMENT: return "misaligned pointer";
        case RT_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case RT_ERR_CUDA: return "CUDA runtime error";
        case RT_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case RT_ERR_VALUE_RANGE: return "value out of range";
        default: return "unknown status";
    }
}

int rt_version(void) { return 100; }

int rt_qgemm_auto_path(int fmt, int64_t M, int64_t N, int64_t K) {
    if ((fmt != 4 && fmt != 8) || M < 0 || N < 1 || K < 1) return -1;
    if (K % (fmt == 4 ? 32 : 16) != 0) return -1;
    return pick_path(M, K, RT_PATH_AUTO);
}

int rt_qgemm_plan(int fmt, int64_t M, int64_t N, int64_t K, int path) {
    if ((fmt != 4 && fmt != 8) || M < 0 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim ||
        K > kMaxDim)
        return -1;
    if (K % (fmt == 4 ? 32 : 16) != 0) return -1;
    const int p = pick_path(M, K, path);
    if (p < 0) return -1;
    if (p == RT_PATH_SIMT) return RT_KERNEL_SIMT;
    return rtq::xs_supported(static_cast<int>(M), static_cast<int>(N), static_cast<int>(K))
               ? RT_KERNEL_TC_X_RESIDENT
               : RT_KERNEL_TC_W_STATIONARY;
}

rt_status rt_qgemm_q4(const float *X, const uint8_t *Wq, const uint16_t *scale_min, float *Y,
                      int64_t M, int64_t N, int64_t K, int path, void *stream) {
    rt_status st = validate(X, Wq, scale_min, Y, M, N, K, N * (K / 2), N * (K / 32) * 4, 4, 32);
    if (st != RT_OK) return st;
    const int p = pick_path(M, K, path);
    if (p == -1) return RT_ERR_UNSUPPORTED_SHAPE;
    if (p < 0) return RT_ERR_INVALID_ARG;
    if (M == 0) return RT_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p == RT_PATH_SIMT)
        return from_cuda(rtq::launch_simt_q4(X, Wq, scale_min, Y, static_cast<int>(M),
                                             static_cast<int>(N), static_cast<int>(K), s));
    unsigned *status = nullptr;
    if ((st = status_word(&status)) != RT_OK) return st;
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    const bool bf16 = p == RT_PATH_TC_BF16;
    if (rtq::xs_supported(m, n, k))
        return from_cuda(rtq::launch_xs_q4(X, Wq, scale_min, Y, m, n, k, bf16, status, s));
    return from_cuda(rtq::launch_tc_q4(X, Wq, scale_min, Y, m, n, k, bf16, status, s));
}

rt_status rt_qgemm_q8(const float *X, const int8_t *Wq, const float *scale, float *Y, int64_t M,
                      int64_t N, int64_t K, int path, void *stream) {
    rt_status st = validate(X, Wq, scale, Y, M, N, K, N * K, N * 4, 4, 16);
    if (st != RT_OK) return st;
    const int p = pick_path(M, K, path);
    if (p == -1) return RT_ERR_UNSUPPORTED_SHAPE;
    if (p < 0) return RT_ERR_INVALID_ARG;
    if (M == 0) return RT_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p == RT_PATH_SIMT)
        return from_cuda(rtq::launch_simt_q8(X, Wq, scale, Y, static_cast<int>(M),
                                             static_cast<int>(N), static_cast<int>(K), s));
    unsigned *status = nullptr;
    if ((st = status_word(&status)) != RT_OK) return st;
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    const bool bf16 = p == RT_PATH_TC_BF16;
    if (rtq::xs_supported(m, n, k))
        return from_cuda(rtq::launch_xs_q8(X, Wq, scale, Y, m, n, k, bf16, status, s));
    return from_cuda(rtq::launch_tc_q8(X, Wq, scale, Y, m, n, k, bf16, status, s));
}

rt_status rt_qblock_project(const rt_qblock *blk, int64_t M, const float *X_qkvg,
                            const float *X_o, const float *X_ffn, const float *X_w2,
                            float *Y_qkvg, float *Y_o, float *Y_13, float *Y_2, int path,
                            void *stream) {
    if (!blk || blk->d_model < 1 || blk->d_ff < 1) return RT_ERR_INVALID_ARG;
    const int64_t d = blk->d_model, f = blk->d_ff;
    rt_status st;
    if ((st = rt_qgemm_q4(X_qkvg, blk->qkvg, blk->qkvg_sm, Y_qkvg, M, 4 * d, d, path, stream)) !=
        RT_OK)
        return st;
    if ((st = rt_qgemm_q8(X_o, blk->wo, blk->wo_s, Y_o, M, d, d, path, stream)) != RT_OK)
        return st;
    if ((st = rt_qgemm_q4(X_ffn, blk->w13, blk->w13_sm, Y_13, M, 2 * f, d, path, stream)) !=
        RT_OK)
        return st;
    return rt_qgemm_q8(X_w2, blk->w2, blk->w2_s, Y_2, M, d, f, path, stream);
}

static rt_status validate_dequant(const void *Wq, const void *S, const void *W, int64_t N,
                                  int64_t K, int64_t granule, uintptr_t salign) {
    if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim) return RT_ERR_INVALID_ARG;
    if (K % granule != 0) return RT_ERR_UNSUPPORTED_SHAPE;
    if (!Wq || !S || !W) return RT_ERR_INVALID_ARG;
    if (!aligned(Wq, 16) || !aligned(W, 16) || !aligned(S, salign)) return RT_ERR_ALIGNMENT;
    return RT_OK;
}

rt_status rt_dequant_q4_f32(const uint8_t *Wq, const uint16_t *scale_min, float *W_out,
                            int64_t N, int64_t K, void *stream) {
    rt_status st = validate_dequant(Wq, scale_min, W_out, N, K, 32, 4);
    if (st != RT_OK) return st;
    return from_cuda(rtq::launch_dequant_q4_f32(Wq, scale_min, W_out, static_cast<int>(N),
                                                static_cast<int>(K),
                                                static_cast<cudaStream_t>(stream)));
}

rt_status rt_dequant_q8_f32(const int8_t *Wq, const float *scale, float *W_out, int64_t N,
                            int64_t K, void *stream) {
    rt_status st = validate_dequant(Wq, scale, W_out, N, K, 16, 4);
    if (st != RT_OK) return st;
    return from_cuda(rtq::launch_dequant_q8_f32(Wq, scale, W_out, static_cast<int>(N),
                                                static_cast<int>(K),
                                                static_cast<cudaStream_t>(stream)));
}

rt_status rt_dequant_q4_bf16(const uint8_t *Wq, const uint16_t *scale_min, uint16_t *W_out,
                             int64_t N, int64_t K, void *stream) {
    rt_status st = validate_dequant(Wq, scale_min, W_out, N, K, 32, 4);
    if (st != RT_OK) return st;
    return from_cuda(rtq::launch_dequant_q4_16(Wq, scale_min, W_out, static_cast<int>(N),
                                               static_cast<int>(K), true,
                                               static_cast<cudaStream_t>(stream)));
}

rt_status rt_dequant_q4_f16(const uint8_t *Wq, const uint16_t *scale_min, uint16_t *W_out,
                            int64_t N, int64_t K, void *stream) {
    rt_status st = validate_dequant(Wq, scale_min, W_out, N, K, 32, 4);
    if (st != RT_OK) return st;
    return from_cuda(rtq::launch_dequant_q4_16(Wq, scale_min, W_out, static_cast<int>(N),
                                               static_cast<int>(K), false,
                                               static_cast<cudaStream_t>(stream)));
}

rt_status rt_device_status(void *stream, int *device_status) {
    if (!device_status) return RT_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return RT_ERR_CUDA;
    unsigned *p = nullptr;
    rt_status st = status_word(&p);
    if (st != RT_OK) return st;
    unsigned v = 0;
    if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return RT_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
            return RT_ERR_CUDA;
    }
    *device_status = v ? RT_ERR_DEVICE_TIMEOUT : RT_OK;
    return RT_OK;
}

}  // extern "C"
