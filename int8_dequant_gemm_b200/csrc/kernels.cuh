// Launchers of the device kernels, called only by the C ABI layer (api.cu,
// noalloc.cu), and the per-device control block the tensor-core kernels read.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/rtq.h"

namespace rtq {

constexpr int kMaxDevices = 64;

// Weight formats (the `fmt` arguments): q4 g32 with (scale, min), q8 with a
// row scale, FP8 E4M3 without scale.  The e4m3 payload has the q8 layout
// (one byte per weight, [N, K]); kernels treat it as q8 with another byte
// conversion and no scale.
constexpr int kFmtQ4 = 4;
constexpr int kFmtQ8 = 8;
constexpr int kFmtE4M3 = 3;
inline bool fmt_valid(int f) { return f == kFmtQ4 || f == kFmtQ8 || f == kFmtE4M3; }

// Per-device control block, one __device__ instance (api.cu).  Every
// tensor-core kernel reads `wait_ns` and `inject` at its start and ORs status
// bits into `status`; rt_device_status() reads and clears the bits.
//   status  bit kStatusTimeout: a bounded mbarrier wait gave up;
//           bit kStatusRange:   an activation was not a finite fp16 value
//                               after rounding (|x| >= 65520, inf or NaN).
//   inject  test hook (rt_debug_inject): 1 makes the first producer arrival
//           of every CTA go missing, so a consumer's bounded wait runs out;
//           0 in normal operation.
//   wait_ns bound of every mbarrier wait (default kWaitLimitNs, 2 s).
struct DevCtl {
    unsigned status;
    unsigned inject;
    unsigned long long wait_ns;
};
constexpr unsigned kStatusTimeout = 5u;
constexpr unsigned kStatusRange = 6u;

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on device `dev`,
// once per device.  cudaFuncSetAttribute is idempotent, so two host threads
// that both see the flag clear only repeat the call.
template <typename Kernel>
cudaError_t smem_attr_once(Kernel kernel, int bytes, int dev, std::atomic<bool> (&done)[kMaxDevices]) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
    return e;
}

// fp32 CUDA-core path: one thread per output row, MT activation rows per block.
// Every GEMM launcher takes `bias`: NULL, or fp32 [N] added to each output
// row in the epilogue (Y = X * W^T + bias, one fused multiply-add with the
// q8 row scale).
cudaError_t launch_simt(int fmt, const float *X, const void *Wq, const void *S, const float *bias,
                        float *Y, int M, int N, int K, cudaStream_t s);

// tcgen05 path: 128 weight rows x BN activation rows per CTA, fp16 operands
// in swizzled shared memory, fp32 accumulator in TMEM.
cudaError_t launch_tc(int fmt, const float *X, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s);

// Up to kMaxGroup independent projections with the same M (1..128) in one
// launch of the same tcgen05 tile code: X [M, K] fp32, Wq/S as for
// rt_qgemm_q4 (fmt 4) or rt_qgemm_q8 (fmt 8), Y [M, N] fp32; K a multiple of
// 64.  Arguments are validated by the caller.
constexpr int kMaxGroup = 4;
struct GroupProblem {
    const float *X;
    const void *Wq;
    const void *S;
    const float *bias;
    float *Y;
    int N, K, fmt;
};
cudaError_t launch_tc_group(const GroupProblem *probs, int count, int M, DevCtl *ctl,
                            cudaStream_t s);

// Activation pre-pass of the TMA-fed kernels (prep.cu): X fp32 [M, K] ->
// fp16 [M, K] in the operand chunk order, into Xh (M * K * 2 bytes); latches
// kStatusRange for an activation fp16 cannot hold.  launch_cvt_x16_group
// rounds up to kMaxGroup such tensors (each M x K[i], K[i] a multiple of 8)
// in one launch.  launch_cvt_x16_lean: the same rounding as one 128-thread
// block per SM of at most 64 registers a thread (one warp per sub-partition),
// which fits beside a CTA of the activation-resident kernel, for an input
// rounded on a second stream while that kernel runs (no programmatic
// dependent launch).
cudaError_t launch_cvt_x16(const float *X, void *Xh, int64_t M, int64_t K, DevCtl *ctl,
                           cudaStream_t s);
cudaError_t launch_cvt_x16_lean(const float *X, void *Xh, int64_t M, int64_t K, DevCtl *ctl,
                                cudaStream_t s);
// The lean pre-pass's block: threads and registers a thread; false if the
// runtime cannot report them.
bool cvt_x16_lean_shape(int *threads, int *regs);
cudaError_t launch_cvt_x16_group(const float *const *X, void *const *Xh, const int64_t *K,
                                 int count, int64_t M, DevCtl *ctl, cudaStream_t s);

// tcgen05, activation block resident in shared memory, TMA-streamed weights
// (K a multiple of 128 up to 512, many activation rows); see xs.cu.  Xh is the
// pre-pass output.  launch_xs_group runs up to kMaxGroup such products with
// the same M in one persistent launch (xs_group_supported: the lists it
// takes: K a multiple of 128 up to 512, q4 scales 16-byte aligned).
struct XsInput {
    int fmt;
    const void *Xh;
    const void *Wq;
    const void *S;
    const float *bias;
    float *Y;
    int N, K;
};
bool xs_supported(int M, int N, int K);
bool xs_group_supported(const XsInput *in, int count, int M);
// Whether a block of `threads` threads of `regs` registers and no shared
// memory fits on an SM beside one CTA of the build launch_xs_group runs for
// this list (per sub-partition registers, shared memory, threads).
bool xs_group_leaves_room(const XsInput *in, int count, int M, int threads, int regs);
cudaError_t launch_xs(int fmt, const void *Xh, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s);
cudaError_t launch_xs_group(const XsInput *in, int count, int M, DevCtl *ctl, cudaStream_t s);

// The same activation-resident product on CTA pairs (cta_group::2, 256 weight
// rows per MMA), rounding fp32 X to fp16 inside the kernel; see xp.cu.  Same
// shapes as launch_xs; the plan takes it from kXpMinM activation rows up:
// measured against the pre-pass + launch_xs, it ties at M = 8192 to 16384
// and is 4 to 20 % faster at M = 32768 and 65536, while at M = 4096 the
// rounding of each CTA's first activation block costs more than the
// pre-pass saves.
constexpr int kXpMinM = 16384;

// Clusters of two CTAs of `kernel` (with this launch's block and shared
// memory) that the device can hold at once.  Pairs must sit on two SMs of one
// GPC, so the count can be below SMs / 2; a persistent grid larger than it
// would run its last clusters as a second wave.  Cached per device.
template <typename Kernel>
int resident_pairs(Kernel kernel, const cudaLaunchConfig_t &cfg, int dev,
                   std::atomic<int> (&cache)[kMaxDevices]) {
    if (dev < 0 || dev >= kMaxDevices) return 1;
    int n = cache[dev].load(std::memory_order_acquire);
    if (n > 0) return n;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(2 * (sms / 2), 1, 1);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    q.attrs = attr;
    q.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, kernel, &q) != cudaSuccess || c < 1) {
        cudaGetLastError();
        c = sms / 2;
    }
    cache[dev].store(c, std::memory_order_release);
    return c;
}

cudaError_t launch_xp(int fmt, const float *X, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s);

// tcgen05, persistent weight-stationary tiles with both operands TMA-staged
// (more than 128 activation rows, any K of the format's TMA granule); see ws.cu.
bool ws_supported(int fmt, int M, int N, int K);
// Activation rows per weight-streamed tile for this shape and SM count.
int ws_tile_rows(int M, int N, int sms);
// x_ready: Xh was complete before this launch (a pre-pass on another stream,
// joined by an event), so the activation loads need not wait for the previous
// grid in the stream; the grid still completes only after that grid has.
cudaError_t launch_ws(int fmt, const void *Xh, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s,
                      bool x_ready = false);

// tcgen05, a list of independent projections with the same M (1..128) in
// persistent launches that stream every projection's weights back to back;
// see pl.cu.  pl_supported: the shapes it takes; pl_workspace_bytes: bytes of
// the fp16 activation images (one per distinct (X, K)); launch_pl_batch runs
// the image pre-pass and the list launches.  Arguments are validated by the
// caller.
struct PlInput {
    int fmt;
    const float *X;
    const void *Wq;
    const void *S;
    const float *bias;
    float *Y;
    int N, K;
};
bool pl_supported(int fmt, int M, int64_t N, int K);
size_t pl_workspace_bytes(const PlInput *in, int count, int M);
cudaError_t launch_pl_batch(const PlInput *in, int count, int M, void *ws, DevCtl *ctl,
                            cudaStream_t s);

// dequantization exports (same __device__ routines as the GEMMs)
cudaError_t launch_dequant_q4_f32(const uint8_t *Wq, const uint16_t *SM, float *W, int N, int K,
                                  cudaStream_t s);
cudaError_t launch_dequant_q4_f16(const uint8_t *Wq, const uint16_t *SM, uint16_t *W, int N,
                                  int K, cudaStream_t s);
cudaError_t launch_dequant_q8_f32(const int8_t *Wq, const float *S, float *W, int N, int K,
                                  cudaStream_t s);
cudaError_t launch_dequant_e4m3(const uint8_t *Wq, void *W, int N, int K, bool f16,
                                cudaStream_t s);

// Argument checks of rt_qgemm_q4 / rt_qgemm_q8 / rt_gemm_e4m3 (fmt 4 / 8 / 3;
// S is unused and may be null for e4m3) and the control block of the current
// device (api.cu).
rt_status check_gemm_args(int fmt, const float *X, const void *Wq, const void *S, const float *Y,
                          int64_t M, int64_t N, int64_t K);
rt_status device_ctl(DevCtl **out);
// rt_qgemm_plan's kernel for this call's scale pointer: q4 scales that are
// not 16-byte aligned move a TMA-fed plan to the weight-stationary kernel.
int plan_with_scales(int fmt, int64_t M, int64_t N, int64_t K, int path, const void *S);

// Largest M the SIMT path takes under RT_PATH_AUTO, per format: where a
// single call of the fp32 SIMT kernel beats the tensor-core kernels in the M
// sweep of the q4 512->2048 and q8 2048->512 projections (weights rotated
// beyond L2): q4 up to M = 16 (ahead by 7 % at M = 8, level at 16), q8 and
// e4m3 only at M = 1 (the tensor-core kernel is ahead from M = 2).
constexpr int auto_simt_max_m(int fmt) { return fmt == kFmtQ4 ? 16 : 1; }

}  // namespace rtq
