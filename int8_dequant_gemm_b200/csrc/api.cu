// C ABI of the library (declared in include/rtq.h): argument validation, the
// M-based choice between the SIMT and tensor-core kernels, the per-block
// projection driver and the per-device control block (status bits, the wait
// bound and the fault-injection test hook).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/rtq.h"
#include "kernels.cuh"
#include "ptx.cuh"

// The control block every tensor-core kernel reads (see rtq::DevCtl).
__device__ rtq::DevCtl g_rtq_ctl = {0u, 0u, rtq::kWaitLimitNs};

namespace {

using rtq::DevCtl;
using rtq::kMaxDevices;
std::mutex g_ctl_mu;
DevCtl *g_ctl_ptr[kMaxDevices] = {nullptr};

// Device address of the control block on the current device (looked up once).
rt_status ctl_block(DevCtl **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RT_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RT_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_ctl_mu);
    if (!g_ctl_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_rtq_ctl) != cudaSuccess) return RT_ERR_CUDA;
        g_ctl_ptr[dev] = static_cast<DevCtl *>(p);
    }
    *out = g_ctl_ptr[dev];
    return RT_OK;
}

// Per-(device, stream) workspace for the activation pre-pass of the TMA-fed
// kernels: M * K 16-bit values.  Grown on demand (never during stream
// capture) and kept until rt_workspace_release().
struct WorkspaceEntry {
    int dev;
    cudaStream_t stream;
    void *ptr;
    size_t bytes;
};
std::mutex g_ws_mu;
std::vector<WorkspaceEntry> g_ws;

rt_status workspace(cudaStream_t s, size_t need, void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    WorkspaceEntry *e = nullptr;
    for (auto &w : g_ws)
        if (w.dev == dev && w.stream == s) e = &w;
    if (e && e->bytes >= need) {
        *out = e->ptr;
        return RT_OK;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return RT_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return RT_ERR_WORKSPACE;
    const size_t gran = size_t(2) << 20;
    const size_t bytes = (need + gran - 1) / gran * gran;
    if (e) {
        // the old buffer may still be read by queued work on this stream
        if (cudaStreamSynchronize(s) != cudaSuccess || cudaFree(e->ptr) != cudaSuccess)
            return RT_ERR_CUDA;
        e->ptr = nullptr;
        e->bytes = 0;
    }
    void *p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return RT_ERR_CUDA;
    if (e) {
        e->ptr = p;
        e->bytes = bytes;
    } else {
        g_ws.push_back({dev, s, p, bytes});
    }
    *out = p;
    return RT_OK;
}

// A second stream and two events per (device, stream), on which pre-passes
// run beside the stream's own launches (run_list).  Created on first need
// outside any stream capture, kept until rt_workspace_release().
struct SideStream {
    cudaStream_t stream;
    cudaEvent_t fork, join;
};
struct SideEntry {
    int dev;
    cudaStream_t owner;
    SideStream side;
};
std::vector<SideEntry> g_side;   // guarded by g_ws_mu

// The side stream of `s`; false if it does not exist and cannot be created
// now (inside a capture, or a creation failed).
bool side_stream(cudaStream_t s, SideStream *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (const SideEntry &e : g_side)
        if (e.dev == dev && e.owner == s) {
            *out = e.side;
            return true;
        }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone)
        return false;
    SideStream n = {};
    if (cudaStreamCreateWithFlags(&n.stream, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming) != cudaSuccess) {
        cudaStreamDestroy(n.stream);
        return false;
    }
    if (cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming) != cudaSuccess) {
        cudaEventDestroy(n.fork);
        cudaStreamDestroy(n.stream);
        return false;
    }
    g_side.push_back({dev, s, n});
    *out = n;
    return true;
}

inline bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline bool overlap(const void *a, int64_t abytes, const void *b, int64_t bbytes) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

// Validation shared by the formats.  wbytes/sbytes: sizes of the payload and
// the scale tensor (sbytes 0: the format has none and S is not read);
// salign: the scales' required alignment.
rt_status validate(const float *X, const void *Wq, const void *S, const float *Y, int64_t M,
                   int64_t N, int64_t K, int64_t wbytes, int64_t sbytes, uintptr_t salign,
                   int64_t k_granule) {
    if (M < 0 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
        return RT_ERR_INVALID_ARG;
    if (K % k_granule != 0) return RT_ERR_UNSUPPORTED_SHAPE;
    if (!Wq || (sbytes > 0 && !S)) return RT_ERR_INVALID_ARG;
    if (M > 0 && (!X || !Y)) return RT_ERR_INVALID_ARG;
    if (!aligned(Wq, 16) || (sbytes > 0 && !aligned(S, salign))) return RT_ERR_ALIGNMENT;
    if (M > 0 && (!aligned(X, 16) || !aligned(Y, 16))) return RT_ERR_ALIGNMENT;
    if (M > 0) {
        const int64_t ybytes = M * N * 4;
        if (overlap(Y, ybytes, X, M * K * 4) || overlap(Y, ybytes, Wq, wbytes) ||
            (sbytes > 0 && overlap(Y, ybytes, S, sbytes)))
            return RT_ERR_INVALID_ARG;
    }
    return RT_OK;
}

// The optional fp32 bias of a GEMM: 4-byte aligned, not overlapping Y.
rt_status check_bias(const float *bias, const float *Y, int64_t M, int64_t N) {
    if (!bias) return RT_OK;
    if (!aligned(bias, 4)) return RT_ERR_ALIGNMENT;
    if (M > 0 && overlap(Y, M * N * 4, bias, N * 4)) return RT_ERR_INVALID_ARG;
    return RT_OK;
}

// Bytes of the packed codes and of the scales of an N x K weight.
int64_t code_bytes(int fmt, int64_t N, int64_t K) { return fmt == 4 ? N * (K / 2) : N * K; }
int64_t scale_bytes(int fmt, int64_t N, int64_t K) {
    return fmt == 4 ? N * (K / 32) * 4 : (fmt == 8 ? N * 4 : 0);
}

int pick_kernel(int fmt, int64_t M, int64_t N, int64_t K, int p) {
    if (p == RT_PATH_SIMT) return RT_KERNEL_SIMT;
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    if (rtq::xs_supported(m, n, k))
        return m >= rtq::kXpMinM ? RT_KERNEL_TC_X_RESIDENT_PAIR : RT_KERNEL_TC_X_RESIDENT;
    if (rtq::ws_supported(fmt, m, n, k)) return RT_KERNEL_TC_W_STREAMED;
    return RT_KERNEL_TC_W_STATIONARY;
}

// The TMA-fed kernels read q4 (scale, min) rows through a tensor map, whose
// base must be 16-byte aligned; a q4 call whose scales are only 4-byte
// aligned runs on the weight-stationary kernel instead (any M).
int kernel_for_scales(int kern, int fmt, const void *S) {
    const bool tma = kern == RT_KERNEL_TC_X_RESIDENT || kern == RT_KERNEL_TC_W_STREAMED ||
                     kern == RT_KERNEL_TC_X_RESIDENT_PAIR;
    return (tma && fmt == 4 && !aligned(S, 16)) ? RT_KERNEL_TC_W_STATIONARY : kern;
}

int pick_path(int fmt, int64_t M, int64_t K, int path) {
    const bool tc_ok = (K % 64) == 0;
    if (path == RT_PATH_TC) return tc_ok ? path : -1;
    if (path == RT_PATH_SIMT) return RT_PATH_SIMT;
    if (path != RT_PATH_AUTO) return -2;
    return (M <= rtq::auto_simt_max_m(fmt) || !tc_ok) ? RT_PATH_SIMT : RT_PATH_TC;
}

inline rt_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RT_OK : RT_ERR_CUDA; }

// Runs a validated GEMM on the kernel the plan picks.
rt_status run_gemm(int fmt, const float *X, const void *Wq, const void *S, const float *bias,
                   float *Y, int64_t M,
                   int64_t N, int64_t K, int path, void *stream) {
    const int p = pick_path(fmt, M, K, path);
    if (p == -1) return RT_ERR_UNSUPPORTED_SHAPE;
    if (p < 0) return RT_ERR_INVALID_ARG;
    if (M == 0) return RT_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    const int kern = kernel_for_scales(pick_kernel(fmt, M, N, K, p), fmt, S);
    if (kern == RT_KERNEL_SIMT) return from_cuda(rtq::launch_simt(fmt, X, Wq, S, bias, Y, m, n, k, s));
    DevCtl *ctl = nullptr;
    rt_status st = ctl_block(&ctl);
    if (st != RT_OK) return st;
    if (kern == RT_KERNEL_TC_W_STATIONARY)
        return from_cuda(rtq::launch_tc(fmt, X, Wq, S, bias, Y, m, n, k, ctl, s));
    if (kern == RT_KERNEL_TC_X_RESIDENT_PAIR)
        return from_cuda(rtq::launch_xp(fmt, X, Wq, S, bias, Y, m, n, k, ctl, s));
    void *xh = nullptr;
    if ((st = workspace(s, static_cast<size_t>(M) * K * 2, &xh)) != RT_OK) return st;
    cudaError_t e = rtq::launch_cvt_x16(X, xh, M, K, ctl, s);
    if (e != cudaSuccess) return RT_ERR_CUDA;
    if (kern == RT_KERNEL_TC_X_RESIDENT)
        return from_cuda(rtq::launch_xs(fmt, xh, Wq, S, bias, Y, m, n, k, ctl, s));
    return from_cuda(rtq::launch_ws(fmt, xh, Wq, S, bias, Y, m, n, k, ctl, s));
}

}  // namespace

namespace rtq {

// The checks rt_qgemm_q4 (fmt 4), rt_qgemm_q8 (fmt 8) and rt_gemm_e4m3
// (fmt 3) apply; also used by the fixed-scratch entry point in noalloc.cu.
rt_status check_gemm_args(int fmt, const float *X, const void *Wq, const void *S, const float *Y,
                          int64_t M, int64_t N, int64_t K) {
    if (!rtq::fmt_valid(fmt)) return RT_ERR_INVALID_ARG;
    return validate(X, Wq, S, Y, M, N, K, code_bytes(fmt, N, K), scale_bytes(fmt, N, K), 4,
                    fmt == 4 ? 32 : 16);
}

rt_status device_ctl(DevCtl **out) { return ctl_block(out); }

int plan_with_scales(int fmt, int64_t M, int64_t N, int64_t K, int path, const void *S) {
    const int kern = rt_qgemm_plan(fmt, M, N, K, path);
    return kern < 0 ? kern : kernel_for_scales(kern, fmt, S);
}

}  // namespace rtq

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
        case RT_ERR_WORKSPACE: return "workspace must grow during stream capture";
        case RT_ERR_SCRATCH_LIMIT: return "problem needs more than the fixed scratch array holds";
        case RT_ERR_OPERAND_RANGE: return "an activation is not a finite fp16 value";
        case RT_ERR_UNSUPPORTED_DEVICE: return "device index beyond the library's limit";
        case RT_ERR_IO: return "file cannot be opened or mapped";
        case RT_ERR_FORMAT: return "malformed checkpoint file or tensor";
        case RT_ERR_NOT_FOUND: return "no tensor of that name";
        default: return "unknown status";
    }
}

int rt_version(void) { return 200; }

int rt_qgemm_auto_path(int fmt, int64_t M, int64_t N, int64_t K) {
    if (!rtq::fmt_valid(fmt) || M < 0 || N < 1 || K < 1) return -1;
    if (K % (fmt == 4 ? 32 : 16) != 0) return -1;
    return pick_path(fmt, M, K, RT_PATH_AUTO);
}

int rt_qgemm_plan(int fmt, int64_t M, int64_t N, int64_t K, int path) {
    if (!rtq::fmt_valid(fmt) || M < 0 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim ||
        K > kMaxDim)
        return -1;
    if (K % (fmt == 4 ? 32 : 16) != 0) return -1;
    const int p = pick_path(fmt, M, K, path);
    if (p < 0) return -1;
    return pick_kernel(fmt, M, N, K, p);
}

rt_status rt_qgemm_q4(const float *X, const uint8_t *Wq, const uint16_t *scale_min, float *Y,
                      int64_t M, int64_t N, int64_t K, int path, void *stream) {
    rt_status st = validate(X, Wq, scale_min, Y, M, N, K, N * (K / 2), N * (K / 32) * 4, 4, 32);
    if (st != RT_OK) return st;
    return run_gemm(4, X, Wq, scale_min, nullptr, Y, M, N, K, path, stream);
}

rt_status rt_qgemm_q8(const float *X, const int8_t *Wq, const float *scale, float *Y, int64_t M,
                      int64_t N, int64_t K, int path, void *stream) {
    rt_status st = validate(X, Wq, scale, Y, M, N, K, N * K, N * 4, 4, 16);
    if (st != RT_OK) return st;
    return run_gemm(8, X, Wq, scale, nullptr, Y, M, N, K, path, stream);
}

rt_status rt_qgemm(int fmt, const float *X, const void *Wq, const void *scales, const float *bias,
                   float *Y, int64_t M, int64_t N, int64_t K, int path, void *stream) {
    rt_status st = rtq::check_gemm_args(fmt, X, Wq, scales, Y, M, N, K);
    if (st == RT_OK) st = check_bias(bias, Y, M, N);
    if (st != RT_OK) return st;
    return run_gemm(fmt, X, Wq, scales, bias, Y, M, N, K, path, stream);
}

rt_status rt_gemm_e4m3(const float *X, const uint8_t *W, float *Y, int64_t M, int64_t N,
                       int64_t K, int path, void *stream) {
    rt_status st = rtq::check_gemm_args(rtq::kFmtE4M3, X, W, nullptr, Y, M, N, K);
    if (st != RT_OK) return st;
    return run_gemm(rtq::kFmtE4M3, X, W, nullptr, nullptr, Y, M, N, K, path, stream);
}

int64_t rt_workspace_bytes(int fmt, int64_t M, int64_t N, int64_t K, int path) {
    const int kern = rt_qgemm_plan(fmt, M, N, K, path);
    if (kern < 0) return -1;
    if (kern == RT_KERNEL_TC_X_RESIDENT || kern == RT_KERNEL_TC_W_STREAMED) return M * K * 2;
    return 0;
}

rt_status rt_workspace_reserve(int64_t bytes, void *stream) {
    if (bytes < 0) return RT_ERR_INVALID_ARG;
    void *p = nullptr;
    return workspace(static_cast<cudaStream_t>(stream), static_cast<size_t>(bytes), &p);
}

rt_status rt_workspace_release(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    if (cudaDeviceSynchronize() != cudaSuccess) return RT_ERR_CUDA;
    for (auto it = g_ws.begin(); it != g_ws.end();) {
        if (it->dev == dev) {
            cudaFree(it->ptr);
            it = g_ws.erase(it);
        } else {
            ++it;
        }
    }
    for (auto it = g_side.begin(); it != g_side.end();) {
        if (it->dev == dev) {
            cudaEventDestroy(it->side.fork);
            cudaEventDestroy(it->side.join);
            cudaStreamDestroy(it->side.stream);
            it = g_side.erase(it);
        } else {
            ++it;
        }
    }
    return RT_OK;
}

}  // extern "C"

namespace {

// One projection of a block: format, activations, packed weights, output.
struct BlockProj {
    int fmt;
    const float *X;
    const void *W, *S;
    const float *bias;
    float *Y;
    int64_t N, K;
};

// Runs validated projections with the same M on `stream`.  Those that take
// the one-CTA activation-resident kernel run, in list order, in launches of
// up to kMaxGroup of them (a chunk of one runs as a plain call): one pre-pass
// launch rounds the chunk's activations into slices of the workspace, then
// one launch of the kernel walks all of the chunk's tiles, so the chunk
// shares one pipeline fill and drain and one wave tail.  The others run one
// call each.  When a chunk runs beside calls that stage their activations
// too (the weight-streamed kernel), those calls' pre-passes run on the
// stream's second stream while the first chunk computes (in blocks that fit
// beside its CTAs), each into a slice of its own, and the stream waits for
// them before their GEMM launches, which come after the chunks.  The
// workspace is sized once, before anything is queued.
// How run_list runs a list: its chunks (list indices that share one
// activation-resident launch), the kernel of every entry, the entries outside
// the chunks that stage their activations, the workspace they need, and
// whether the lean pre-pass fits beside the first chunk's CTAs.
struct ListPlan {
    std::vector<int> chunk_of, kern_of;
    std::vector<std::vector<int>> chunks;
    std::vector<int> staged;
    int64_t chunk_need = 0, single_need = 0, staged_sum = 0;
    bool side_fits = false;
};

ListPlan plan_list(const BlockProj *p, int count, int64_t M, int path) {
    ListPlan L;
    L.chunk_of.assign(static_cast<size_t>(count), -1);
    L.kern_of.assign(static_cast<size_t>(count), 0);
    std::vector<int> open;
    auto close = [&]() {
        if (open.size() >= 2) {
            std::vector<rtq::XsInput> in;
            int64_t bytes = 0;
            for (int i : open) {
                in.push_back({p[i].fmt, nullptr, p[i].W, p[i].S, p[i].bias, p[i].Y,
                              static_cast<int>(p[i].N), static_cast<int>(p[i].K)});
                bytes += M * p[i].K * 2;
            }
            if (rtq::xs_group_supported(in.data(), static_cast<int>(in.size()),
                                        static_cast<int>(M))) {
                for (int i : open) L.chunk_of[i] = static_cast<int>(L.chunks.size());
                L.chunks.push_back(open);
                L.chunk_need = std::max(L.chunk_need, bytes);
            }
        }
        open.clear();
    };
    for (int i = 0; i < count; ++i) {
        const BlockProj &q = p[i];
        const int kern = kernel_for_scales(
            pick_kernel(q.fmt, M, q.N, q.K, pick_path(q.fmt, M, q.K, path)), q.fmt, q.S);
        L.kern_of[i] = kern;
        if (kern == RT_KERNEL_TC_X_RESIDENT) {
            open.push_back(i);
            if (static_cast<int>(open.size()) == rtq::kMaxGroup) close();
        }
    }
    close();
    // calls outside the chunks that stage their activations
    for (int i = 0; i < count; ++i) {
        if (L.chunk_of[i] >= 0) continue;
        if (L.kern_of[i] == RT_KERNEL_TC_X_RESIDENT || L.kern_of[i] == RT_KERNEL_TC_W_STREAMED) {
            L.staged.push_back(i);
            L.single_need = std::max(L.single_need, M * p[i].K * 2);
            L.staged_sum += M * p[i].K * 2;
        }
    }
    // the side stream's pre-passes must fit beside the first chunk's CTAs,
    // or they would hold SMs the chunk's persistent CTAs wait for
    if (!L.staged.empty() && !L.chunks.empty()) {
        rtq::XsInput in0[rtq::kMaxGroup];
        const std::vector<int> &c0 = L.chunks.front();
        for (size_t g = 0; g < c0.size(); ++g) {
            const BlockProj &q = p[c0[g]];
            in0[g] = {q.fmt, nullptr, q.W, q.S, q.bias, q.Y, static_cast<int>(q.N),
                      static_cast<int>(q.K)};
        }
        int lt = 0, lr = 0;
        L.side_fits = rtq::cvt_x16_lean_shape(&lt, &lr) &&
                      rtq::xs_group_leaves_room(in0, static_cast<int>(c0.size()),
                                                static_cast<int>(M), lt, lr);
    }
    return L;
}

rt_status run_list(const BlockProj *p, int count, int64_t M, int path, void *stream) {
    if (M == 0) return RT_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const ListPlan L = plan_list(p, count, M, path);
    const std::vector<int> &chunk_of = L.chunk_of, &kern_of = L.kern_of, &staged = L.staged;
    const std::vector<std::vector<int>> &chunks = L.chunks;
    const int64_t chunk_need = L.chunk_need, single_need = L.single_need;
    const int64_t staged_sum = L.staged_sum;
    rt_status st;
    if (chunks.empty()) {
        for (int i = 0; i < count; ++i) {
            const BlockProj &q = p[i];
            if ((st = run_gemm(q.fmt, q.X, q.W, q.S, q.bias, q.Y, M, q.N, q.K, path, stream)) !=
                RT_OK)
                return st;
        }
        return RT_OK;
    }
    void *ws = nullptr;
    DevCtl *ctl = nullptr;
    SideStream side = {};
    const bool overlap = L.side_fits && side_stream(s, &side);
    const int64_t need = overlap ? chunk_need + staged_sum : std::max(chunk_need, single_need);
    if ((st = workspace(s, static_cast<size_t>(need), &ws)) != RT_OK ||
        (st = ctl_block(&ctl)) != RT_OK)
        return st;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    // slices of the staged calls' activations (overlap only), after the chunks'
    std::vector<void *> slice(static_cast<size_t>(count), nullptr);
    if (overlap) {
        int64_t off = chunk_need;              // M * K * 2: multiples of 256 bytes
        for (int i : staged) {
            slice[i] = wsb + off;
            off += M * p[i].K * 2;
        }
    }
    bool forked = false;
    cudaError_t e = cudaSuccess;
    for (size_t c = 0; c < chunks.size() && e == cudaSuccess; ++c) {
        const int n = static_cast<int>(chunks[c].size());
        rtq::XsInput in[rtq::kMaxGroup];
        const float *xs[rtq::kMaxGroup];
        void *xh[rtq::kMaxGroup];
        int64_t ks[rtq::kMaxGroup];
        int64_t off = 0;
        for (int g = 0; g < n; ++g) {
            const BlockProj &q = p[chunks[c][static_cast<size_t>(g)]];
            xs[g] = q.X;
            xh[g] = wsb + off;
            ks[g] = q.K;
            in[g] = {q.fmt, xh[g], q.W, q.S, q.bias, q.Y, static_cast<int>(q.N),
                     static_cast<int>(q.K)};
            off += M * q.K * 2;
        }
        e = rtq::launch_cvt_x16_group(xs, xh, ks, n, M, ctl, s);
        if (e == cudaSuccess && overlap && !forked) {
            // the staged calls' pre-passes start once everything before this
            // point on the stream has completed, beside the chunk's GEMM
            forked = true;
            e = cudaEventRecord(side.fork, s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(side.stream, side.fork, 0);
            for (size_t k = 0; k < staged.size() && e == cudaSuccess; ++k) {
                const BlockProj &q = p[staged[k]];
                e = rtq::launch_cvt_x16_lean(q.X, slice[staged[k]], M, q.K, ctl, side.stream);
            }
            const cudaError_t e2 = cudaEventRecord(side.join, side.stream);
            if (e == cudaSuccess) e = e2;
        }
        if (e == cudaSuccess) e = rtq::launch_xs_group(in, n, static_cast<int>(M), ctl, s);
    }
    // the stream waits for the side stream's pre-passes after the chunks'
    // launches (and always, so that a capture stays whole)
    if (forked) {
        const cudaError_t e3 = cudaStreamWaitEvent(s, side.join, 0);
        if (e == cudaSuccess) e = e3;
    }
    if (e != cudaSuccess) return RT_ERR_CUDA;
    for (int i = 0; i < count; ++i) {
        const BlockProj &q = p[i];
        if (chunk_of[i] >= 0) continue;
        if (!overlap || slice[i] == nullptr) {
            if ((st = run_gemm(q.fmt, q.X, q.W, q.S, q.bias, q.Y, M, q.N, q.K, path, stream)) !=
                RT_OK)
                return st;
            continue;
        }
        const int m = static_cast<int>(M), n = static_cast<int>(q.N), k = static_cast<int>(q.K);
        e = kern_of[i] == RT_KERNEL_TC_X_RESIDENT
                ? rtq::launch_xs(q.fmt, slice[i], q.W, q.S, q.bias, q.Y, m, n, k, ctl, s)
                : rtq::launch_ws(q.fmt, slice[i], q.W, q.S, q.bias, q.Y, m, n, k, ctl, s, true);
        if (e != cudaSuccess) return RT_ERR_CUDA;
    }
    return RT_OK;
}

// 1 if the block's four projections run as one grouped launch, 0 if one call
// each, -1 if a format or size is rejected (shapes only; no pointers).
int block_route(const int fmt[4], int64_t M, int64_t d, int64_t f, int path) {
    if (d < 1 || f < 1 || d > kMaxDim / 4 || f > kMaxDim / 2) return -1;
    const int64_t NK[4][2] = {{4 * d, d}, {d, d}, {2 * f, d}, {d, f}};
    bool fused = M >= 1 && M <= 128;
    for (int i = 0; i < 4; ++i) {
        if (!rtq::fmt_valid(fmt[i])) return -1;
        const int kern = rt_qgemm_plan(fmt[i], M, NK[i][0], NK[i][1], path);
        if (kern < 0) return -1;
        fused = fused && kern == RT_KERNEL_TC_W_STATIONARY;
    }
    return fused ? 1 : 0;
}

rt_status block_run(const BlockProj p[4], int64_t M, int64_t d, int64_t f, int path,
                    void *stream) {
    // Every projection is checked before any is enqueued.
    rt_status st;
    int fmts[4];
    for (int i = 0; i < 4; ++i) {
        const BlockProj &q = p[i];
        if (!rtq::fmt_valid(q.fmt)) return RT_ERR_INVALID_ARG;
        fmts[i] = q.fmt;
        if ((st = rtq::check_gemm_args(q.fmt, q.X, q.W, q.S, q.Y, M, q.N, q.K)) != RT_OK ||
            (st = check_bias(q.bias, q.Y, M, q.N)) != RT_OK)
            return st;
        const int pp = pick_path(q.fmt, M, q.K, path);
        if (pp == -1) return RT_ERR_UNSUPPORTED_SHAPE;
        if (pp < 0) return RT_ERR_INVALID_ARG;
    }
    // The four products may run concurrently: no output may overlap another
    // projection's output or inputs.
    if (M > 0) {
        for (int i = 0; i < 4; ++i) {
            const int64_t yb = M * p[i].N * 4;
            for (int j = 0; j < 4; ++j) {
                if (j == i) continue;
                const int64_t wb = code_bytes(p[j].fmt, p[j].N, p[j].K);
                const int64_t sb = scale_bytes(p[j].fmt, p[j].N, p[j].K);
                if (overlap(p[i].Y, yb, p[j].Y, M * p[j].N * 4) ||
                    overlap(p[i].Y, yb, p[j].X, M * p[j].K * 4) || overlap(p[i].Y, yb, p[j].W, wb) ||
                    (sb > 0 && overlap(p[i].Y, yb, p[j].S, sb)) ||
                    (p[j].bias && overlap(p[i].Y, yb, p[j].bias, p[j].N * 4)))
                    return RT_ERR_INVALID_ARG;
            }
        }
    }
    if (block_route(fmts, M, d, f, path) == 1) {
        DevCtl *ctl = nullptr;
        if ((st = ctl_block(&ctl)) != RT_OK) return st;
        rtq::GroupProblem g[4];
        for (int i = 0; i < 4; ++i)
            g[i] = {p[i].X, p[i].W, p[i].S, p[i].bias, p[i].Y, static_cast<int>(p[i].N),
                    static_cast<int>(p[i].K), p[i].fmt};
        return from_cuda(rtq::launch_tc_group(g, 4, static_cast<int>(M), ctl,
                                              static_cast<cudaStream_t>(stream)));
    }
    return run_list(p, 4, M, path, stream);
}

// The int4 card's mixed recipe: qkvg and w13 in q4, wo and w2 in q8.
constexpr int kMixedFmt[4] = {4, 8, 4, 8};

// rt_qblock_route / rt_qblock_route_fmt: the route bits of a block.
int block_route_bits(const BlockProj p[4], int64_t M, int64_t d, int64_t f, int path) {
    int fmts[4];
    for (int i = 0; i < 4; ++i) fmts[i] = p[i].fmt;
    const int r = block_route(fmts, M, d, f, path);
    if (r < 0) return -1;
    if (r == 1) return RT_ROUTE_GROUPED_SMALL_M;
    if (M <= 0) return 0;
    const ListPlan L = plan_list(p, 4, M, path);
    int bits = 0;
    if (!L.chunks.empty()) bits |= RT_ROUTE_X_RESIDENT_GROUP;
    if (!L.chunks.empty() && L.side_fits) bits |= RT_ROUTE_SIDE_PREPASS;
    return bits;
}

}  // namespace

extern "C" {

int rt_qblock_fused(int64_t M, int64_t d_model, int64_t d_ff, int path) {
    return block_route(kMixedFmt, M, d_model, d_ff, path);
}

rt_status rt_qblock_project(const rt_qblock *blk, int64_t M, const float *X_qkvg,
                            const float *X_o, const float *X_ffn, const float *X_w2,
                            float *Y_qkvg, float *Y_o, float *Y_13, float *Y_2, int path,
                            void *stream) {
    if (!blk || blk->d_model < 1 || blk->d_ff < 1) return RT_ERR_INVALID_ARG;
    const int64_t d = blk->d_model, f = blk->d_ff;
    const BlockProj p[4] = {{4, X_qkvg, blk->qkvg, blk->qkvg_sm, nullptr, Y_qkvg, 4 * d, d},
                            {8, X_o, blk->wo, blk->wo_s, nullptr, Y_o, d, d},
                            {4, X_ffn, blk->w13, blk->w13_sm, nullptr, Y_13, 2 * f, d},
                            {8, X_w2, blk->w2, blk->w2_s, nullptr, Y_2, d, f}};
    return block_run(p, M, d, f, path, stream);
}

int rt_qblock_route(const rt_qblock *blk, int64_t M, int path) {
    if (!blk || blk->d_model < 1 || blk->d_ff < 1 || M < 0 || M > kMaxDim) return -1;
    const int64_t d = blk->d_model, f = blk->d_ff;
    const BlockProj p[4] = {{4, nullptr, blk->qkvg, blk->qkvg_sm, nullptr, nullptr, 4 * d, d},
                            {8, nullptr, blk->wo, blk->wo_s, nullptr, nullptr, d, d},
                            {4, nullptr, blk->w13, blk->w13_sm, nullptr, nullptr, 2 * f, d},
                            {8, nullptr, blk->w2, blk->w2_s, nullptr, nullptr, d, f}};
    return block_route_bits(p, M, d, f, path);
}

int rt_qblock_route_fmt(const rt_qblock_fmt *blk, int64_t M, int path) {
    if (!blk || blk->d_model < 1 || blk->d_ff < 1 || M < 0 || M > kMaxDim) return -1;
    const rt_qweight *w[4] = {&blk->qkvg, &blk->wo, &blk->w13, &blk->w2};
    for (int i = 0; i < 4; ++i)
        if (w[i]->reserved != 0 || !rtq::fmt_valid(w[i]->fmt)) return -1;
    const int64_t d = blk->d_model, f = blk->d_ff;
    const BlockProj p[4] = {{w[0]->fmt, nullptr, w[0]->Wq, w[0]->scales, w[0]->bias, nullptr, 4 * d, d},
                            {w[1]->fmt, nullptr, w[1]->Wq, w[1]->scales, w[1]->bias, nullptr, d, d},
                            {w[2]->fmt, nullptr, w[2]->Wq, w[2]->scales, w[2]->bias, nullptr, 2 * f, d},
                            {w[3]->fmt, nullptr, w[3]->Wq, w[3]->scales, w[3]->bias, nullptr, d, f}};
    return block_route_bits(p, M, d, f, path);
}

int rt_qblock_fused_fmt(const rt_qblock_fmt *blk, int64_t M, int path) {
    if (!blk) return -1;
    const rt_qweight *w[4] = {&blk->qkvg, &blk->wo, &blk->w13, &blk->w2};
    int fmts[4];
    for (int i = 0; i < 4; ++i) {
        if (w[i]->reserved != 0) return -1;
        fmts[i] = w[i]->fmt;
    }
    return block_route(fmts, M, blk->d_model, blk->d_ff, path);
}

rt_status rt_qblock_project_fmt(const rt_qblock_fmt *blk, int64_t M, const float *X_qkvg,
                                const float *X_o, const float *X_ffn, const float *X_w2,
                                float *Y_qkvg, float *Y_o, float *Y_13, float *Y_2, int path,
                                void *stream) {
    if (!blk || blk->d_model < 1 || blk->d_ff < 1) return RT_ERR_INVALID_ARG;
    const rt_qweight *w[4] = {&blk->qkvg, &blk->wo, &blk->w13, &blk->w2};
    for (int i = 0; i < 4; ++i)
        if (w[i]->reserved != 0) return RT_ERR_INVALID_ARG;
    const int64_t d = blk->d_model, f = blk->d_ff;
    const rt_qweight &a = blk->qkvg, &b = blk->wo, &c = blk->w13, &e = blk->w2;
    const BlockProj p[4] = {{a.fmt, X_qkvg, a.Wq, a.scales, a.bias, Y_qkvg, 4 * d, d},
                            {b.fmt, X_o, b.Wq, b.scales, b.bias, Y_o, d, d},
                            {c.fmt, X_ffn, c.Wq, c.scales, c.bias, Y_13, 2 * f, d},
                            {e.fmt, X_w2, e.Wq, e.scales, e.bias, Y_2, d, f}};
    return block_run(p, M, d, f, path, stream);
}

}  // extern "C"

// ---------------------------------------------------------------- batches
namespace {

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Checks a list and returns the route it takes: RT_KERNEL_TC_LIST, 0 for one
// call per projection, or a negative rt_status for a rejected list.
int batch_route(const rt_qproj *list, int count, int64_t M, int path) {
    if (count < 0 || (count > 0 && !list) || M < 0 || M > kMaxDim) return -RT_ERR_INVALID_ARG;
    if (path != RT_PATH_AUTO && path != RT_PATH_SIMT && path != RT_PATH_TC)
        return -RT_ERR_INVALID_ARG;
    bool tc_all = true, list_ok = M >= 1 && M <= 128;
    int64_t tiles = 0;
    for (int i = 0; i < count; ++i) {
        const rt_qproj &q = list[i];
        if (!rtq::fmt_valid(q.fmt) || q.reserved != 0) return -RT_ERR_INVALID_ARG;
        rt_status st = rtq::check_gemm_args(q.fmt, q.X, q.Wq, q.scales, q.Y, M, q.N, q.K);
        if (st == RT_OK) st = check_bias(q.bias, q.Y, M, q.N);
        if (st != RT_OK) return -st;
        const int p = pick_path(q.fmt, M, q.K, path);
        if (p == -1) return -RT_ERR_UNSUPPORTED_SHAPE;
        tc_all = tc_all && p == RT_PATH_TC;
        // the list kernel reads q4 (scale, min) rows through a TMA map: 16-byte base
        list_ok = list_ok &&
                  rtq::pl_supported(q.fmt, static_cast<int>(M), q.N, static_cast<int>(q.K)) &&
                  (q.fmt != 4 || aligned(q.scales, 16));
        tiles += (q.N + 127) / 128;
    }
    // the projections may run concurrently: no output may overlap another
    // projection's output or inputs (sorted sweep over the address ranges)
    if (M > 0 && count > 1) {
        struct Range {
            uintptr_t lo, hi;
            bool out;
        };
        std::vector<Range> r;
        r.reserve(static_cast<size_t>(count) * 4);
        for (int i = 0; i < count; ++i) {
            const rt_qproj &q = list[i];
            const int64_t wb = code_bytes(q.fmt, q.N, q.K);
            const int64_t sb = scale_bytes(q.fmt, q.N, q.K);
            auto add = [&](const void *p, int64_t n, bool out) {
                const uintptr_t a = reinterpret_cast<uintptr_t>(p);
                r.push_back({a, a + static_cast<uintptr_t>(n), out});
            };
            add(q.Y, M * q.N * 4, true);
            add(q.X, M * q.K * 4, false);
            add(q.Wq, wb, false);
            if (sb > 0) add(q.scales, sb, false);
            if (q.bias) add(q.bias, q.N * 4, false);
        }
        std::sort(r.begin(), r.end(), [](const Range &a, const Range &b) { return a.lo < b.lo; });
        // In address order, each range is checked against the furthest end
        // reached so far: an output against every earlier range, an input
        // against earlier outputs.  (Overlaps within one projection are
        // already rejected above, and inputs may share memory.)
        uintptr_t end_any = 0, end_out = 0;
        for (const Range &x : r) {
            if (x.out ? end_any > x.lo : end_out > x.lo) return -RT_ERR_INVALID_ARG;
            end_any = std::max(end_any, x.hi);
            if (x.out) end_out = std::max(end_out, x.hi);
        }
    }
    if (!tc_all || !list_ok || count == 0) return 0;
    if (path == RT_PATH_AUTO && tiles < sm_count()) return 0;
    return RT_KERNEL_TC_LIST;
}

}  // namespace

extern "C" {

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

rt_status rt_dequant_e4m3_f32(const uint8_t *Wq, float *W_out, int64_t N, int64_t K,
                              void *stream) {
    rt_status st = validate_dequant(Wq, W_out, W_out, N, K, 16, 4);
    if (st != RT_OK) return st;
    return from_cuda(rtq::launch_dequant_e4m3(Wq, W_out, static_cast<int>(N), static_cast<int>(K),
                                              false, static_cast<cudaStream_t>(stream)));
}

rt_status rt_dequant_e4m3_f16(const uint8_t *Wq, uint16_t *W_out, int64_t N, int64_t K,
                              void *stream) {
    rt_status st = validate_dequant(Wq, W_out, W_out, N, K, 16, 4);
    if (st != RT_OK) return st;
    return from_cuda(rtq::launch_dequant_e4m3(Wq, W_out, static_cast<int>(N), static_cast<int>(K),
                                              true, static_cast<cudaStream_t>(stream)));
}

rt_status rt_dequant_q4_f16(const uint8_t *Wq, const uint16_t *scale_min, uint16_t *W_out,
                            int64_t N, int64_t K, void *stream) {
    rt_status st = validate_dequant(Wq, scale_min, W_out, N, K, 32, 4);
    if (st != RT_OK) return st;
    return from_cuda(rtq::launch_dequant_q4_f16(Wq, scale_min, W_out, static_cast<int>(N),
                                                static_cast<int>(K),
                                                static_cast<cudaStream_t>(stream)));
}

int rt_qgemm_batch_plan(const rt_qproj *list, int count, int64_t M, int path) {
    const int r = batch_route(list, count, M, path);
    return r < 0 ? -1 : r;
}

rt_status rt_qgemm_batch(const rt_qproj *list, int count, int64_t M, int path, void *stream) {
    const int route = batch_route(list, count, M, path);
    if (route < 0) return static_cast<rt_status>(-route);
    if (M == 0 || count == 0) return RT_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (route != RT_KERNEL_TC_LIST) {
        std::vector<BlockProj> p(static_cast<size_t>(count));
        for (int i = 0; i < count; ++i) {
            const rt_qproj &q = list[i];
            p[i] = {q.fmt, q.X, q.Wq, q.scales, q.bias, q.Y, q.N, q.K};
        }
        return run_list(p.data(), count, M, path, stream);
    }
    DevCtl *ctl = nullptr;
    rt_status st = ctl_block(&ctl);
    if (st != RT_OK) return st;
    std::vector<rtq::PlInput> in(static_cast<size_t>(count));
    for (int i = 0; i < count; ++i) {
        const rt_qproj &q = list[i];
        in[i] = {q.fmt, q.X, q.Wq, q.scales, q.bias, q.Y, static_cast<int>(q.N),
                 static_cast<int>(q.K)};
    }
    void *ws = nullptr;
    const size_t need = rtq::pl_workspace_bytes(in.data(), count, static_cast<int>(M));
    if ((st = workspace(s, need, &ws)) != RT_OK) return st;
    return from_cuda(rtq::launch_pl_batch(in.data(), count, static_cast<int>(M), ws, ctl, s));
}

rt_status rt_device_status(void *stream, int *device_status) {
    if (!device_status) return RT_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return RT_ERR_CUDA;
    DevCtl *ctl = nullptr;
    rt_status st = ctl_block(&ctl);
    if (st != RT_OK) return st;
    unsigned v = 0;
    if (cudaMemcpy(&v, &ctl->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
        return RT_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(&ctl->status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
            return RT_ERR_CUDA;
    }
    *device_status = (v & (1u << rtq::kStatusTimeout))  ? RT_ERR_DEVICE_TIMEOUT
                     : (v & (1u << rtq::kStatusRange)) ? RT_ERR_OPERAND_RANGE
                                                       : RT_OK;
    return RT_OK;
}

rt_status rt_debug_inject(int mode, int64_t wait_ns) {
    if (mode < 0 || mode > 1 || wait_ns < 0) return RT_ERR_INVALID_ARG;
    DevCtl *ctl = nullptr;
    rt_status st = ctl_block(&ctl);
    if (st != RT_OK) return st;
    if (cudaDeviceSynchronize() != cudaSuccess) return RT_ERR_CUDA;
    const unsigned inject = static_cast<unsigned>(mode);
    const unsigned long long ns =
        wait_ns == 0 ? rtq::kWaitLimitNs : static_cast<unsigned long long>(wait_ns);
    if (cudaMemcpy(&ctl->inject, &inject, sizeof inject, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(&ctl->wait_ns, &ns, sizeof ns, cudaMemcpyHostToDevice) != cudaSuccess)
        return RT_ERR_CUDA;
    return RT_OK;
}

}  // extern "C"
