// fp32 CUDA-core kernels: the exact-rounding path (weights dequantized to
// fp32 with one rounding -- exactly, for q8 codes and e4m3 values -- fp32 FMA
// accumulation) and the automatic path at the smallest M (q4: M <= 16, q8 and
// e4m3: M = 1).
//
// Layout of work: each thread owns one output row o of W and MT activation
// rows, staged per CTA in shared memory.  Inside the K loop every lane of a
// warp reads the same activation address (a shared-memory broadcast), so
// shared memory bandwidth is not the limit; the weight stream is one 16-byte
// load per thread per step (a q4 group, or 16 q8 codes) that L1 completes to
// full sectors on the following step.
//
// One thread per row gives only N threads, too few to keep the weight stream
// in flight (N = 512 for the q8 projections), so K is split across a cluster
// of up to 8 CTAs: each stages and sums its K slice, writes its per-row
// partials to shared memory, and after a cluster barrier CTA rank r sums a
// 1/ksplit share of the (row, activation row) outputs over the cluster in rank
// order (deterministic) and stores them.
#include <algorithm>

#include "dequant.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rtq {
namespace {

constexpr int kSimtThreads = 128;                 // weight rows per CTA
constexpr int kSimtMaxSmem = 160 * 1024;          // activations (<= 128 KB) + partials

// X rows m0 .. m0 + mt - 1, columns [k0, k0 + Ks), as MT x Ks floats.
template <int MT>
__device__ __forceinline__ void stage_x(const float *__restrict__ X, float4 *xs4, int m0, int mt,
                                        int K, int k0, int Ks) {
    const int K4 = Ks / 4;
    for (int i = threadIdx.x; i < MT * K4; i += blockDim.x) {
        const int r = i / K4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < mt) v = ldg_f4(X + static_cast<size_t>(m0 + r) * K + k0 + (i - r * K4) * 4);
        xs4[i] = v;
    }
}

// Sum of the K slice [k0, k0 + Ks) of row o (valid: o < N) into acc[MT].
template <int MT, int FMT>
__device__ __forceinline__ void simt_slice(const float *xs, const void *__restrict__ Wq,
                                           const void *__restrict__ S, int o, bool valid, int K,
                                           int k0, int Ks, float (&acc)[MT]) {
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    if (!valid) return;
    if (FMT == 4) {
        const uint8_t *wrow = static_cast<const uint8_t *>(Wq) + static_cast<size_t>(o) * (K / 2);
        const uint32_t *srow = static_cast<const uint32_t *>(S) + static_cast<size_t>(o) * (K / 32);
        for (int g = 0; g < Ks / 32; ++g) {
            const int kg = k0 / 32 + g;
            const uint4 p = ldg_v4(wrow + kg * 16);
            float sc, mn;
            q4_scale_min(__ldg(srow + kg), sc, mn);
            const uint32_t words[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float w[8];
                q4_word_f32(words[c], sc, mn, w);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const float4 *xr = reinterpret_cast<const float4 *>(xs + m * Ks + g * 32 + c * 8);
                    const float4 a = xr[0], b = xr[1];
                    float t = acc[m];
                    t = fmaf(a.x, w[0], t);
                    t = fmaf(a.y, w[1], t);
                    t = fmaf(a.z, w[2], t);
                    t = fmaf(a.w, w[3], t);
                    t = fmaf(b.x, w[4], t);
                    t = fmaf(b.y, w[5], t);
                    t = fmaf(b.z, w[6], t);
                    t = fmaf(b.w, w[7], t);
                    acc[m] = t;
                }
            }
        }
    } else {
        // q8: the row scale is factored out of the K sum and applied once at
        // the end, Y = scale[o] * sum_k x * q.  e4m3: the same loop over one
        // byte per weight, values exact in fp32, no scale.
        const int8_t *wrow = static_cast<const int8_t *>(Wq) + static_cast<size_t>(o) * K + k0;
        for (int kk = 0; kk < Ks; kk += 16) {
            const uint4 p = ldg_v4(wrow + kk);
            const uint32_t words[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float w0, w1, w2, w3;
                if (FMT == kFmtE4M3) {
                    w0 = e4m3_byte_f32(words[c], 0);
                    w1 = e4m3_byte_f32(words[c], 1);
                    w2 = e4m3_byte_f32(words[c], 2);
                    w3 = e4m3_byte_f32(words[c], 3);
                } else {
                    w0 = q8_byte_f32(words[c], 0);
                    w1 = q8_byte_f32(words[c], 1);
                    w2 = q8_byte_f32(words[c], 2);
                    w3 = q8_byte_f32(words[c], 3);
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const float4 a = *reinterpret_cast<const float4 *>(xs + m * Ks + kk + c * 4);
                    float t = acc[m];
                    t = fmaf(a.x, w0, t);
                    t = fmaf(a.y, w1, t);
                    t = fmaf(a.z, w2, t);
                    t = fmaf(a.w, w3, t);
                    acc[m] = t;
                }
            }
        }
    }
}

template <int MT, int FMT>
__global__ void __launch_bounds__(kSimtThreads)
    simt_kernel(const float *__restrict__ X, const void *__restrict__ Wq,
                const void *__restrict__ S, const float *__restrict__ bias, float *__restrict__ Y,
                int M, int N, int K, int ksplit) {
    extern __shared__ float4 xs4[];
    const float *xs = reinterpret_cast<const float *>(xs4);
    const int Ks = K / ksplit;
    const int k0 = static_cast<int>(blockIdx.z) * Ks;
    const int m0 = blockIdx.x * MT;
    const int mt = min(MT, M - m0);
    const int o0 = blockIdx.y * kSimtThreads;
    const int o = o0 + threadIdx.x;
    const bool valid = o < N;
    // the weights do not depend on the previous kernel in the stream
    if (valid) {
        const int step = FMT == 4 ? 256 : 128;   // one prefetch per 128-byte line
        const char *w = static_cast<const char *>(Wq) +
                        (FMT == 4 ? static_cast<size_t>(o) * (K / 2) + k0 / 2
                                  : static_cast<size_t>(o) * K + k0);
        for (int k = 0; k < Ks; k += step) prefetch_l2(w + (FMT == 4 ? k / 2 : k));
    }
    pdl_wait_prior_grid();
    stage_x<MT>(X, xs4, m0, mt, K, k0, Ks);
    __syncthreads();
    pdl_launch_dependents();

    float acc[MT];
    simt_slice<MT, FMT>(xs, Wq, S, o, valid, K, k0, Ks, acc);
    const float sc = (FMT == 8 && valid) ? __ldg(static_cast<const float *>(S) + o) : 1.f;
    const float b = (bias && valid) ? __ldg(bias + o) : 0.f;
    if (ksplit == 1) {
        if (valid) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < mt) Y[static_cast<size_t>(m0 + m) * N + o] = fmaf(acc[m], sc, b);
        }
        return;
    }
    // split K: partials [MT][kSimtThreads] after the staged activations
    float *part = reinterpret_cast<float *>(xs4) + MT * Ks;
#pragma unroll
    for (int m = 0; m < MT; ++m) part[m * kSimtThreads + threadIdx.x] = acc[m];
    cluster_sync();                           // all partials written
    const int share = MT * kSimtThreads / ksplit;
    const int beg = static_cast<int>(cluster_ctarank()) * share;
    const uint32_t pbase = smem_addr(part);
    for (int i = threadIdx.x; i < share; i += kSimtThreads) {
        const int idx = beg + i, m = idx / kSimtThreads, row = idx % kSimtThreads;
        const uint32_t off = pbase + static_cast<uint32_t>(idx * 4);
        float v = ld_cluster_f32(cluster_map(off, 0));
        for (int r = 1; r < ksplit; ++r) v += ld_cluster_f32(cluster_map(off, static_cast<uint32_t>(r)));
        const int oo = o0 + row;
        if (m < mt && oo < N) {
            const float s8 = FMT == 8 ? __ldg(static_cast<const float *>(S) + oo) : 1.f;
            const float bb = bias ? __ldg(bias + oo) : 0.f;
            Y[static_cast<size_t>(m0 + m) * N + oo] = fmaf(v, s8, bb);
        }
    }
    cluster_sync();                           // peers are done reading this CTA's partials
}

// K slices: up to 8, while the grid stays within about four CTAs per SM and
// each slice keeps whole q4 groups (32) and 16-byte q8 loads, at least 64
// wide.
int pick_simt_ksplit(int M, int N, int K, int MT) {
    const long ctas = static_cast<long>((M + MT - 1) / MT) * ((N + kSimtThreads - 1) / kSimtThreads);
    int ks = 1;
    while (ks < 8 && K % (2 * ks * 64) == 0 && ctas * ks * 2 <= 4 * 148) ks *= 2;
    return ks;
}

template <int MT, int FMT>
cudaError_t launch_simt_mt(const float *X, const void *Wq, const void *S, const float *bias,
                           float *Y, int M, int N, int K, cudaStream_t s) {
    const int ksplit = pick_simt_ksplit(M, N, K, MT);
    const size_t smem = static_cast<size_t>(MT) * (K / ksplit) * sizeof(float) +
                        (ksplit > 1 ? static_cast<size_t>(MT) * kSimtThreads * sizeof(float) : 0);
    // The limit is raised once per device to the largest size any call asks
    // for (staged activations of at most 128 KB plus the partials), so calls
    // from several host threads never lower it under one another.
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(simt_kernel<MT, FMT>, kSimtMaxSmem, dev, attr_done)) != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((M + MT - 1) / MT, (N + kSimtThreads - 1) / kSimtThreads, ksplit);
    cfg.blockDim = dim3(kSimtThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = static_cast<unsigned>(ksplit);
    cfg.attrs = attr;
    cfg.numAttrs = ksplit > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, simt_kernel<MT, FMT>, X, Wq, S, bias, Y, M, N, K, ksplit);
}

template <int MT>
cudaError_t launch_simt_fmt(int fmt, const float *X, const void *Wq, const void *S,
                            const float *bias, float *Y, int M, int N, int K, cudaStream_t s) {
    if (fmt == kFmtQ4) return launch_simt_mt<MT, kFmtQ4>(X, Wq, S, bias, Y, M, N, K, s);
    if (fmt == kFmtQ8) return launch_simt_mt<MT, kFmtQ8>(X, Wq, S, bias, Y, M, N, K, s);
    return launch_simt_mt<MT, kFmtE4M3>(X, Wq, S, bias, Y, M, N, K, s);
}

}  // namespace

// Activation rows per block: as many as M needs up to 8, capped so the staged
// activations stay within 128 KB of shared memory.
cudaError_t launch_simt(int fmt, const float *X, const void *Wq, const void *S, const float *bias,
                        float *Y, int M, int N, int K, cudaStream_t s) {
    int mt = M >= 8 ? 8 : (M >= 4 ? 4 : (M >= 2 ? 2 : 1));
    while (mt > 1 && static_cast<size_t>(mt) * K * sizeof(float) > 128 * 1024) mt /= 2;
    switch (mt) {
        case 8: return launch_simt_fmt<8>(fmt, X, Wq, S, bias, Y, M, N, K, s);
        case 4: return launch_simt_fmt<4>(fmt, X, Wq, S, bias, Y, M, N, K, s);
        case 2: return launch_simt_fmt<2>(fmt, X, Wq, S, bias, Y, M, N, K, s);
        default: return launch_simt_fmt<1>(fmt, X, Wq, S, bias, Y, M, N, K, s);
    }
}

namespace {

// ----------------------------------------------------------- dequant exports
__global__ void dequant_q4_f32_kernel(const uint8_t *__restrict__ Wq,
                                      const uint32_t *__restrict__ SM, float *__restrict__ W,
                                      int N, int K) {
    const int G = K / 32;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(N) * G) return;
    const int64_t o = idx / G, g = idx % G;
    const uint4 p = ldg_nc_v4(Wq + o * (K / 2) + g * 16);
    float sc, mn;
    q4_scale_min(__ldg(SM + o * G + g), sc, mn);
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    float *dst = W + o * K + g * 32;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float w[8];
        q4_word_f32(words[c], sc, mn, w);
        reinterpret_cast<float4 *>(dst + c * 8)[0] = make_float4(w[0], w[1], w[2], w[3]);
        reinterpret_cast<float4 *>(dst + c * 8)[1] = make_float4(w[4], w[5], w[6], w[7]);
    }
}

__global__ void dequant_q4_f16_kernel(const uint8_t *__restrict__ Wq,
                                      const uint32_t *__restrict__ SM, uint16_t *__restrict__ W,
                                      int N, int K) {
    const int G = K / 32;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(N) * G) return;
    const int64_t o = idx / G, g = idx % G;
    const uint4 p = ldg_nc_v4(Wq + o * (K / 2) + g * 16);
    uint32_t s2, m2;
    q4_scale_min_f16x2(__ldg(SM + o * G + g), s2, m2);
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    uint4 *dst = reinterpret_cast<uint4 *>(W + o * K + g * 32);
#pragma unroll
    for (int c = 0; c < 4; ++c) dst[c] = chunk_to_natural(q4_word_f16(words[c], s2, m2));
}

__global__ void dequant_q8_f32_kernel(const int8_t *__restrict__ Wq, const float *__restrict__ S,
                                      float *__restrict__ W, int N, int K) {
    const int C = K / 16;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(N) * C) return;
    const int64_t o = idx / C, c = idx % C;
    const uint4 p = ldg_nc_v4(Wq + o * K + c * 16);
    const float sc = __ldg(S + o);
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    float *dst = W + o * K + c * 16;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        reinterpret_cast<float4 *>(dst)[j] =
            make_float4(q8_byte_f32(words[j], 0) * sc, q8_byte_f32(words[j], 1) * sc,
                        q8_byte_f32(words[j], 2) * sc, q8_byte_f32(words[j], 3) * sc);
    }
}

// e4m3 codes -> fp32 (f16 = false) or fp16 bits (f16 = true, the tensor-core
// operand), natural order, 16 codes per thread.
__global__ void dequant_e4m3_kernel(const uint8_t *__restrict__ Wq, void *__restrict__ W, int N,
                                    int K, bool f16) {
    const int C = K / 16;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(N) * C) return;
    const int64_t o = idx / C, c = idx % C;
    const uint4 p = ldg_nc_v4(Wq + o * K + c * 16);
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    if (f16) {
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(W) + o * K + c * 16);
        dst[0] = chunk_to_natural(e4m3_words_f16(words[0], words[1]));
        dst[1] = chunk_to_natural(e4m3_words_f16(words[2], words[3]));
    } else {
        float *dst = static_cast<float *>(W) + o * K + c * 16;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            reinterpret_cast<float4 *>(dst)[j] =
                make_float4(e4m3_byte_f32(words[j], 0), e4m3_byte_f32(words[j], 1),
                            e4m3_byte_f32(words[j], 2), e4m3_byte_f32(words[j], 3));
    }
}

inline unsigned blocks_for(int64_t n, int threads) {
    return static_cast<unsigned>((n + threads - 1) / threads);
}

}  // namespace

cudaError_t launch_dequant_q4_f32(const uint8_t *Wq, const uint16_t *SM, float *W, int N, int K,
                                  cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(N) * (K / 32);
    dequant_q4_f32_kernel<<<blocks_for(n, 256), 256, 0, s>>>(
        Wq, reinterpret_cast<const uint32_t *>(SM), W, N, K);
    return cudaGetLastError();
}

cudaError_t launch_dequant_q4_f16(const uint8_t *Wq, const uint16_t *SM, uint16_t *W, int N,
                                  int K, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(N) * (K / 32);
    const uint32_t *sm = reinterpret_cast<const uint32_t *>(SM);
    dequant_q4_f16_kernel<<<blocks_for(n, 256), 256, 0, s>>>(Wq, sm, W, N, K);
    return cudaGetLastError();
}

cudaError_t launch_dequant_q8_f32(const int8_t *Wq, const float *S, float *W, int N, int K,
                                  cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(N) * (K / 16);
    dequant_q8_f32_kernel<<<blocks_for(n, 256), 256, 0, s>>>(Wq, S, W, N, K);
    return cudaGetLastError();
}

cudaError_t launch_dequant_e4m3(const uint8_t *Wq, void *W, int N, int K, bool f16,
                                cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(N) * (K / 16);
    dequant_e4m3_kernel<<<blocks_for(n, 256), 256, 0, s>>>(Wq, W, N, K, f16);
    return cudaGetLastError();
}

}  // namespace rtq
