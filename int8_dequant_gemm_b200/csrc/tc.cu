// tcgen05 tensor-core path (sm_100a).
//
// The product is computed weight-stationary and transposed:
//   D[o, m] = sum_k  W_hat[o, k] * X[m, k]       (D = Y^T tile)
// with the 128 weight rows of a tile as the MMA's M dimension and BN activation
// rows (16 <= BN <= 256, a multiple of 16) as its N dimension, so a small batch
// such as M = 80 fills one MMA column tile and the 128-row weight tile keeps
// the instruction at full height.  The fp32 accumulator lives in TMEM: lane i
// holds weight row o0 + i, column j holds activation row m0 + j.
//
// Operands are fp16 by default (q4 weights rounded once from their fp32
// value, q8 codes exact, activations rounded to nearest-even) or bf16 on
// request; both use tcgen05.mma kind::f16 at the same rate.  fp16 keeps 11
// significant bits against bf16's 8, at the price of the fp16 range
// (|X| <= 65504).
//
// One CTA = 8 converter warps + 1 MMA warp.  Per 64-wide K step the converter
// warps
//   - read the packed weight slice (q4: 32 B of codes + one (scale, min) word
//     per group and row; q8: 64 B of codes per row), dequantize it in
//     registers and store 16-bit operands into the A stage,
//   - read the fp32 activation slice, round it to the operand type and store it
//     into the B stage,
// both in the K-major 128-byte-swizzle layout the MMA descriptors describe,
// then fence the generic->async proxy and arrive on the stage's `full`
// mbarrier.  One thread of the MMA warp waits on `full`, issues four
// tcgen05.mma (K = 16 each) and commits to the stage's `empty` mbarrier, which
// hands the stage back to the converters once the tensor core has read it.
// After the last K step a final commit releases the epilogue: the converter
// warps read TMEM (32x32b loads, one weight row per thread), apply the q8 row
// scale in fp32 and store fp32 Y with 128-byte coalesced rows.
//
// Every mbarrier wait is bounded; a wait that gives up latches
// RT_ERR_DEVICE_TIMEOUT in the device status word and the CTA winds down.
#include <algorithm>

#include "dequant.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rtq {
namespace {

constexpr int kTileO = 128;                      // weight rows per tile (MMA M)
constexpr int kTileK = 64;                       // K per stage: one 128-byte bf16 row
constexpr int kConvWarps = 8;
constexpr int kConvThreads = kConvWarps * 32;    // 256
constexpr int kTcThreads = kConvThreads + 32;    // + MMA warp
constexpr int kAStageBytes = kTileO * 128;       // 16 KB
constexpr int kMaxSmem = 227 * 1024;
constexpr unsigned kStatusTimeout = 5u;          // RT_ERR_DEVICE_TIMEOUT

__host__ __device__ inline int tc_stage_bytes(int bn) { return kAStageBytes + bn * 128; }

__host__ __device__ inline int tc_smem_bytes(int bn, int stages) {
    return 1024 + stages * tc_stage_bytes(bn) + (2 * stages + 1) * 8 + 16;
}

__host__ __device__ inline uint32_t tmem_cols_for(int bn) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(bn)) c <<= 1;
    return c;
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// A stage, q4: thread t handles row t/2 and group (t&1) of the 64-wide slice.
template <Op16 OP>
__device__ __forceinline__ void fill_a_q4(uint32_t sA, const uint8_t *__restrict__ Wq,
                                          const uint32_t *__restrict__ SM, int o0, int k0, int N,
                                          int K, int t) {
    const int r = t >> 1, g = t & 1;
    const int o = o0 + r;
    uint4 p = make_uint4(0, 0, 0, 0);
    float sc = 0.f, mn = 0.f;
    if (o < N) {
        p = ldg_nc_v4(Wq + static_cast<size_t>(o) * (K / 2) + k0 / 2 + g * 16);
        q4_scale_min(ldg_nc_u32(SM + static_cast<size_t>(o) * (K / 32) + k0 / 32 + g), sc, mn);
    }
    sts_v4(sA + swz(r, 4 * g + 0), q4_word_op<OP>(p.x, sc, mn));
    sts_v4(sA + swz(r, 4 * g + 1), q4_word_op<OP>(p.y, sc, mn));
    sts_v4(sA + swz(r, 4 * g + 2), q4_word_op<OP>(p.z, sc, mn));
    sts_v4(sA + swz(r, 4 * g + 3), q4_word_op<OP>(p.w, sc, mn));
}

// A stage, q8: thread t handles row t/2 and 32-byte half (t&1) of the slice.
// Codes go in as exact 16-bit integers; the row scale is applied after the MMA.
template <Op16 OP>
__device__ __forceinline__ void fill_a_q8(uint32_t sA, const int8_t *__restrict__ Wq, int o0,
                                          int k0, int N, int K, int t) {
    const int r = t >> 1, h = t & 1;
    const int o = o0 + r;
    uint4 p0 = make_uint4(0, 0, 0, 0), p1 = make_uint4(0, 0, 0, 0);
    if (o < N) {
        const int8_t *src = Wq + static_cast<size_t>(o) * K + k0 + h * 32;
        p0 = ldg_nc_v4(src);
        p1 = ldg_nc_v4(src + 16);
    }
    sts_v4(sA + swz(r, 4 * h + 0), q8_words_op<OP>(p0.x, p0.y));
    sts_v4(sA + swz(r, 4 * h + 1), q8_words_op<OP>(p0.z, p0.w));
    sts_v4(sA + swz(r, 4 * h + 2), q8_words_op<OP>(p1.x, p1.y));
    sts_v4(sA + swz(r, 4 * h + 3), q8_words_op<OP>(p1.z, p1.w));
}

// B stage: BN activation rows x 64 fp32 -> 16-bit, 8 values (one chunk) per unit.
template <Op16 OP>
__device__ __forceinline__ void fill_b(uint32_t sB, const float *__restrict__ X, int m0, int k0,
                                       int M, int K, int BN, int t) {
    const int units = BN * 8;
#pragma unroll 4
    for (int u = t; u < units; u += kConvThreads) {
        const int r = u >> 3, c = u & 7;
        const int m = m0 + r;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (m < M) {
            const float *src = X + static_cast<size_t>(m) * K + k0 + c * 8;
            a = ldg_f4(src);
            b = ldg_f4(src + 4);
        }
        sts_v4(sB + swz(r, c), make_uint4(pack2<OP>(a.x, a.y), pack2<OP>(a.z, a.w),
                                          pack2<OP>(b.x, b.y), pack2<OP>(b.z, b.w)));
    }
}

template <int FMT, Op16 OP>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_qgemm_kernel(const float *__restrict__ X, const void *__restrict__ Wq,
                    const void *__restrict__ S, float *__restrict__ Y, int M, int N, int K,
                    int BN, int stages, unsigned *status) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw);
    const int stage_bytes = tc_stage_bytes(BN);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + stages * stage_bytes);
    uint64_t *empty = full + stages;
    uint64_t *done = empty + stages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    const uint32_t tmem_cols = tmem_cols_for(BN);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int o0 = blockIdx.x * kTileO;
    const int m0 = blockIdx.y * BN;
    const int nk = K / kTileK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], kConvThreads);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    pdl_wait_prior_grid();

    if (warp < kConvWarps) {
        const int t = threadIdx.x;
        for (int ks = 0; ks < nk && ok; ++ks) {
            const int s = ks % stages;
            if (ks >= stages && !mbar_wait(&empty[s], static_cast<uint32_t>((ks / stages) - 1) & 1u)) {
                ok = false;
                break;
            }
            const uint32_t sA = base + s * stage_bytes;
            const uint32_t sB = sA + kAStageBytes;
            if (FMT == 4)
                fill_a_q4<OP>(sA, static_cast<const uint8_t *>(Wq), static_cast<const uint32_t *>(S),
                          o0, ks * kTileK, N, K, t);
            else
                fill_a_q8<OP>(sA, static_cast<const int8_t *>(Wq), o0, ks * kTileK, N, K, t);
            fill_b<OP>(sB, X, m0, ks * kTileK, M, K, BN, t);
            fence_proxy_async_smem();
            mbar_arrive(&full[s]);
        }
        pdl_launch_dependents();
        // ---------------------------------------------------------- epilogue
        if (ok) ok = mbar_wait(done, 0);
        // tcgen05.ld is warp-collective: the whole warp takes the epilogue or none of it
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after_sync();
            const int q = warp & 3;            // TMEM lane quadrant of this warp
            const int half = warp >> 2;        // which half of the columns
            const int row = q * 32 + lane;
            const int o = o0 + row;
            float sc = 1.f;
            if (FMT == 8 && o < N) sc = __ldg(static_cast<const float *>(S) + o);
            const int ncol = BN / 2;
            const int c0 = half * ncol;
            for (int c = c0; c < c0 + ncol; c += 8) {
                uint32_t v[8];
                tmem_ld_x8(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c), v);
                tmem_ld_wait();
                if (o < N) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int m = m0 + c + j;
                        if (m < M) Y[static_cast<size_t>(m) * N + o] = __uint_as_float(v[j]) * sc;
                    }
                }
            }
        }
    } else if (lane == 0) {
        // -------------------------------------------------------- MMA issuer
        const uint32_t idesc = idesc_f16kind_f32acc(kTileO, BN, static_cast<uint32_t>(OP));
        for (int ks = 0; ks < nk; ++ks) {
            const int s = ks % stages;
            if (!mbar_wait(&full[s], static_cast<uint32_t>(ks / stages) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t sA = base + s * stage_bytes;
            const uint32_t sB = sA + kAStageBytes;
            const uint64_t adesc = sw128_kmajor_desc(sA);
            const uint64_t bdesc = sw128_kmajor_desc(sB);
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
                // +32 bytes per 16-element K step -> +2 in the 16-byte address field
                tc_mma_f16kind(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                            (ks > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&empty[s]);
        }
        if (ok) tc_commit(done);
    }
    __syncwarp();
    if (!ok) atomicOr(status, 1u << kStatusTimeout);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, tmem_cols);
    }
}

template <int FMT, Op16 OP>
cudaError_t launch_tc(const float *X, const void *Wq, const void *S, float *Y, int M, int N,
                      int K, unsigned *status, cudaStream_t st) {
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(tc_qgemm_kernel<FMT, OP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxSmem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int BN = M <= 256 ? std::max(16, (M + 15) / 16 * 16) : 256;
    const int nk = K / kTileK;
    int stages = (kMaxSmem - 1024 - 256) / tc_stage_bytes(BN);
    stages = std::max(1, std::min({stages, 6, nk}));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((N + kTileO - 1) / kTileO, (M + BN - 1) / BN, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = tc_smem_bytes(BN, stages);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tc_qgemm_kernel<FMT, OP>, X, Wq, S, Y, M, N, K, BN, stages,
                              status);
}

}  // namespace

cudaError_t launch_tc_q4(const float *X, const uint8_t *Wq, const uint16_t *SM, float *Y, int M,
                         int N, int K, bool bf16, unsigned *status, cudaStream_t s) {
    return bf16 ? launch_tc<4, Op16::bf16>(X, Wq, SM, Y, M, N, K, status, s)
                : launch_tc<4, Op16::f16>(X, Wq, SM, Y, M, N, K, status, s);
}

cudaError_t launch_tc_q8(const float *X, const int8_t *Wq, const float *S, float *Y, int M, int N,
                         int K, bool bf16, unsigned *status, cudaStream_t s) {
    return bf16 ? launch_tc<8, Op16::bf16>(X, Wq, S, Y, M, N, K, status, s)
                : launch_tc<8, Op16::f16>(X, Wq, S, Y, M, N, K, status, s);
}

}  // namespace rtq
