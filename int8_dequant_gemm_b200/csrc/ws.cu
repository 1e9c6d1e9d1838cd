// tcgen05 path for many activation rows and long K (K > 512): weight tile
// stationary, TMA streams both operands' raw data through a stage ring.
//
// Tile product as in tc.cu / xs.cu, D[o, m] = sum_k W_hat[o, k] * X[m, k],
// 128 weight rows (MMA M) x 128 activation rows (MMA N), full K per tile.
// A persistent CTA (one per SM) walks tiles t = blockIdx.x, + gridDim.x, ...
// in weight-tile-fastest order, so concurrently running CTAs share activation
// tiles in L2.
//
// Per 64-wide K step one stage holds
//   A: the 128 x 64 dequantized weights (written by the dequantizers from
//      TMA-staged packed codes, as in xs.cu), and
//   B: the 128 x 64 16-bit activations, one TMA box from the pre-converted
//      activations (prep.cu) in the 128-byte-swizzled operand layout.
// Roles (15 warps): warps 0-7 dequantizers (two groups of 128 threads on
// alternate K steps, thread = weight row), warp 8 MMA issuer, warps 9-12
// epilogue (double-buffered TMEM accumulators), warp 13 weight TMA (codes and,
// for q4, (scale, min) blocks of up to 16 words per row), warp 14 activation
// TMA.
//
// Every mbarrier wait is bounded; a wait that gives up latches
// RT_ERR_DEVICE_TIMEOUT in the device status word and the CTA winds down.
#include <algorithm>

#include "kernels.cuh"
#include "tmapipe.cuh"

namespace rtq {
namespace {

constexpr int kWsTileM = 128;                 // activation rows per tile (MMA N)
constexpr int kDeqGroups = 2;
constexpr int kDeqThreads = kTileRows;                   // 128 per group
constexpr int kDeqWarps = kDeqGroups * 4;                // 8
constexpr int kMmaWarp = kDeqWarps;                      // 8
constexpr int kEpiWarp0 = kMmaWarp + 1;                  // 9
constexpr int kEpiThreads = 128;
constexpr int kWTmaWarp = kEpiWarp0 + 4;                 // 13
constexpr int kXTmaWarp = kWTmaWarp + 1;                 // 14
constexpr int kWsThreads = (kXTmaWarp + 1) * 32;         // 480
constexpr int kStages = 4;
constexpr int kStageBytes = 2 * kOpStage;                // A + B, 32 KB
constexpr int kRaw = 6;
constexpr int kRawSlot = 8 * 1024;
constexpr int kScaleSlot = 8 * 1024;                     // 128 rows x 16 words
constexpr int kScaleWords = 16;                          // (scale, min) words per chunk row
constexpr int kChunkSteps = kScaleWords / 2;             // K steps covered by one chunk
constexpr uint32_t kWsTmemCols = 256;
constexpr unsigned kStatusTimeout = 5u;

struct WsLayout {
    int st_off, raw_off, sc_off, bar_off, total;
};

__host__ __device__ inline WsLayout ws_layout() {
    WsLayout L;
    L.st_off = 0;
    L.raw_off = kStages * kStageBytes;
    L.sc_off = L.raw_off + kRaw * kRawSlot;
    L.bar_off = L.sc_off + 2 * kScaleSlot;
    // a_full/b_full/st_empty[kStages], raw_full/empty[kRaw], sc_full/empty[2],
    // acc_full/empty[2], + TMEM address slot
    L.total = L.bar_off + (3 * kStages + 2 * kRaw + 4 + 4) * 8 + 16;
    return L;
}

template <int FMT, Op16 OP>
__global__ void __launch_bounds__(kWsThreads, 1)
    ws_qgemm_kernel(const __grid_constant__ CUtensorMap w_map,
                    const __grid_constant__ CUtensorMap s_map,
                    const __grid_constant__ CUtensorMap x_map, const float *__restrict__ S8,
                    float *__restrict__ Y, int M, int N, int K, int n_o_tiles, int n_tiles,
                    unsigned *status) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const WsLayout L = ws_layout();
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *a_full = bars;
    uint64_t *b_full = a_full + kStages;
    uint64_t *st_empty = b_full + kStages;
    uint64_t *raw_full = st_empty + kStages;
    uint64_t *raw_empty = raw_full + kRaw;
    uint64_t *sc_full = raw_empty + kRaw;
    uint64_t *sc_empty = sc_full + 2;
    uint64_t *acc_full = sc_empty + 2;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / kAtomK;
    const int n_chunks = (nk + kChunkSteps - 1) / kChunkSteps;
    const int G = gridDim.x;
    const uint32_t raw_bytes = kTileRows * (FMT == 4 ? 32 : 64);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&a_full[s], kDeqThreads);
            mbar_init(&b_full[s], 1);
            mbar_init(&st_empty[s], 1);
        }
        for (int i = 0; i < kRaw; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], kDeqThreads);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sc_full[b], 1);
            mbar_init(&sc_empty[b], kDeqGroups * kDeqThreads);
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiThreads);
        }
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kWsTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == kWTmaWarp) {
        // ============================================================ weight TMA
        if (lane == 0) {
            int j = 0, q = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += G) {
                const int y0 = (t % n_o_tiles) * kTileRows;
                for (int ks = 0; ks < nk; ++ks, ++j) {
                    if (FMT == 4 && ks % kChunkSteps == 0) {
                        const int b = q & 1;
                        if (q >= 2 &&
                            !mbar_wait(&sc_empty[b], static_cast<uint32_t>((q / 2) - 1) & 1u)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(&sc_full[b], kTileRows * kScaleWords * 4);
                        tma_load_2d(base + L.sc_off + b * kScaleSlot, &s_map,
                                    (ks / kChunkSteps) * kScaleWords, y0, &sc_full[b]);
                        ++q;
                    }
                    const int slot = j % kRaw;
                    if (j >= kRaw &&
                        !mbar_wait(&raw_empty[slot], static_cast<uint32_t>((j / kRaw) - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&raw_full[slot], raw_bytes);
                    tma_load_2d(base + L.raw_off + slot * kRawSlot, &w_map,
                                ks * (FMT == 4 ? 32 : 64), y0, &raw_full[slot]);
                }
            }
        }
        __syncwarp();
    } else if (warp == kXTmaWarp) {
        // ============================================================ activation TMA
        if (lane == 0) {
            pdl_wait_prior_grid();     // the 16-bit activations come from the pre-pass
            int j = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += G) {
                const int m0 = (t / n_o_tiles) * kWsTileM;
                for (int ks = 0; ks < nk; ++ks, ++j) {
                    const int s = j % kStages;
                    if (j >= kStages &&
                        !mbar_wait(&st_empty[s], static_cast<uint32_t>((j / kStages) - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&b_full[s], kWsTileM * 128);
                    tma_load_2d(base + L.st_off + s * kStageBytes + kOpStage, &x_map,
                                ks * kAtomK, m0, &b_full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp < kDeqWarps) {
        // ============================================================ dequantizers
        const int g = warp >> 2;
        const int r = threadIdx.x & (kDeqThreads - 1);
        int tile_local = 0;
        for (int t = blockIdx.x; t < n_tiles && ok; t += G, ++tile_local) {
            for (int c = 0; c < n_chunks && ok; ++c) {
                const int q = tile_local * n_chunks + c;
                const int b = q & 1;
                if (FMT == 4 && !mbar_wait(&sc_full[b], static_cast<uint32_t>(q / 2) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t sc_row = base + L.sc_off + b * kScaleSlot + r * (kScaleWords * 4);
                const int ks_end = min(nk, (c + 1) * kChunkSteps);
                for (int ks = c * kChunkSteps + g; ks < ks_end; ks += kDeqGroups) {
                    const int j = tile_local * nk + ks;
                    const int slot = j % kRaw;
                    if (!mbar_wait(&raw_full[slot], static_cast<uint32_t>(j / kRaw) & 1u)) {
                        ok = false;
                        break;
                    }
                    const RowRaw R = load_row_raw<FMT>(base + L.raw_off + slot * kRawSlot, r,
                                                       sc_row + (ks % kChunkSteps) * 8);
                    const int s = j % kStages;
                    if (j >= kStages &&
                        !mbar_wait(&st_empty[s], static_cast<uint32_t>((j / kStages) - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    store_row_op<FMT, OP>(R, base + L.st_off + s * kStageBytes, r);
                    fence_proxy_async_smem();
                    mbar_arrive(&a_full[s]);
                    mbar_arrive(&raw_empty[slot]);   // after its contents were consumed
                }
                if (!ok) break;
                if (FMT == 4) mbar_arrive(&sc_empty[b]);
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            const uint32_t idesc =
                idesc_f16kind_f32acc(kTileRows, kWsTileM, static_cast<uint32_t>(OP));
            int j = 0, tile_local = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += G, ++tile_local) {
                const int b = tile_local & 1;
                if (tile_local >= 2 &&
                    !mbar_wait(&acc_empty[b], static_cast<uint32_t>((tile_local / 2) - 1) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d = tmem + static_cast<uint32_t>(b * kWsTileM);
                for (int ks = 0; ks < nk; ++ks, ++j) {
                    const int s = j % kStages;
                    const uint32_t par = static_cast<uint32_t>(j / kStages) & 1u;
                    if (!mbar_wait(&a_full[s], par) || !mbar_wait(&b_full[s], par)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sa = base + L.st_off + s * kStageBytes;
                    const uint64_t adesc = sw128_kmajor_desc(sa);
                    const uint64_t bdesc = sw128_kmajor_desc(sa + kOpStage);
#pragma unroll
                    for (int kk = 0; kk < kAtomK / 16; ++kk)
                        tc_mma_f16kind(d, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                       (ks > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&st_empty[s]);
                }
                if (!ok) break;
                tc_commit(&acc_full[b]);
            }
        }
        __syncwarp();
    } else {
        // ============================================================ epilogue
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t tq = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        int tile_local = 0;
        for (int t = blockIdx.x; t < n_tiles && ok; t += G, ++tile_local) {
            const int b = tile_local & 1;
            ok = mbar_wait(&acc_full[b], static_cast<uint32_t>(tile_local / 2) & 1u);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            const int m0 = (t / n_o_tiles) * kWsTileM;
            const int o = (t % n_o_tiles) * kTileRows + row;
            float sc = 1.f;
            if (FMT == 8 && o < N) sc = __ldg(S8 + o);
            const int mlim = min(kWsTileM, M - m0);
            float *yo = Y + static_cast<size_t>(m0) * N + o;
            for (int c = 0; c < kWsTileM; c += 16) {
                uint32_t v[16];
                tmem_ld_x16(tq + static_cast<uint32_t>(b * kWsTileM + c), v);
                tmem_ld_wait();
                if (o < N) {
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        if (c + jj < mlim)
                            yo[static_cast<size_t>(c + jj) * N] = __uint_as_float(v[jj]) * sc;
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&acc_empty[b]);
        }
        pdl_launch_dependents();
    }
    if (!ok) atomicOr(status, 1u << kStatusTimeout);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kWsTmemCols);
    }
}

template <int FMT, Op16 OP>
cudaError_t launch_ws(const void *Xh, const void *Wq, const void *S, float *Y, int M, int N,
                      int K, unsigned *status, cudaStream_t st) {
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(ws_qgemm_kernel<FMT, OP>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    CUtensorMap w_map, s_map, x_map;
    bool enc_ok = encode_tma_2d(&x_map, OP == Op16::f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                2, Xh, K, M, kAtomK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (FMT == 4) {
        enc_ok = enc_ok &&
                 encode_tma_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K / 2, N, 32,
                               CU_TENSOR_MAP_SWIZZLE_NONE) &&
                 encode_tma_2d(&s_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, S, K / 32, N,
                               kScaleWords, CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        enc_ok = enc_ok && encode_tma_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K, N, 64,
                                         CU_TENSOR_MAP_SWIZZLE_NONE);
        s_map = w_map;   // unused by the q8 kernel
    }
    if (!enc_ok) return cudaErrorInvalidValue;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_o = (N + kTileRows - 1) / kTileRows;
    const int n_m = (M + kWsTileM - 1) / kWsTileM;
    const int tiles = n_o * n_m;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(std::min(tiles, sms), 1, 1);
    cfg.blockDim = dim3(kWsThreads, 1, 1);
    cfg.dynamicSmemBytes = ws_layout().total + 1024;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ws_qgemm_kernel<FMT, OP>, w_map, s_map, x_map,
                              static_cast<const float *>(S), Y, M, N, K, n_o, tiles, status);
}

}  // namespace

// Shapes the TMA-fed weight-stationary kernel takes: more than one
// 128-row activation tile, and K a multiple of 64 (q8) or 128 (q4: the
// (scale, min) rows are TMA boxes whose global stride K/8 bytes must be a
// multiple of 16).
bool ws_supported(int fmt, int M, int N, int K) {
    (void)N;
    if (M <= kWsTileM) return false;
    return fmt == 4 ? K % 128 == 0 : K % 64 == 0;
}

cudaError_t launch_ws_q4(const void *Xh, const uint8_t *Wq, const uint16_t *SM, float *Y, int M,
                         int N, int K, bool bf16, unsigned *status, cudaStream_t s) {
    return bf16 ? launch_ws<4, Op16::bf16>(Xh, Wq, SM, Y, M, N, K, status, s)
                : launch_ws<4, Op16::f16>(Xh, Wq, SM, Y, M, N, K, status, s);
}

cudaError_t launch_ws_q8(const void *Xh, const int8_t *Wq, const float *S, float *Y, int M, int N,
                         int K, bool bf16, unsigned *status, cudaStream_t s) {
    return bf16 ? launch_ws<8, Op16::bf16>(Xh, Wq, S, Y, M, N, K, status, s)
                : launch_ws<8, Op16::f16>(Xh, Wq, S, Y, M, N, K, status, s);
}

}  // namespace rtq
