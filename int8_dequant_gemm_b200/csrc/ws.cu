// tcgen05 path for many activation rows and long K (K > 512): weight tile
// stationary, TMA streams both operands' raw data through a stage ring.
//
// Tile product as in tc.cu / xs.cu, D[o, m] = sum_k W_hat[o, k] * X[m, k],
// 128 weight rows (MMA M) x bn activation rows (MMA N), full K per tile.
// A persistent CTA (one per SM) walks tiles t = blockIdx.x, + gridDim.x, ...
// in weight-tile-fastest order, so concurrently running CTAs share activation
// tiles in L2.  bn is chosen per launch (a multiple of 32 from 64 to 192,
// ws_tile_rows): a tile takes about as long as its dequantization plus its
// MMAs, so the widest tile is the cheapest per output unless the tile count
// leaves a last wave mostly empty (M = 4096, N = 512: 88 tiles of 192 rows on
// 148 SMs, against 128 tiles of 128 rows in the same single wave).
//
// Per pair of 64-wide K steps one A stage holds the 128 x 128 dequantized
// weights in 64 TMEM columns (written with tcgen05.st by the dequantizers
// from TMA-staged packed codes, as in xs.cu); per K step one B stage holds the
// bn x 64 fp16 activations in shared memory, one TMA box from the
// pre-converted activations (prep.cu) in the 128-byte-swizzled operand
// layout.  The A and B rings are separate: TMEM holds two 192-column
// accumulators and two 64-column A stages (512 columns); shared memory holds
// six B stages.
// Roles (20 warps): warps 0-7 dequantizers (thread (r, h) converts step h of
// every step pair of weight row r, as in xs.cu), warp 8 MMA issuer (fed by
// the waiter, warp 19, through a named barrier, per step pair, as in xs.cu),
// warps 9-16
// epilogue (two per TMEM lane quadrant, double-buffered accumulators), warp 17
// weight TMA (codes and, for q4, (scale, min) blocks of up to 16 words per
// row), warp 18 activation TMA.
//
// Every mbarrier wait is bounded; a wait that gives up latches
// RT_ERR_DEVICE_TIMEOUT in the device status word and the CTA winds down: the
// TMA threads wait (bounded) for the copies they issued, the MMA thread for the
// MMAs it issued, before the CTA releases its shared memory and TMEM.
#include <algorithm>

#include "kernels.cuh"
#include "tmapipe.cuh"

namespace rtq {
namespace {

constexpr int kWsTileM = 192;                 // widest activation tile (MMA N)
constexpr int kWsTileMin = 64;
constexpr int kDeqGroups = 2;                            // two K halves per step
constexpr int kDeqThreads = kTileRows;                   // 128 per group
constexpr int kDeqWarps = kDeqGroups * 4;                // 8
constexpr int kMmaWarp = kDeqWarps;                      // 8
constexpr int kEpiWarp0 = kMmaWarp + 1;                  // 9
constexpr int kEpiWarps = 8;                             // two per TMEM lane quadrant
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kWTmaWarp = kEpiWarp0 + kEpiWarps;         // 17
constexpr int kXTmaWarp = kWTmaWarp + 1;                 // 18
constexpr int kWaitWarp = kXTmaWarp + 1;                 // 19
constexpr int kWsThreads = (kWaitWarp + 1) * 32;         // 640
constexpr uint32_t kMmaBar = 1;                          // named barrier: waiter <-> MMA warp
constexpr int kStages = 6;                               // B stages (shared memory)
constexpr int kStageBytes = kWsTileM * 128;              // 24 KB: up to 192 rows x 64 K
constexpr int kAStages = 2;                              // A stages (TMEM), two K steps each
constexpr int kRaw = 3;                                  // packed-code ring depth (step pairs)
// Two K steps of packed codes per TMA box (128 rows x 64 B for q4, x 128 B for
// q8, swizzled), as in xs.cu: a box costs about the same per row at any width.
__host__ __device__ constexpr int raw_slot_bytes(int fmt) { return kTileRows * (fmt == 4 ? 64 : 128); }
constexpr int kScaleSlot = 8 * 1024;                     // 128 rows x 16 words
constexpr int kScaleWords = 16;                          // (scale, min) words per chunk row
constexpr int kChunkSteps = kScaleWords / 2;             // K steps covered by one chunk
constexpr uint32_t kAccCols = 2 * kWsTileM;              // 2 accumulators x up to 192 columns
constexpr uint32_t kAStageCols = kAtomK;                 // 2 x 64 16-bit values per lane
constexpr uint32_t kWsTmemCols = 512;
static_assert(kAccCols + kAStages * kAStageCols <= kWsTmemCols, "TMEM budget");
static_assert(kWsTileM % 32 == 0 && kWsTileMin % 32 == 0,
              "an epilogue warp's bn / 2 columns are a multiple of 16");

struct WsLayout {
    int st_off, raw_off, sc_off, bar_off, total;
};

__host__ __device__ inline WsLayout ws_layout() {
    WsLayout L;
    L.st_off = 0;
    L.raw_off = kStages * kStageBytes;
    L.sc_off = L.raw_off + kRaw * raw_slot_bytes(8);   // sized for the larger q8 slots
    L.bar_off = L.sc_off + 2 * kScaleSlot;
    // a_full/a_empty[kAStages], b_full/b_empty[kStages], raw_full/empty[kRaw],
    // sc_full/empty[2], acc_full/empty[2], drain, + TMEM address slot
    L.total = L.bar_off + (2 * kAStages + 2 * kStages + 2 * kRaw + 4 + 4 + 1) * 8 + 16;
    return L;
}

// One output row's values for columns c .. c + W - 1 (Y rows m0 + c + jj, at
// stride rs), scaled and biased; the first `avail` of them are inside M.
template <int W>
__device__ __forceinline__ void store_cols(float *p, size_t rs, const uint32_t (&v)[W], int avail,
                                           float sc, float bo) {
    if (avail >= W) {
#pragma unroll
        for (int jj = 0; jj < W; ++jj) p[jj * rs] = fmaf(__uint_as_float(v[jj]), sc, bo);
    } else {
#pragma unroll
        for (int jj = 0; jj < W; ++jj)
            if (jj < avail) p[jj * rs] = fmaf(__uint_as_float(v[jj]), sc, bo);
    }
}

template <int FMT>
__global__ void __launch_bounds__(kWsThreads, 1)
    ws_qgemm_kernel(const __grid_constant__ CUtensorMap w_map,
                    const __grid_constant__ CUtensorMap s_map,
                    const __grid_constant__ CUtensorMap x_map, const float *__restrict__ S8,
                    const float *__restrict__ bias, float *__restrict__ Y, int M, int N, int K,
                    int bn, int n_o_tiles, int n_tiles, int x_ready, DevCtl *ctl) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const WsLayout L = ws_layout();
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *a_full = bars;
    uint64_t *a_empty = a_full + kAStages;
    uint64_t *b_full = a_empty + kAStages;
    uint64_t *b_empty = b_full + kStages;
    uint64_t *raw_full = b_empty + kStages;
    uint64_t *raw_empty = raw_full + kRaw;
    uint64_t *sc_full = raw_empty + kRaw;
    uint64_t *sc_empty = sc_full + 2;
    uint64_t *acc_full = sc_empty + 2;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;          // MMA thread's completion wait after an abort
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    // waiter -> MMA warp abort flags, one per K-step parity
    volatile uint32_t *mma_abort = tmem_slot + 1;
    const unsigned long long *lim = &ctl->wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / kAtomK;
    const int n_chunks = (nk + kChunkSteps - 1) / kChunkSteps;
    const int G = gridDim.x;
    constexpr int kRawSlot = raw_slot_bytes(FMT);
    const uint32_t raw_bytes = kRawSlot;
    const int npairs = (nk + 1) / 2;                 // step pairs per tile (q8 K may be odd)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], kDeqGroups * kDeqThreads);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        for (int i = 0; i < kRaw; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], kDeqGroups * kDeqThreads);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sc_full[b], 1);
            mbar_init(&sc_empty[b], kDeqGroups * kDeqThreads);
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiThreads);
        }
        mbar_init(drain, 1);
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
    // The next kernel in the stream may be scheduled from here on: whatever it
    // reads of this one's output it reads after its own wait for this grid's
    // completion, and its CTAs take SMs only as this grid's leave them.
    pdl_launch_dependents();
    bool ok = true;

    if (warp == kWTmaWarp) {
        // ============================================================ weight TMA
        // (Test hook: with `inject` the first packed-code box is never
        // requested, so the dequantizers' wait for it runs out.)
        if (lane == 0) {
            int j = 0, q = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += G) {
                const int y0 = (t % n_o_tiles) * kTileRows;
                for (int p = 0; p < npairs; ++p, ++j) {
                    const int ks = 2 * p;
                    if (FMT == 4 && ks % kChunkSteps == 0) {
                        const int b = q & 1;
                        if (q >= 2 &&
                            !mbar_wait(&sc_empty[b], static_cast<uint32_t>((q / 2) - 1) & 1u,
                                       lim)) {
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
                        !mbar_wait(&raw_empty[slot], static_cast<uint32_t>((j / kRaw) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    if (j == 0 && ctl->inject) continue;
                    mbar_expect_tx(&raw_full[slot], raw_bytes);
                    tma_load_2d(base + L.raw_off + slot * kRawSlot, &w_map,
                                p * (FMT == 4 ? 64 : 128), y0, &raw_full[slot]);
                }
            }
            // Before the CTA may exit, every box this thread requested has
            // landed (immediate unless a consumer gave up).  Load number i of
            // a ring slot completes that slot's phase i.
            for (int i = 0; i < kRaw && i < j; ++i) {
                const int last_j = i + ((j - 1 - i) / kRaw) * kRaw;
                if (!(last_j == 0 && ctl->inject))
                    mbar_wait(&raw_full[i], static_cast<uint32_t>(last_j / kRaw) & 1u, lim);
            }
            for (int i = 0; i < 2 && i < q; ++i) {
                const int last_q = i + ((q - 1 - i) / 2) * 2;
                mbar_wait(&sc_full[i], static_cast<uint32_t>(last_q / 2) & 1u, lim);
            }
        }
        __syncwarp();
    } else if (warp == kXTmaWarp) {
        // ============================================================ activation TMA
        if (lane == 0) {
            // the 16-bit activations come from the pre-pass, the previous
            // grid in the stream -- unless they were complete before this
            // launch (x_ready), which then starts at once
            if (!x_ready) pdl_wait_prior_grid();
            int j = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += G) {
                const int m0 = (t / n_o_tiles) * bn;
                for (int ks = 0; ks < nk; ++ks, ++j) {
                    const int s = j % kStages;
                    if (j >= kStages &&
                        !mbar_wait(&b_empty[s], static_cast<uint32_t>((j / kStages) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&b_full[s], static_cast<uint32_t>(bn * 128));
                    tma_load_2d(base + L.st_off + s * kStageBytes, &x_map,
                                ks * kAtomK, m0, &b_full[s]);
                }
            }
            // every requested activation box has landed before the CTA exits
            for (int i = 0; i < kStages && i < j; ++i) {
                const int last_j = i + ((j - 1 - i) / kStages) * kStages;
                mbar_wait(&b_full[i], static_cast<uint32_t>(last_j / kStages) & 1u, lim);
            }
        }
        __syncwarp();
    } else if (warp < kDeqWarps) {
        // ============================================================ dequantizers
        const int h = warp >> 2;                     // step h of every step pair
        const int r = threadIdx.x & (kDeqThreads - 1);
        const uint32_t ta = tmem + kAccCols + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                            static_cast<uint32_t>(32 * h);
        int tile_local = 0, ja = 0;                  // ja: A stages (step pairs) so far
        for (int t = blockIdx.x; t < n_tiles && ok; t += G, ++tile_local) {
            for (int c = 0; c < n_chunks && ok; ++c) {
                const int q = tile_local * n_chunks + c;
                const int b = q & 1;
                uint32_t sw[kChunkSteps] = {};
                if (FMT == 4) {
                    if (!mbar_wait(&sc_full[b], static_cast<uint32_t>(q / 2) & 1u, lim)) {
                        ok = false;
                        break;
                    }
                    load_scale_pairs(base + L.sc_off + b * kScaleSlot + r * (kScaleWords * 4), r,
                                     h, sw);
                    fence_proxy_async_smem();       // sw depends on every word read
                    mbar_arrive(&sc_empty[b]);
                }
#pragma unroll
                for (int kp = 0; kp < kChunkSteps / 2; ++kp) {
                    const int ks0 = c * kChunkSteps + 2 * kp;     // first step of the pair
                    if (ks0 >= nk) break;
                    const int jp = tile_local * npairs + (ks0 >> 1);   // step pair of the raw ring
                    const int slot = jp % kRaw;
                    if (!mbar_wait(&raw_full[slot], static_cast<uint32_t>(jp / kRaw) & 1u, lim)) {
                        ok = false;
                        break;
                    }
                    // step ks0 + h of the pair, both K halves (an odd K leaves
                    // the last pair's second step to nobody); converted before
                    // the stage wait, as in xs.cu
                    const bool mine = ks0 + h < nk;
                    const uint32_t raw = base + L.raw_off + slot * kRawSlot;
                    uint32_t w0[16], w1[16];
                    if (mine) {
                        half_words<FMT>(load_half_raw2<FMT>(raw, r, 0, h, sw[2 * kp]), w0);
                        half_words<FMT>(load_half_raw2<FMT>(raw, r, 1, h, sw[2 * kp + 1]), w1);
                    }
                    fence_proxy_async_smem();           // the slot's reads are consumed
                    mbar_arrive(&raw_empty[slot]);
                    const int st = ja & (kAStages - 1);
                    if (ja >= kAStages &&
                        !mbar_wait(&a_empty[st], static_cast<uint32_t>((ja / kAStages) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    if (mine) {
                        tmem_st_x16(ta + static_cast<uint32_t>(st) * kAStageCols, w0);
                        tmem_st_x16(ta + static_cast<uint32_t>(st) * kAStageCols + 16, w1);
                        tmem_st_wait();
                    }
                    tc_fence_before_sync();
                    mbar_arrive(&a_full[st]);
                    ++ja;
                }
            }
        }
    } else if (warp == kWaitWarp) {
        // ============================================================ MMA waiter
        // As in xs.cu: the waits of the MMA issuer, handed over per K step
        // through named barrier kMmaBar, so that the issuing thread never
        // waits on an mbarrier after a tcgen05.commit.
        int ja = 0, tile_local = 0;                    // ja: step pairs so far
        for (int t = blockIdx.x; t < n_tiles && ok; t += G, ++tile_local) {
            const int b = tile_local & 1;
            bool good = true;
            if (lane == 0 && tile_local >= 2)
                good = mbar_wait(&acc_empty[b],
                                 static_cast<uint32_t>((tile_local / 2) - 1) & 1u, lim);
            for (int kp = 0; 2 * kp < nk; ++kp, ++ja) {
                const int j0 = tile_local * nk + 2 * kp;      // the pair's first K step
                const bool two = 2 * kp + 1 < nk;
                if (lane == 0) {
                    if (good)
                        good = mbar_wait(&a_full[ja % kAStages],
                                         static_cast<uint32_t>(ja / kAStages) & 1u, lim) &&
                               mbar_wait(&b_full[j0 % kStages],
                                         static_cast<uint32_t>(j0 / kStages) & 1u, lim) &&
                               (!two || mbar_wait(&b_full[(j0 + 1) % kStages],
                                                  static_cast<uint32_t>((j0 + 1) / kStages) & 1u, lim));
                    mma_abort[ja & 1] = good ? 0u : 1u;
                }
                named_bar_sync(kMmaBar, 64);
                if (__shfl_sync(0xffffffffu, good ? 1 : 0, 0) == 0) {
                    ok = false;
                    break;
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        const uint32_t idesc = idesc_f16_f32acc(kTileRows, bn);
        constexpr uint64_t kStageDesc = kStageBytes >> 4;   // descriptor step per B stage
        const uint64_t bdesc0 = sw128_kmajor_desc(base + L.st_off);
        int ja = 0, tile_local = 0;                    // ja: step pairs so far
        bool abort = false;
        for (int t = blockIdx.x; t < n_tiles && !abort; t += G, ++tile_local) {
            const int b = tile_local & 1;
            const uint32_t d = tmem + static_cast<uint32_t>(b * kWsTileM);
            for (int kp = 0; 2 * kp < nk; ++kp, ++ja) {
                named_bar_sync(kMmaBar, 64);           // the waiter saw pair ja's stages full
                if (mma_abort[ja & 1]) {
                    abort = true;
                    break;
                }
                // the whole warp walks the loop; one elected lane issues the
                // pair's MMAs (step u's A in columns 32u .. 32u + 31)
                tc_fence_after_sync();
                const int s = ja % kAStages;
                const int j0 = tile_local * nk + 2 * kp;
                const bool two = 2 * kp + 1 < nk;
                const int sb0 = j0 % kStages, sb1 = (j0 + 1) % kStages;
                const uint32_t at = tmem + kAccCols + static_cast<uint32_t>(s) * kAStageCols;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < kAtomK / 16; ++kk)
                        tc_mma_f16kind_ts(d, at + 8 * kk,
                                          bdesc0 + static_cast<uint64_t>(sb0) * kStageDesc + 2 * kk,
                                          idesc, (kp > 0 || kk > 0) ? 1u : 0u);
                    if (two) {
#pragma unroll
                        for (int kk = 0; kk < kAtomK / 16; ++kk)
                            tc_mma_f16kind_ts(d, at + 32 + 8 * kk,
                                              bdesc0 + static_cast<uint64_t>(sb1) * kStageDesc + 2 * kk,
                                              idesc, 1u);
                    }
                    tc_commit(&a_empty[s]);
                    tc_commit(&b_empty[sb0]);
                    if (two) tc_commit(&b_empty[sb1]);
                }
                __syncwarp();
            }
            if (abort) break;
            if (elect_one()) tc_commit(&acc_full[b]);
            __syncwarp();
        }
        if (abort && lane == 0) {
            // MMAs already issued may still read shared memory and write
            // TMEM: wait (bounded) for them before the CTA releases either
            tc_commit(drain);
            mbar_wait(drain, 0, lim);
        }
        __syncwarp();
    } else {
        // ============================================================ epilogue
        const int qd = warp & 3;
        const int ecols = bn / 2;                       // columns per warp: 32 .. 96
        const int c0 = ((warp - kEpiWarp0) >> 2) * ecols;   // its half of the columns
        const int row = qd * 32 + lane;
        const uint32_t tq = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        int tile_local = 0;
        for (int t = blockIdx.x; t < n_tiles && ok; t += G, ++tile_local) {
            const int b = tile_local & 1;
            ok = mbar_wait(&acc_full[b], static_cast<uint32_t>(tile_local / 2) & 1u, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            const int m0 = (t / n_o_tiles) * bn;
            const int o = (t % n_o_tiles) * kTileRows + row;
            float sc = 1.f, bo = 0.f;
            if (FMT == 8 && o < N) sc = __ldg(S8 + o);
            if (bias && o < N) bo = __ldg(bias + o);
            const int mlim = min(bn, M - m0);
            float *yo = Y + static_cast<size_t>(m0) * N + o;
            const size_t rs = static_cast<size_t>(N);
            const uint32_t tb = tq + static_cast<uint32_t>(b * kWsTileM);
            int c = c0;
            for (; c + 32 <= c0 + ecols; c += 32) {
                uint32_t v[32];
                tmem_ld_x32(tb + static_cast<uint32_t>(c), v);
                tmem_ld_wait();
                if (o < N) store_cols(yo + static_cast<size_t>(c) * rs, rs, v, mlim - c, sc, bo);
            }
            if (c < c0 + ecols) {                       // bn / 2 an odd multiple of 16
                uint32_t v[16];
                tmem_ld_x16(tb + static_cast<uint32_t>(c), v);
                tmem_ld_wait();
                if (o < N) store_cols(yo + static_cast<size_t>(c) * rs, rs, v, mlim - c, sc, bo);
            }
            tc_fence_before_sync();
            mbar_arrive(&acc_empty[b]);
        }
    }
    if (!ok) atomicOr(&ctl->status, 1u << kStatusTimeout);
    // x_ready: this grid completes only after the previous grid in the stream
    // has, as it would had it waited before its activation loads, so a later
    // launch that waits for this grid waits for that one too
    if (x_ready && threadIdx.x == 0) pdl_wait_prior_grid();
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kWsTmemCols);
    }
}

template <int FMT>
cudaError_t launch_ws_fmt(const void *Xh, const void *Wq, const void *S, const float *bias,
                          float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t st,
                          bool x_ready) {
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(ws_qgemm_kernel<FMT>, 227 * 1024, dev, attr_done)) != cudaSuccess)
        return e;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int bn = ws_tile_rows(M, N, sms);
    CUtensorMap w_map, s_map, x_map;
    bool enc_ok = encode_tma_2d(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Xh, K, M, kAtomK,
                                CU_TENSOR_MAP_SWIZZLE_128B, static_cast<uint32_t>(bn));
    if (FMT == 4) {
        enc_ok = enc_ok &&
                 encode_tma_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K / 2, N, 64,
                               CU_TENSOR_MAP_SWIZZLE_64B) &&
                 encode_tma_2d(&s_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, S, K / 32, N,
                               kScaleWords, CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        enc_ok = enc_ok && encode_tma_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K, N, 128,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
        s_map = w_map;   // unused by the q8 kernel
    }
    if (!enc_ok) return cudaErrorInvalidValue;
    const int n_o = (N + kTileRows - 1) / kTileRows;
    const int n_m = (M + bn - 1) / bn;
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
    return cudaLaunchKernelEx(&cfg, ws_qgemm_kernel<FMT>, w_map, s_map, x_map,
                              static_cast<const float *>(S), bias, Y, M, N, K, bn, n_o, tiles,
                              x_ready ? 1 : 0, ctl);
}

}  // namespace

// Activation rows per tile: the multiple of 32 from 64 to 192 with the least
// waves x (400 + bn), waves = ceil(tiles / SMs).  The per-tile cost, 400 + bn
// in units of activation columns of MMA, is fitted to the kernel's measured
// per-wave times (N = 512, K = 2048, M = 4096 and 16384, bn = 128 .. 192): a
// weight tile's dequantization and hand-overs cost about as much as 400
// columns.  Measured, this picks the fastest height of the five on each of
// seven shapes from M = 300 to 65536.  Ties keep the wider tile.
int ws_tile_rows(int M, int N, int sms) {
    const long long n_o = (N + kTileRows - 1) / kTileRows;
    int best = kWsTileM;
    long long best_cost = -1;
    for (int bn = kWsTileM; bn >= kWsTileMin; bn -= 32) {
        const long long tiles = n_o * ((M + bn - 1) / bn);
        const long long waves = (tiles + sms - 1) / sms;
        const long long cost = waves * (400 + bn);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// Shapes the TMA-fed weight-streamed kernel takes: more than 128 activation
// rows, and K a multiple of 64 (q8) or 128 (q4: the (scale, min) rows are TMA
// boxes whose global stride K/8 bytes must be a multiple of 16).
bool ws_supported(int fmt, int M, int N, int K) {
    (void)N;
    if (M <= kTileRows) return false;
    return fmt == 4 ? K % 128 == 0 : K % 64 == 0;
}

cudaError_t launch_ws(int fmt, const void *Xh, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s, bool x_ready) {
    if (fmt == kFmtQ4) return launch_ws_fmt<kFmtQ4>(Xh, Wq, S, bias, Y, M, N, K, ctl, s, x_ready);
    if (fmt == kFmtQ8) return launch_ws_fmt<kFmtQ8>(Xh, Wq, S, bias, Y, M, N, K, ctl, s, x_ready);
    return launch_ws_fmt<kFmtE4M3>(Xh, Wq, S, bias, Y, M, N, K, ctl, s, x_ready);
}

}  // namespace rtq
