// tcgen05 path for many activation rows and short K (K <= 512): activations
// stay resident in shared memory, TMA streams the packed weights past them.
//
// The tile product is the same transposed one as in tc.cu,
//   D[o, m] = sum_k W_hat[o, k] * X[m, k],
// with 128 weight rows as the MMA's M dimension and 192 activation rows as its
// N dimension, but the operands swap roles in memory: a CTA loads one 192-row
// block of the activations (already rounded to fp16 by the pre-pass in
// prep.cu) ONCE -- all of K, 192 x K x 2 bytes of shared memory, as K/64
// TMA boxes in the 128-byte-swizzled operand layout -- and then walks a run of
// weight tiles against it.  Each activation byte crosses L2 once per CTA
// rather than once per 128-row weight tile; the weights (0.6 to 1.3 MB per
// projection, resident in L2) are re-read once per activation block instead.
//
// Work list: the (activation block, weight tile) pairs in activation-major
// order, split into one contiguous run per CTA (one CTA per SM), so a CTA
// changes activation block rarely.
//
// Roles (20 warps):
//   warp 18     activation TMA (one thread): on every change of activation
//               block, once the MMAs on the previous block have completed,
//               K/64 boxes into the resident tile, one transaction barrier.
//   warp 17     weight TMA (one thread): per weight tile the (scale, min)
//               words of its 128 rows (q4), and per 64-wide K step the
//               128-row slice of packed codes, two K steps per TMA box
//               (a box costs about the same per row at any width up to 256
//               bytes), into a ring of kRaw such pairs.
//   warps 0-7   dequantizers: an A stage holds a pair of 64-wide K steps
//               (64 columns).  Thread (r, h) converts step h of every pair of
//               weight row r (32 or 64 bytes of codes) and writes it with
//               tcgen05.st into TMEM lane r of the pair's stage (32 of its 64
//               columns), so one stage hand-over serves two K steps.  The A
//               operand never touches shared memory, which leaves its
//               bandwidth to the MMA's activation reads and the TMA traffic.
//   warp 8      MMA issuer (the warp walks, an elected lane issues): per
//               weight tile, K/128 stages x 8 tcgen05.mma (K = 16, A from
//               TMEM, B from shared memory) into one of two TMEM
//               accumulators.  It waits on no mbarrier.
//   warp 19     MMA waiter: waits for each stage (and the activation block
//               and accumulator) and hands the pair to the issuer through a
//               named barrier.
//   warps 9-16  epilogue, two warps per TMEM lane quadrant: TMEM ->
//               registers (q8 row scale) -> fp32 Y with 128-byte coalesced
//               rows, overlapping the next tile's MMAs.
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

// MMA N.  An M = 128, K = 16 tcgen05.mma costs about the same time for any
// N up to 192 and only a little more at 256, so the tile is as wide as TMEM
// allows with two accumulators and the A stages: 2 x 192 + 2 x 64 = 512
// columns.  192 resident rows of K = 512 also just fit in shared memory.
constexpr int kXsTileM = 192;                 // activation rows per block (MMA N)
constexpr int kXsMaxK = 512;
constexpr int kXAtoms = kXsMaxK / 64;                    // 64-wide K atoms of a resident block
constexpr int kDeqGroups = 2;                            // two K halves per step
constexpr int kDeqThreads = kTileRows;                   // 128 per half
constexpr int kDeqWarps = kDeqGroups * 4;                // 8
constexpr int kMmaWarp = kDeqWarps;                      // 8
constexpr int kEpiWarp0 = kMmaWarp + 1;                  // 9
constexpr int kEpiWarps = 8;                             // two per TMEM lane quadrant
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kEpiCols = kXsTileM / 2;                   // columns per epilogue warp
constexpr int kWTmaWarp = kEpiWarp0 + kEpiWarps;         // 17
constexpr int kXTmaWarp = kWTmaWarp + 1;                 // 18
constexpr int kWaitWarp = kXTmaWarp + 1;                 // 19
constexpr int kXsThreads = (kWaitWarp + 1) * 32;         // 640
constexpr uint32_t kMmaBar = 1;                          // named barrier: waiter <-> MMA warp
constexpr int kXAtom = kXsTileM * 128;                   // 24 KB: 192 rows x 64 K
constexpr int kAStages = 2;                              // A stages in TMEM, two K steps each
constexpr int kRaw = 2;                                  // packed-code ring depth (step pairs)
constexpr uint32_t kAccCols = 2 * kXsTileM;              // 2 accumulators x 192 columns
constexpr uint32_t kAStageCols = kAtomK;                 // 2 x 64 16-bit values per lane
constexpr uint32_t kXsTmemCols = 512;                    // accumulators + A stages, pow2

static_assert(kAccCols + kAStages * kAStageCols <= kXsTmemCols, "TMEM budget");
static_assert(kEpiCols % 32 == 0, "epilogue reads 32 columns at a time");

// Packed codes of two K steps (128 rows x 64 B for q4, x 128 B for q8), and the
// (scale, min) words of a weight tile (q4: 128 rows x 16 words, one box that
// covers K = 512 and is zero-filled past the tensor for shorter K).
constexpr int kScaleWords = 16;
__host__ __device__ constexpr int raw_slot_bytes(int fmt) { return kTileRows * (fmt == 4 ? 64 : 128); }
__host__ __device__ constexpr int scale_slot_bytes(int fmt, int K) {
    return fmt == 4 ? kTileRows * kScaleWords * 4 + 0 * K : 0;
}

struct XsLayout {
    int x_off, raw_off, sc_off, bar_off, total;
};

__host__ __device__ inline XsLayout xs_layout(int fmt, int K) {
    XsLayout L;
    L.x_off = 0;
    L.raw_off = (K / kAtomK) * kXAtom;
    L.sc_off = L.raw_off + kRaw * raw_slot_bytes(fmt);
    L.bar_off = L.sc_off + 2 * scale_slot_bytes(fmt, K);
    // raw_full/empty[kRaw], sc_full/empty[2], a_full/empty[kAStages],
    // x_full[kXAtoms], x_empty, acc_full/empty[2], drain, + TMEM address slot
    L.total = L.bar_off + (2 * kRaw + 4 + 2 * kAStages + kXAtoms + 1 + 4 + 1) * 8 + 16;
    return L;
}

// Iterates a CTA's run of (activation block, weight tile) items with
// incremental counters instead of divisions.
struct ItemCursor {
    int item, last, m_tile, o_tile, n_o;
    __device__ ItemCursor(int first, int last_, int n_o_tiles)
        : item(first), last(last_), m_tile(first / n_o_tiles), o_tile(first % n_o_tiles),
          n_o(n_o_tiles) {}
    __device__ bool valid() const { return item < last; }
    __device__ void next() {
        ++item;
        if (++o_tile == n_o) {
            o_tile = 0;
            ++m_tile;
        }
    }
};

template <int FMT>
__global__ void __launch_bounds__(kXsThreads, 1)
    xs_qgemm_kernel(const __grid_constant__ CUtensorMap w_map,
                    const __grid_constant__ CUtensorMap s_map,
                    const __grid_constant__ CUtensorMap x_map, const float *__restrict__ S8,
                    const float *__restrict__ bias, float *__restrict__ Y, int M, int N, int K,
                    int n_o_tiles, int n_items, DevCtl *ctl) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const XsLayout L = xs_layout(FMT, K);
    constexpr int kRawSlot = raw_slot_bytes(FMT);
    const int kScaleSlot = scale_slot_bytes(FMT, K);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *raw_full = bars;
    uint64_t *raw_empty = raw_full + kRaw;
    uint64_t *sc_full = raw_empty + kRaw;
    uint64_t *sc_empty = sc_full + 2;
    uint64_t *a_full = sc_empty + 2;
    uint64_t *a_empty = a_full + kAStages;
    uint64_t *x_full = a_empty + kAStages;                // one per K atom
    uint64_t *x_empty = x_full + kXAtoms;
    uint64_t *acc_full = x_empty + 1;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;          // MMA thread's completion wait after an abort
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    // waiter -> MMA warp abort flags, one per K-step parity
    volatile uint32_t *mma_abort = tmem_slot + 1;
    const unsigned long long *lim = &ctl->wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / kAtomK;
    const int G = gridDim.x;
    const int first = static_cast<int>((static_cast<long long>(blockIdx.x) * n_items) / G);
    const int last = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * n_items) / G);
    const uint32_t raw_bytes = raw_slot_bytes(FMT);
    const uint32_t sc_bytes = kTileRows * kScaleWords * 4;

    if (threadIdx.x == 0) {
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
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], kDeqGroups * kDeqThreads);
            mbar_init(&a_empty[s], 1);
        }
        for (int a = 0; a < kXAtoms; ++a) mbar_init(&x_full[a], 1);
        mbar_init(x_empty, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kXsTmemCols);
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
        // Packed weights do not depend on the previous kernel in the stream,
        // so this role starts before the dependency wait.  (Test hook: with
        // `inject` the first packed-code box is never requested, so the
        // dequantizers' wait for it runs out.)
        if (lane == 0) {
            int j = 0, n_sc = 0;
            for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
                const int n_local = it.item - first;
                const int y0 = it.o_tile * kTileRows;
                if (FMT == 4) {
                    const int b = n_local & 1;
                    if (n_local >= 2 &&
                        !mbar_wait(&sc_empty[b], static_cast<uint32_t>((n_local / 2) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&sc_full[b], sc_bytes);
                    tma_load_2d(base + L.sc_off + b * kScaleSlot, &s_map, 0, y0, &sc_full[b]);
                    ++n_sc;
                }
                for (int p = 0; p < nk / 2; ++p, ++j) {
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
                const int last_j = i + ((j - 1 - i) / kRaw) * kRaw;   // last load of slot i
                if (!(last_j == 0 && ctl->inject))
                    mbar_wait(&raw_full[i], static_cast<uint32_t>(last_j / kRaw) & 1u, lim);
            }
            for (int i = 0; i < 2 && i < n_sc; ++i) {
                const int last_q = i + ((n_sc - 1 - i) / 2) * 2;
                mbar_wait(&sc_full[i], static_cast<uint32_t>(last_q / 2) & 1u, lim);
            }
        }
        __syncwarp();
    } else if (warp == kXTmaWarp) {
        // ============================================================ activation TMA
        if (lane == 0) {
            pdl_wait_prior_grid();     // the 16-bit activations come from the pre-pass
            int cur_m = -1, x_loads = 0;
            for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
                if (it.m_tile == cur_m) continue;
                cur_m = it.m_tile;
                if (x_loads > 0 &&
                    !mbar_wait(x_empty, static_cast<uint32_t>(x_loads - 1) & 1u, lim)) {
                    ok = false;
                    break;
                }
                // one barrier per atom: the first item's K steps start as
                // their own atoms land instead of after the whole block
                for (int a = 0; a < nk; ++a) {
                    mbar_expect_tx(&x_full[a], static_cast<uint32_t>(kXAtom));
                    tma_load_2d(base + L.x_off + a * kXAtom, &x_map, a * kAtomK,
                                cur_m * kXsTileM, &x_full[a]);
                }
                ++x_loads;
            }
            // every requested activation box has landed before the CTA exits
            if (x_loads > 0)
                for (int a = 0; a < nk; ++a)
                    mbar_wait(&x_full[a], static_cast<uint32_t>(x_loads - 1) & 1u, lim);
        }
        __syncwarp();
    } else if (warp < kDeqWarps) {
        // ============================================================ dequantizers
        const int h = warp >> 2;                     // step h of every step pair
        const int r = threadIdx.x & (kDeqThreads - 1);
        // this warp's 32 TMEM lanes (warp % 4 selects the lane quadrant) and
        // its 32 columns (one K step) of each 64-column A stage
        const uint32_t ta = tmem + kAccCols + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                            static_cast<uint32_t>(32 * h);
        uint32_t jp = 0;                             // step pairs (A stages) so far
        for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            uint32_t sw[kScaleWords / 2] = {};
            if (FMT == 4) {
                if (!mbar_wait(&sc_full[b], static_cast<uint32_t>(n_local / 2) & 1u, lim)) {
                    ok = false;
                    break;
                }
                load_scale_pairs(base + L.sc_off + b * kScaleSlot + r * (kScaleWords * 4), r, h, sw);
                // sw depends on every word read, so the reads have completed
                fence_proxy_async_smem();
                mbar_arrive(&sc_empty[b]);
            }
#pragma unroll
            for (int kp = 0; kp < kXsMaxK / kAtomK / 2; ++kp, ++jp) {
                if (2 * kp >= nk) break;
                const uint32_t jr = n_local * (nk / 2) + kp;          // step pair of the raw ring
                const int slot = jr % kRaw;
                if (!mbar_wait(&raw_full[slot], static_cast<uint32_t>(jr / kRaw) & 1u, lim)) {
                    ok = false;
                    break;
                }
                // step h of the pair, both K halves; convert before waiting for
                // the stage, so only the TMEM stores sit on its round trip
                const uint32_t raw = base + L.raw_off + slot * kRawSlot;
                uint32_t w0[16], w1[16];
                half_words<FMT>(load_half_raw2<FMT>(raw, r, 0, h, sw[2 * kp]), w0);
                half_words<FMT>(load_half_raw2<FMT>(raw, r, 1, h, sw[2 * kp + 1]), w1);
                // the reads are consumed; the proxy fence orders them before
                // the TMA that refills the slot
                fence_proxy_async_smem();
                mbar_arrive(&raw_empty[slot]);
                const uint32_t st = jp & (kAStages - 1);
                if (jp >= kAStages &&
                    !mbar_wait(&a_empty[st], ((jp / kAStages) - 1) & 1u, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                tmem_st_x16(ta + st * kAStageCols, w0);
                tmem_st_x16(ta + st * kAStageCols + 16, w1);
                tmem_st_wait();
                tc_fence_before_sync();
                mbar_arrive(&a_full[st]);
            }
            if (!ok) break;
        }
    } else if (warp == kWaitWarp) {
        // ============================================================ MMA waiter
        // Every mbarrier wait the MMA issuer needs happens here; each K step
        // is handed over through named barrier kMmaBar.  A thread that waits
        // on an mbarrier after issuing tcgen05.commit stalls until its
        // queued MMAs drain, so the issuing thread itself never waits.
        int cur_m = -1, x_loads = 0;
        uint32_t j = 0;
        for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            bool good = true;
            const bool fresh = it.m_tile != cur_m;          // first item of a new block
            if (fresh) {
                cur_m = it.m_tile;
                ++x_loads;
            }
            const uint32_t xpar = static_cast<uint32_t>(x_loads - 1) & 1u;
            // accumulator b must have been drained by the epilogue
            if (lane == 0 && n_local >= 2)
                good = mbar_wait(&acc_empty[b], static_cast<uint32_t>((n_local / 2) - 1) & 1u,
                                 lim);
            for (int kp = 0; 2 * kp < nk; ++kp, ++j) {       // j: step pairs so far
                if (lane == 0) {
                    if (good && fresh) good = mbar_wait(&x_full[2 * kp], xpar, lim);
                    if (good && fresh) good = mbar_wait(&x_full[2 * kp + 1], xpar, lim);
                    if (good)
                        good = mbar_wait(&a_full[j & (kAStages - 1)], (j / kAStages) & 1u, lim);
                    mma_abort[j & 1] = good ? 0u : 1u;
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
        const uint32_t idesc = idesc_f16_f32acc(kTileRows, kXsTileM);
        static_assert(kXsTileM % 16 == 0 && kXsTileM <= 256, "MMA N for M = 128");
        static_assert((kAStages & (kAStages - 1)) == 0, "A ring indexed with a mask");
        constexpr uint64_t kXAtomDesc = kXAtom >> 4;   // descriptor step per X atom
        const uint64_t bdesc0 = sw128_kmajor_desc(base + L.x_off);
        uint32_t j = 0;                                 // step pairs issued so far
        bool abort = false;
        for (ItemCursor it(first, last, n_o_tiles); it.valid() && !abort; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            const uint32_t d = tmem + static_cast<uint32_t>(b * kXsTileM);
            uint64_t bdesc = bdesc0;
            for (int kp = 0; 2 * kp < nk; ++kp, ++j, bdesc += 2 * kXAtomDesc) {
                named_bar_sync(kMmaBar, 64);           // the waiter saw pair j's stage full
                if (mma_abort[j & 1]) {
                    abort = true;
                    break;
                }
                // the whole warp walks the loop; one elected lane issues the
                // pair's 8 MMAs (step u's A in columns 32u .. 32u + 31)
                tc_fence_after_sync();
                const uint32_t at = tmem + kAccCols + (j & (kAStages - 1)) * kAStageCols;
                if (elect_one()) {
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int kk = 0; kk < kAtomK / 16; ++kk)
                            tc_mma_f16kind_ts(d, at + 32 * u + 8 * kk, bdesc + u * kXAtomDesc + 2 * kk,
                                              idesc, (kp > 0 || u > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&a_empty[j & (kAStages - 1)]);
                }
                __syncwarp();
            }
            if (abort) break;
            if (elect_one()) {
                tc_commit(&acc_full[b]);
                // last item of this activation block with another block to
                // follow: release the X tile once these MMAs have completed
                if (it.item + 1 < last && it.o_tile + 1 == n_o_tiles) tc_commit(x_empty);
            }
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
        const int q = warp & 3;                       // TMEM lane quadrant of this warp
        const int c0 = ((warp - kEpiWarp0) >> 2) * kEpiCols;   // its half of the columns
        const int row = q * 32 + lane;
        const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
        for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            ok = mbar_wait(&acc_full[b], static_cast<uint32_t>(n_local / 2) & 1u, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            const int m0 = it.m_tile * kXsTileM;
            const int o = it.o_tile * kTileRows + row;
            float sc = 1.f, bo = 0.f;
            if (FMT == 8 && o < N) sc = __ldg(S8 + o);
            if (bias && o < N) bo = __ldg(bias + o);
            const int mlim = min(kXsTileM, M - m0);
            float *yo = Y + static_cast<size_t>(m0) * N + o;
            const size_t rs = static_cast<size_t>(N);
            for (int c = c0; c < c0 + kEpiCols; c += 32) {
                uint32_t v[32];
                tmem_ld_x32(tq + static_cast<uint32_t>(b * kXsTileM + c), v);
                tmem_ld_wait();
                if (o < N) {
                    float *p = yo + static_cast<size_t>(c) * rs;
                    if (c + 32 <= mlim) {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) p[jj * rs] = fmaf(__uint_as_float(v[jj]), sc, bo);
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            if (c + jj < mlim) p[jj * rs] = fmaf(__uint_as_float(v[jj]), sc, bo);
                    }
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&acc_empty[b]);
        }
    }
    if (!ok) atomicOr(&ctl->status, 1u << kStatusTimeout);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kXsTmemCols);
    }
}

template <int FMT>
cudaError_t launch_xs_fmt(const void *Xh, const void *Wq, const void *S, const float *bias,
                          float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t st) {
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(xs_qgemm_kernel<FMT>, 227 * 1024, dev, attr_done)) != cudaSuccess)
        return e;
    CUtensorMap w_map, s_map, x_map;
    bool enc_ok = encode_tma_2d(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Xh, K, M, kAtomK,
                                CU_TENSOR_MAP_SWIZZLE_128B, kXsTileM);
    if (FMT == 4) {
        enc_ok = enc_ok &&
                 encode_tma_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K / 2, N, 64,
                               CU_TENSOR_MAP_SWIZZLE_64B) &&
                 encode_tma_2d(&s_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, S, K / 32, N, kScaleWords,
                               CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        enc_ok = enc_ok && encode_tma_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K, N, 128,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
        s_map = w_map;   // unused by the q8 kernel
    }
    if (!enc_ok) return cudaErrorInvalidValue;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_o = (N + kTileRows - 1) / kTileRows;
    const int n_m = (M + kXsTileM - 1) / kXsTileM;
    const int items = n_o * n_m;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(std::min(items, sms), 1, 1);
    cfg.blockDim = dim3(kXsThreads, 1, 1);
    cfg.dynamicSmemBytes = xs_layout(FMT, K).total + 1024;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, xs_qgemm_kernel<FMT>, w_map, s_map, x_map,
                              static_cast<const float *>(S), bias, Y, M, N, K, n_o, items, ctl);
}

}  // namespace

// Shapes the activation-resident kernel takes: K a multiple of 128 up to 512
// (the (scale, min) rows are TMA boxes, whose global stride K/8 bytes must be
// a multiple of 16; 192 rows of K = 512 fill the shared memory) and more than
// 128 activation rows (fewer go to the weight-stationary kernel).
bool xs_supported(int M, int N, int K) {
    (void)N;
    return K % 128 == 0 && K <= kXsMaxK && M > kTileRows;
}

cudaError_t launch_xs(int fmt, const void *Xh, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s) {
    if (fmt == kFmtQ4) return launch_xs_fmt<kFmtQ4>(Xh, Wq, S, bias, Y, M, N, K, ctl, s);
    if (fmt == kFmtQ8) return launch_xs_fmt<kFmtQ8>(Xh, Wq, S, bias, Y, M, N, K, ctl, s);
    return launch_xs_fmt<kFmtE4M3>(Xh, Wq, S, bias, Y, M, N, K, ctl, s);
}

}  // namespace rtq
