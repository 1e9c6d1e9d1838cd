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
// Work list: one launch takes up to kMaxGroup problems with the same number of
// activation rows M (one projection, or the K <= 512 projections of a
// transformer block).  Its items are the (problem, activation block, weight
// tile) triples in problem-major, then activation-major order, split into one
// contiguous run per CTA (one CTA per SM), so a CTA changes activation block
// rarely, and a block's problems share one pipeline fill and drain and one
// wave tail instead of one each.  Problems may differ in N, K and weight
// format: a launch whose problems share one format runs the build for that
// format; a launch that mixes q4 with q8 / e4m3 runs the mixed build, which
// sizes every packed-code slot for two q8 steps and reads the q4 (scale, min)
// words of the next item straight from global memory one item ahead instead
// of staging them with TMA (the resident block and two 16 KB code slots leave
// no room for the scale boxes).
//
// Roles (20 warps):
//   warp 18     activation TMA (one thread): on every change of activation
//               block, once the MMAs on the previous block have completed,
//               K/64 boxes into the resident tile, one transaction barrier
//               each (atoms beyond the problem's K complete empty, so every
//               atom barrier completes once per block whatever K is).
//   warp 17     weight TMA (one thread): per weight tile the (scale, min)
//               words of its 128 rows (q4 build), and per 64-wide K step the
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
//               registers (q8 row scale, bias) -> fp32 Y with 128-byte
//               coalesced rows, overlapping the next tile's MMAs.
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
constexpr int kFmtMixed = 0;                             // build for launches that mix formats
// Registers a thread, at most: 20 warps of 88 leave 2304 registers in each of
// the SM's four sub-partitions, room for one 64-register warp of the side
// stream's pre-pass (cvt_x16_lean_kernel) beside every CTA.
constexpr int kXsMaxRegs = 88;

static_assert(kAccCols + kAStages * kAStageCols <= kXsTmemCols, "TMEM budget");
static_assert(kEpiCols % 32 == 0, "epilogue reads 32 columns at a time");

// Packed codes of two K steps (128 rows x 64 B for q4, x 128 B for q8 and
// e4m3; the mixed build sizes every slot for q8), and the (scale, min) words
// of a weight tile (q4 build: 128 rows x 16 words, one box that covers
// K = 512 and is zero-filled past the tensor for shorter K).
constexpr int kScaleWords = 16;
__host__ __device__ constexpr int raw_slot_bytes(int fmt) { return kTileRows * (fmt == 4 ? 64 : 128); }
__host__ __device__ constexpr int scale_slot_bytes(int fmt) {
    return fmt == 4 ? kTileRows * kScaleWords * 4 : 0;
}

struct XsLayout {
    int x_off, raw_off, sc_off, bar_off, total;
};

// Shared-memory layout of a launch whose largest K is K.
__host__ __device__ inline XsLayout xs_layout(int fmt, int K) {
    XsLayout L;
    L.x_off = 0;
    L.raw_off = (K / kAtomK) * kXAtom;
    L.sc_off = L.raw_off + kRaw * raw_slot_bytes(fmt);
    L.bar_off = L.sc_off + 2 * scale_slot_bytes(fmt);
    // raw_full/empty[kRaw], sc_full/empty[2], a_full/empty[kAStages],
    // x_full[kXAtoms], x_empty, acc_full/empty[2], drain, + TMEM address slot
    L.total = L.bar_off + (2 * kRaw + 4 + 2 * kAStages + kXAtoms + 1 + 4 + 1) * 8 + 16;
    return L;
}

// One problem of a launch.  S: q4 (scale, min) words [N, K/32] or q8 fp32
// row scales [N] (unused for e4m3).  item0: its first item in the launch's
// list; n_o: its 128-row weight tiles.
struct XsProblem {
    CUtensorMap w_map;     // packed codes, two K steps per box
    CUtensorMap s_map;     // q4 (scale, min) words (q4 build only)
    CUtensorMap x_map;     // fp16 activations from the pre-pass, 64 x 192 boxes
    const void *S;
    const float *bias;
    float *Y;
    int N, K, fmt, n_o, item0;
};

struct XsParams {
    XsProblem p[kMaxGroup];
    int count, M, n_m, n_items;
};

// Iterates a CTA's run of (problem, activation block, weight tile) items
// with incremental counters instead of divisions.
struct ItemCursor {
    int item, last, pi, m_tile, o_tile, n_o;
    __device__ ItemCursor(const XsParams &P, int first, int last_) : item(first), last(last_) {
        pi = 0;
        while (pi + 1 < P.count && first >= P.p[pi + 1].item0) ++pi;
        n_o = P.p[pi].n_o;
        const int local = first - P.p[pi].item0;
        m_tile = local / n_o;
        o_tile = local % n_o;
    }
    __device__ bool valid() const { return item < last; }
    // identifies the resident activation block the item needs
    __device__ int block() const { return pi * 65536 + m_tile; }
    __device__ void next(const XsParams &P) {
        ++item;
        if (++o_tile == n_o) {
            o_tile = 0;
            if (++m_tile == P.n_m && pi + 1 < P.count) {
                m_tile = 0;
                n_o = P.p[++pi].n_o;
            }
        }
    }
};

__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// Mixed build: thread (r, h)'s (scale, min) words of weight row o of a q4
// problem -- the words of groups 4k + 2h and 4k + 2h + 1, k = 0..3, as
// load_scale_pairs takes them from a staged box -- read from global memory
// (8-byte loads; the host checks 16-byte alignment of S).  Zero for rows
// past N and for groups past K, as the staged box's fill gives.
__device__ __forceinline__ void scale_pairs_global(const XsProblem &q, int o, int h,
                                                   uint32_t (&sw)[kScaleWords / 2]) {
#pragma unroll
    for (int i = 0; i < kScaleWords / 2; ++i) sw[i] = 0u;
    if (o >= q.N) return;
    const int groups = q.K / 32;
    const uint32_t *row = static_cast<const uint32_t *>(q.S) + static_cast<size_t>(o) * groups;
#pragma unroll
    for (int k = 0; k < kScaleWords / 4; ++k) {
        if (4 * k < groups) {
            const uint2 v = ldg_nc_v2(row + 4 * k + 2 * h);
            sw[2 * k] = v.x;
            sw[2 * k + 1] = v.y;
        }
    }
}

// One thread's half step of a pair slot: FMT's conversion, or the problem's
// format in the mixed build.
template <int FMT>
__device__ __forceinline__ void convert_half(int fmt, uint32_t raw, int r, int half, int h,
                                             uint32_t smw, uint32_t (&w)[16]) {
    if (FMT != kFmtMixed) {
        half_words<FMT>(load_half_raw2<FMT>(raw, r, half, h, smw), w);
    } else if (fmt == kFmtQ4) {
        half_words<kFmtQ4>(load_half_raw2<kFmtQ4>(raw, r, half, h, smw), w);
    } else if (fmt == kFmtQ8) {
        half_words<kFmtQ8>(load_half_raw2<kFmtQ8>(raw, r, half, h, smw), w);
    } else {
        half_words<kFmtE4M3>(load_half_raw2<kFmtE4M3>(raw, r, half, h, smw), w);
    }
}

template <int FMT>
__global__ void __maxnreg__(kXsMaxRegs)
    xs_qgemm_kernel(const __grid_constant__ XsParams P, int k_max, DevCtl *ctl) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const XsLayout L = xs_layout(FMT, k_max);
    constexpr int kRawSlot = raw_slot_bytes(FMT);
    constexpr int kScaleSlot = scale_slot_bytes(FMT);
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
    const int G = gridDim.x;
    const int first = static_cast<int>((static_cast<long long>(blockIdx.x) * P.n_items) / G);
    const int last = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * P.n_items) / G);
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
            for (ItemCursor it(P, first, last); it.valid() && ok; it.next(P)) {
                const XsProblem &q = P.p[it.pi];
                const int fmt = FMT != kFmtMixed ? FMT : q.fmt;
                const int nk = q.K / kAtomK;
                const int y0 = it.o_tile * kTileRows;
                if (FMT == kFmtQ4) {
                    const int n_local = it.item - first;
                    const int b = n_local & 1;
                    if (n_local >= 2 &&
                        !mbar_wait(&sc_empty[b], static_cast<uint32_t>((n_local / 2) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&sc_full[b], sc_bytes);
                    tma_load_2d(base + L.sc_off + b * kScaleSlot, &q.s_map, 0, y0, &sc_full[b]);
                    ++n_sc;
                }
                const int box_x = fmt == kFmtQ4 ? 64 : 128;      // bytes of codes per pair row
                const uint32_t box_bytes = static_cast<uint32_t>(raw_slot_bytes(fmt));
                for (int p = 0; p < nk / 2; ++p, ++j) {
                    const int slot = j % kRaw;
                    if (j >= kRaw &&
                        !mbar_wait(&raw_empty[slot], static_cast<uint32_t>((j / kRaw) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    if (j == 0 && ctl->inject) continue;
                    mbar_expect_tx(&raw_full[slot], box_bytes);
                    tma_load_2d(base + L.raw_off + slot * kRawSlot, &q.w_map, p * box_x, y0,
                                &raw_full[slot]);
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
            int cur = -1, x_loads = 0;
            for (ItemCursor it(P, first, last); it.valid() && ok; it.next(P)) {
                if (it.block() == cur) continue;
                cur = it.block();
                if (x_loads > 0 &&
                    !mbar_wait(x_empty, static_cast<uint32_t>(x_loads - 1) & 1u, lim)) {
                    ok = false;
                    break;
                }
                const XsProblem &q = P.p[it.pi];
                const int nk = q.K / kAtomK;
                // one barrier per atom: the first item's K steps start as
                // their own atoms land instead of after the whole block
                for (int a = 0; a < nk; ++a) {
                    mbar_expect_tx(&x_full[a], static_cast<uint32_t>(kXAtom));
                    tma_load_2d(base + L.x_off + a * kXAtom, &q.x_map, a * kAtomK,
                                it.m_tile * kXsTileM, &x_full[a]);
                }
                for (int a = nk; a < kXAtoms; ++a) mbar_arrive(&x_full[a]);
                ++x_loads;
            }
            // every requested activation box has landed before the CTA exits
            if (x_loads > 0)
                for (int a = 0; a < kXAtoms; ++a)
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
        uint32_t jr = 0;                             // step pairs of the raw ring so far
        uint32_t jp = 0;                             // step pairs (A stages) so far
        // mixed build: the (scale, min) words of the next item, loaded one
        // item ahead so their latency hides behind a whole item
        uint32_t sw_next[kScaleWords / 2] = {};
        if (FMT == kFmtMixed && first < last) {
            const ItemCursor it0(P, first, last);
            const XsProblem &q0 = P.p[it0.pi];
            if (q0.fmt == kFmtQ4) scale_pairs_global(q0, it0.o_tile * kTileRows + r, h, sw_next);
        }
        for (ItemCursor it(P, first, last); it.valid() && ok; it.next(P)) {
            const XsProblem &q = P.p[it.pi];
            const int fmt = FMT != kFmtMixed ? FMT : q.fmt;
            const int nk = q.K / kAtomK;
            uint32_t sw[kScaleWords / 2] = {};
            if (FMT == kFmtQ4) {
                const int n_local = it.item - first;
                const int b = n_local & 1;
                if (!mbar_wait(&sc_full[b], static_cast<uint32_t>(n_local / 2) & 1u, lim)) {
                    ok = false;
                    break;
                }
                load_scale_pairs(base + L.sc_off + b * kScaleSlot + r * (kScaleWords * 4), r, h, sw);
                // sw depends on every word read, so the reads have completed
                fence_proxy_async_smem();
                mbar_arrive(&sc_empty[b]);
            } else if (FMT == kFmtMixed) {
#pragma unroll
                for (int i = 0; i < kScaleWords / 2; ++i) sw[i] = sw_next[i];
                ItemCursor nx = it;
                nx.next(P);
                if (nx.valid()) {
                    const XsProblem &qn = P.p[nx.pi];
                    if (qn.fmt == kFmtQ4)
                        scale_pairs_global(qn, nx.o_tile * kTileRows + r, h, sw_next);
                }
            }
#pragma unroll
            for (int kp = 0; kp < kXsMaxK / kAtomK / 2; ++kp, ++jp, ++jr) {
                if (2 * kp >= nk) break;
                const int slot = jr % kRaw;
                if (!mbar_wait(&raw_full[slot], (jr / kRaw) & 1u, lim)) {
                    ok = false;
                    break;
                }
                // step h of the pair, both K halves; convert before waiting for
                // the stage, so only the TMEM stores sit on its round trip
                const uint32_t raw = base + L.raw_off + slot * kRawSlot;
                uint32_t w0[16], w1[16];
                convert_half<FMT>(fmt, raw, r, 0, h, sw[2 * kp], w0);
                convert_half<FMT>(fmt, raw, r, 1, h, sw[2 * kp + 1], w1);
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
        int cur = -1, x_loads = 0;
        uint32_t j = 0;
        for (ItemCursor it(P, first, last); it.valid() && ok; it.next(P)) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            const int nk = P.p[it.pi].K / kAtomK;
            bool good = true;
            const bool fresh = it.block() != cur;           // first item of a new block
            if (fresh) {
                cur = it.block();
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
        for (ItemCursor it(P, first, last); it.valid() && !abort; it.next(P)) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            const int nk = P.p[it.pi].K / kAtomK;
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
                if (it.item + 1 < last && it.o_tile + 1 == it.n_o) tc_commit(x_empty);
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
        const int qd = warp & 3;                      // TMEM lane quadrant of this warp
        const int c0 = ((warp - kEpiWarp0) >> 2) * kEpiCols;   // its half of the columns
        const int row = qd * 32 + lane;
        const uint32_t tq = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        for (ItemCursor it(P, first, last); it.valid() && ok; it.next(P)) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            ok = mbar_wait(&acc_full[b], static_cast<uint32_t>(n_local / 2) & 1u, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            const XsProblem &q = P.p[it.pi];
            const int fmt = FMT != kFmtMixed ? FMT : q.fmt;
            const int N = q.N;
            const int m0 = it.m_tile * kXsTileM;
            const int o = it.o_tile * kTileRows + row;
            float sc = 1.f, bo = 0.f;
            if (fmt == kFmtQ8 && o < N) sc = __ldg(static_cast<const float *>(q.S) + o);
            if (q.bias && o < N) bo = __ldg(q.bias + o);
            const int mlim = min(kXsTileM, P.M - m0);
            float *yo = q.Y + static_cast<size_t>(m0) * N + o;
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

// Fills one problem's maps; false if the driver rejects one.
bool xs_problem(XsProblem &q, const XsInput &in, int build, int M) {
    q.S = in.S;
    q.bias = in.bias;
    q.Y = in.Y;
    q.N = in.N;
    q.K = in.K;
    q.fmt = in.fmt;
    q.n_o = (in.N + kTileRows - 1) / kTileRows;
    bool ok = encode_tma_2d(&q.x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, in.Xh, in.K, M, kAtomK,
                            CU_TENSOR_MAP_SWIZZLE_128B, kXsTileM);
    if (in.fmt == kFmtQ4)
        ok = ok && encode_tma_2d(&q.w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, in.Wq, in.K / 2, in.N,
                                 64, CU_TENSOR_MAP_SWIZZLE_64B);
    else
        ok = ok && encode_tma_2d(&q.w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, in.Wq, in.K, in.N,
                                 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (build == kFmtQ4)
        ok = ok && encode_tma_2d(&q.s_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, in.S, in.K / 32, in.N,
                                 kScaleWords, CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        q.s_map = q.w_map;   // unused by this build
    return ok;
}

template <int FMT>
cudaError_t launch_xs_build(const XsParams &P, int k_max, DevCtl *ctl, cudaStream_t st) {
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(xs_qgemm_kernel<FMT>, 227 * 1024, dev, attr_done)) != cudaSuccess)
        return e;
    const int smem = xs_layout(FMT, k_max).total + 1024;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(std::min(P.n_items, sms), 1, 1);
    cfg.blockDim = dim3(kXsThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, xs_qgemm_kernel<FMT>, P, k_max, ctl);
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

bool xs_group_supported(const XsInput *in, int count, int M) {
    if (count < 1 || count > kMaxGroup) return false;
    for (int i = 0; i < count; ++i) {
        if (!fmt_valid(in[i].fmt) || !xs_supported(M, in[i].N, in[i].K)) return false;
        // q4 scale words: a tensor map (one-format build) or 8-byte loads
        // (mixed build) -- 16-byte aligned either way
        if (in[i].fmt == kFmtQ4 && reinterpret_cast<uintptr_t>(in[i].S) % 16 != 0) return false;
    }
    return true;
}

bool xs_group_leaves_room(const XsInput *in, int count, int M, int threads, int regs) {
    if (!xs_group_supported(in, count, M) || threads < 1 || regs < 1) return false;
    bool mixed = false;
    int k_max = 0;
    for (int i = 0; i < count; ++i) {
        mixed = mixed || in[i].fmt != in[0].fmt;
        k_max = std::max(k_max, in[i].K);
    }
    const int build = mixed ? kFmtMixed : in[0].fmt;
    // registers a thread of each build, looked up once (the same binary on
    // every device)
    static std::atomic<int> regs_of[4];
    const int bi = build == kFmtQ4 ? 0 : build == kFmtQ8 ? 1 : build == kFmtE4M3 ? 2 : 3;
    int own_regs = regs_of[bi].load(std::memory_order_acquire);
    if (own_regs == 0) {
        cudaFuncAttributes fa = {};
        const cudaError_t e =
            bi == 0   ? cudaFuncGetAttributes(&fa, xs_qgemm_kernel<kFmtQ4>)
            : bi == 1 ? cudaFuncGetAttributes(&fa, xs_qgemm_kernel<kFmtQ8>)
            : bi == 2 ? cudaFuncGetAttributes(&fa, xs_qgemm_kernel<kFmtE4M3>)
                      : cudaFuncGetAttributes(&fa, xs_qgemm_kernel<kFmtMixed>);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        own_regs = fa.numRegs;
        regs_of[bi].store(own_regs, std::memory_order_release);
    }
    int dev = 0, sm_regs = 0, sm_smem = 0, sm_threads = 0, reserved = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sm_regs, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sm_threads, cudaDevAttrMaxThreadsPerMultiProcessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    // registers are allocated per warp in units of 8 a thread and split
    // between the SM's four sub-partitions, over which a block's warps spread
    auto warp_regs = [](int r) { return (r + 7) / 8 * 8 * 32; };
    const int own_warps = kXsThreads / 32, other_warps = (threads + 31) / 32;
    const int per_sub = (own_warps + 3) / 4 * warp_regs(own_regs) +
                        (other_warps + 3) / 4 * warp_regs(regs);
    const int smem = xs_layout(build, k_max).total + 1024 + 2 * reserved;
    return per_sub <= sm_regs / 4 && smem <= sm_smem && kXsThreads + threads <= sm_threads;
}

cudaError_t launch_xs_group(const XsInput *in, int count, int M, DevCtl *ctl, cudaStream_t s) {
    if (!xs_group_supported(in, count, M)) return cudaErrorInvalidValue;
    bool mixed = false;
    int k_max = 0;
    for (int i = 0; i < count; ++i) {
        mixed = mixed || in[i].fmt != in[0].fmt;
        k_max = std::max(k_max, in[i].K);
    }
    const int build = mixed ? kFmtMixed : in[0].fmt;
    XsParams P = {};
    P.count = count;
    P.M = M;
    P.n_m = (M + kXsTileM - 1) / kXsTileM;
    int items = 0;
    for (int i = 0; i < count; ++i) {
        if (!xs_problem(P.p[i], in[i], build, M)) return cudaErrorInvalidValue;
        P.p[i].item0 = items;
        items += P.n_m * P.p[i].n_o;
    }
    P.n_items = items;
    if (build == kFmtQ4) return launch_xs_build<kFmtQ4>(P, k_max, ctl, s);
    if (build == kFmtQ8) return launch_xs_build<kFmtQ8>(P, k_max, ctl, s);
    if (build == kFmtE4M3) return launch_xs_build<kFmtE4M3>(P, k_max, ctl, s);
    return launch_xs_build<kFmtMixed>(P, k_max, ctl, s);
}

cudaError_t launch_xs(int fmt, const void *Xh, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s) {
    const XsInput in = {fmt, Xh, Wq, S, bias, Y, N, K};
    return launch_xs_group(&in, 1, M, ctl, s);
}

}  // namespace rtq
