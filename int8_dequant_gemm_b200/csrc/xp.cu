// tcgen05 path for many activation rows and short K (K <= 512) on CTA pairs:
// the activation-resident design of xs.cu with one MMA over two SMs
// (cta_group::2), which halves the activation block each SM keeps and leaves
// room to round the fp32 activations to fp16 inside the kernel.
//
// Tile product, as in tc.cu / xs.cu: D[o, m] = sum_k W_hat[o, k] * X[m, k],
// here with 256 weight rows as the MMA's M dimension (128 per CTA: rank r of
// the pair holds weight tile 2 * op + r of item op) and 192 activation rows as
// its N dimension (96 per CTA: rank r holds rows m0 + 96 r .. m0 + 96 r + 95 of
// the block m0 = 192 * m_tile, all of K, as fp16 in the 128-byte-swizzled
// operand layout, 96 x K x 2 bytes).  Each CTA's TMEM holds D for its own 128
// weight rows and all 192 activation rows, so each CTA stores its own part of
// Y.  Per SM the MMA work, the dequantization and the Y stores are those of
// xs.cu; the resident activations and their loads are halved.
//
// Activations: fp32 X goes straight from HBM into a ring of staging slots by
// TMA (96 rows x 32 values per box), and at every change of activation block
// the epilogue warps round it to fp16 into the resident tile (those warps are
// idle there: the block's first tile needs the activations, and the last
// tile of the previous block has been stored).  The staging TMA runs ahead,
// so the next block's first boxes are already in shared memory.
//
// The plan takes this kernel from 16384 activation rows up (kXpMinM): the
// pair interval is the dequantizers' one, as in xs.cu, so what it saves is
// the pre-pass's traffic and launch, and at a few items per CTA the rounding
// of the first block costs more than that.
//
// Work list: (activation block, weight-tile pair) items in activation-major
// order, one contiguous run per pair.  Roles, in each CTA of the pair (20
// warps):
//   warps 0-7   dequantizers (as in xs.cu), into this CTA's TMEM A stages;
//               one lane per warp arrives on the even CTA's a_full.
//   warp 8      MMA issuer, even CTA only: 8 tcgen05.mma.cta_group::2 per pair
//               of K steps; commits go to both CTAs (multicast).
//   warps 9-16  epilogue (this CTA's 128 weight rows x 192 activation rows)
//               and activation rounding; one lane per warp arrives on the
//               even CTA's acc_empty and x_full.
//   warp 17     weight TMA (this CTA's weight tile).
//   warp 18     activation staging TMA.
//   warp 19     MMA waiter, even CTA only (as in xs.cu).
// The arrivals that cross to the even CTA use the default (CTA-scope)
// release: a cluster-scope release costs about as much as a cluster-wide
// fence, 1.5K cycles per stage, measured; each signal follows either
// tcgen05.wait::st with tcgen05.fence::before_thread_sync (TMEM data), a
// proxy fence after the shared-memory writes the peer's MMA reads, or reads
// that are complete, as in the usual pairing of a 2-SM MMA's producers with
// its issuing CTA.
//
// Every mbarrier wait is bounded; a wait that gives up latches
// RT_ERR_DEVICE_TIMEOUT and the CTAs wind down: the TMA threads wait (bounded)
// for the copies they issued, the MMA thread for the MMAs it issued, and both
// CTAs meet at a cluster barrier before either releases TMEM or exits, since
// the even CTA's MMAs read the odd CTA's shared memory and TMEM.
#include <algorithm>

#include "kernels.cuh"
#include "tmapipe.cuh"

namespace rtq {
namespace {

// 192 activation rows per block fill TMEM with two accumulators and two A
// stages (2 x 192 + 2 x 64 columns); 160 rows with three A stages and 128
// rows with four measured 6 % and 13 % slower at M = 65536 (the pair
// interval is the dequantizers', so narrower tiles only add items).
constexpr int kXpBlockRows = 192;                        // activation rows per block (MMA N)
constexpr int kXpHalfRows = kXpBlockRows / 2;            // per CTA
constexpr int kXpMaxK = 512;
constexpr int kXAtoms = kXpMaxK / 64;                    // 64-wide K atoms of a resident block
constexpr int kXPairs = kXAtoms / 2;
constexpr int kDeqGroups = 2;
constexpr int kDeqThreads = kTileRows;                   // 128 per K half
constexpr int kDeqWarps = kDeqGroups * 4;                // 8
constexpr int kMmaWarp = kDeqWarps;                      // 8
constexpr int kEpiWarp0 = kMmaWarp + 1;                  // 9
constexpr int kEpiWarps = 8;                             // two per TMEM lane quadrant
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kEpiCols = kXpBlockRows / 2;               // columns per epilogue warp (x16 tail)
constexpr int kWTmaWarp = kEpiWarp0 + kEpiWarps;         // 17
constexpr int kXTmaWarp = kWTmaWarp + 1;                 // 18
constexpr int kWaitWarp = kXTmaWarp + 1;                 // 19
constexpr int kXpThreads = (kWaitWarp + 1) * 32;         // 640
constexpr uint32_t kMmaBar = 1;                          // named barrier: waiter <-> MMA warp
constexpr int kXAtom = kXpHalfRows * 128;                // 12 KB: 96 rows x 64 K (fp16)
constexpr int kStgBox = kXpHalfRows * 128;               // 12 KB: 96 rows x 32 K (fp32)
constexpr int kStg = 8;                                  // staging ring (boxes)
constexpr int kAStages = 2;                              // A stages in TMEM, two K steps each
constexpr int kRaw = 2;                                  // packed-code ring depth (step pairs)
constexpr uint32_t kAccCols = 2 * kXpBlockRows;          // 2 accumulators x 192 columns
constexpr uint32_t kAStageCols = kAtomK;                 // 2 x 64 16-bit values per lane
constexpr uint32_t kXpTmemCols = 512;
constexpr uint16_t kBoth = 3;                            // multicast mask: both CTAs
constexpr int kCvtChunks = 2 * kXpHalfRows * 4;          // 16-byte chunks per atom
constexpr int kCvtPerThread = (kCvtChunks + kEpiThreads - 1) / kEpiThreads;

static_assert(kAccCols + kAStages * kAStageCols <= kXpTmemCols, "TMEM budget");
static_assert(kEpiCols % 16 == 0, "epilogue reads 32 columns at a time, then 16");
static_assert(kXpHalfRows % 8 == 0 && kXpBlockRows % 32 == 0, "MMA N and swizzle groups");
static_assert(kXAtom % 1024 == 0 && kStgBox % 1024 == 0, "swizzle atoms stay aligned");
static_assert(kStg >= 4, "the rounding waits for the four staging boxes of a K pair");

constexpr int kScaleWords = 16;
__host__ __device__ constexpr int raw_slot_bytes(int fmt) { return kTileRows * (fmt == 4 ? 64 : 128); }
__host__ __device__ constexpr int scale_slot_bytes(int fmt) {
    return fmt == 4 ? kTileRows * kScaleWords * 4 : 0;
}

struct XpLayout {
    int x_off, stg_off, raw_off, sc_off, bar_off, total;
};

__host__ __device__ inline XpLayout xp_layout(int fmt, int K) {
    XpLayout L;
    L.x_off = 0;
    L.stg_off = (K / kAtomK) * kXAtom;
    L.raw_off = L.stg_off + kStg * kStgBox;
    L.sc_off = L.raw_off + kRaw * raw_slot_bytes(fmt);
    L.bar_off = L.sc_off + 2 * scale_slot_bytes(fmt);
    // raw_full/empty[kRaw], sc_full/empty[2], a_full/empty[kAStages],
    // stg_full/empty[kStg], x_full[kXPairs], acc_full/empty[2], drain,
    // + TMEM address slot
    L.total = L.bar_off +
              (2 * kRaw + 4 + 2 * kAStages + 2 * kStg + kXPairs + 4 + 1) * 8 + 16;
    return L;
}

struct ItemCursor {
    int item, last, m_tile, op, n_op;
    __device__ ItemCursor(int first, int last_, int n_op_)
        : item(first), last(last_), m_tile(first / n_op_), op(first % n_op_), n_op(n_op_) {}
    __device__ bool valid() const { return item < last; }
    __device__ void next() {
        ++item;
        if (++op == n_op) {
            op = 0;
            ++m_tile;
        }
    }
};

// Epilogue threads (et = 0 .. 255): round one 64-wide K atom of this CTA's 96
// activation rows from the two fp32 staging boxes s0 (K values 0..31 of the
// atom) and s1 (32..63) into the resident tile's atom `xa`.  Staging boxes
// are 96 rows of 128 bytes in the 128-byte swizzle (16-byte chunk j of row r
// at j ^ (r & 7)); chunk (r, c) of the resident atom holds the 8 values
// 8c .. 8c+7 in the operand order at c ^ (r & 7).  A quarter warp reads rows
// r, r + 1 (r even) of one box, which puts its eight 16-byte reads on eight
// different bank groups.  Returns non-zero for a value that is not a finite
// fp16 number after rounding.
__device__ __forceinline__ uint32_t round_atom(uint32_t s0, uint32_t s1, uint32_t xa, int et) {
    uint32_t bad = 0;
#pragma unroll
    for (int i = 0; i < kCvtPerThread; ++i) {
        const int u = et + kEpiThreads * i;                 // 0 .. kCvtChunks - 1
        if (kCvtChunks % kEpiThreads != 0 && u >= kCvtChunks) break;
        const int h = u / (kXpHalfRows * 4);                // which box
        const int v = u - h * (kXpHalfRows * 4);
        const int r = v >> 2, cc = v & 3;
        const uint32_t row = (h ? s1 : s0) + static_cast<uint32_t>(r * 128);
        const uint32_t sw = static_cast<uint32_t>(r & 7);
        const uint4 a = lds_v4(row + (((2u * cc) ^ sw) << 4));
        const uint4 b = lds_v4(row + (((2u * cc + 1u) ^ sw) << 4));
        const float4 fa = make_float4(__uint_as_float(a.x), __uint_as_float(a.y),
                                      __uint_as_float(a.z), __uint_as_float(a.w));
        const float4 fb = make_float4(__uint_as_float(b.x), __uint_as_float(b.y),
                                      __uint_as_float(b.z), __uint_as_float(b.w));
        const uint4 w = x8_f16(fa, fb);
        bad |= f16x2_nonfinite(make_uint2(w.x, w.y)) | f16x2_nonfinite(make_uint2(w.z, w.w));
        const uint32_t c = static_cast<uint32_t>(4 * h + cc);
        sts_v4(xa + static_cast<uint32_t>(r * 128) + ((c ^ sw) << 4), w);
    }
    return bad;
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
__global__ void __launch_bounds__(kXpThreads, 1)
    xp_qgemm_kernel(const __grid_constant__ CUtensorMap w_map,
                    const __grid_constant__ CUtensorMap s_map,
                    const __grid_constant__ CUtensorMap x_map, const float *__restrict__ S8,
                    const float *__restrict__ bias, float *__restrict__ Y, int M, int N, int K,
                    int n_op, int n_items, DevCtl *ctl) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const XpLayout L = xp_layout(FMT, K);
    constexpr int kRawSlot = raw_slot_bytes(FMT);
    constexpr int kScaleSlot = scale_slot_bytes(FMT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *raw_full = bars;
    uint64_t *raw_empty = raw_full + kRaw;
    uint64_t *sc_full = raw_empty + kRaw;
    uint64_t *sc_empty = sc_full + 2;
    uint64_t *a_full = sc_empty + 2;              // even CTA's: 2 x 256 arrivals
    uint64_t *a_empty = a_full + kAStages;        // each CTA's: one multicast commit
    uint64_t *stg_full = a_empty + kAStages;
    uint64_t *stg_empty = stg_full + kStg;
    uint64_t *x_full = stg_empty + kStg;          // even CTA's: 2 x 256 arrivals per K pair
    uint64_t *acc_full = x_full + kXPairs;        // each CTA's: one multicast commit
    uint64_t *acc_empty = acc_full + 2;           // even CTA's: 2 x 256 arrivals
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *mma_abort = tmem_slot + 1;
    const unsigned long long *lim = &ctl->wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int nk = K / kAtomK;
    const int pairs = gridDim.x / 2;
    const int pid = blockIdx.x / 2;
    const int first = static_cast<int>((static_cast<long long>(pid) * n_items) / pairs);
    const int last = static_cast<int>((static_cast<long long>(pid + 1) * n_items) / pairs);
    // the even CTA's copies of the barriers both CTAs arrive on
    auto at_leader = [](uint64_t *bar) { return cluster_map(smem_addr(bar), 0); };

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRaw; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], kDeqGroups * kDeqThreads);
        }
        // the barriers both CTAs arrive on take one arrival per warp (an
        // elected lane after __syncwarp), which keeps the cross-SM arrivals
        // at 8 per CTA and stage
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sc_full[b], 1);
            mbar_init(&sc_empty[b], kDeqGroups * kDeqThreads);
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * kEpiWarps);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], 2 * kDeqWarps);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < kStg; ++s) {
            mbar_init(&stg_full[s], 1);
            mbar_init(&stg_empty[s], kEpiThreads);
        }
        for (int p = 0; p < kXPairs; ++p) mbar_init(&x_full[p], 2 * kEpiWarps);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, kXpTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    // both CTAs' barriers exist and their TMEM is allocated before either
    // arrives remotely or issues an MMA
    cluster_sync();
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
            int j = 0, n_sc = 0;
            for (ItemCursor it(first, last, n_op); it.valid() && ok; it.next()) {
                const int n_local = it.item - first;
                const int y0 = (2 * it.op + static_cast<int>(rank)) * kTileRows;
                if (FMT == 4) {
                    const int b = n_local & 1;
                    if (n_local >= 2 &&
                        !mbar_wait(&sc_empty[b], static_cast<uint32_t>((n_local / 2) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&sc_full[b], kTileRows * kScaleWords * 4);
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
                    mbar_expect_tx(&raw_full[slot], kRawSlot);
                    tma_load_2d(base + L.raw_off + slot * kRawSlot, &w_map,
                                p * (FMT == 4 ? 64 : 128), y0, &raw_full[slot]);
                }
            }
            for (int i = 0; i < kRaw && i < j; ++i) {
                const int last_j = i + ((j - 1 - i) / kRaw) * kRaw;
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
        // ============================================================ activation staging TMA
        // For each activation block in the run: 2 * nk boxes of 96 rows x 32
        // fp32 values (this CTA's half of the block), in atom order, through
        // the staging ring; rows past M read as zero.
        if (lane == 0) {
            pdl_wait_prior_grid();     // X may be the output of the previous kernel
            int cur_m = -1, j = 0;
            for (ItemCursor it(first, last, n_op); it.valid() && ok; it.next()) {
                if (it.m_tile == cur_m) continue;
                cur_m = it.m_tile;
                const int y0 = cur_m * kXpBlockRows + static_cast<int>(rank) * kXpHalfRows;
                for (int q = 0; q < 2 * nk; ++q, ++j) {
                    const int slot = j % kStg;
                    if (j >= kStg &&
                        !mbar_wait(&stg_empty[slot], static_cast<uint32_t>((j / kStg) - 1) & 1u,
                                   lim)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&stg_full[slot], kStgBox);
                    tma_load_2d(base + L.stg_off + slot * kStgBox, &x_map, q * 32, y0,
                                &stg_full[slot]);
                }
            }
            for (int i = 0; i < kStg && i < j; ++i) {
                const int last_j = i + ((j - 1 - i) / kStg) * kStg;
                mbar_wait(&stg_full[i], static_cast<uint32_t>(last_j / kStg) & 1u, lim);
            }
        }
        __syncwarp();
    } else if (warp < kDeqWarps) {
        // ============================================================ dequantizers
        const int h = warp >> 2;
        const int r = threadIdx.x & (kDeqThreads - 1);
        const uint32_t ta = tmem + kAccCols + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                            static_cast<uint32_t>(32 * h);
        uint32_t jp = 0;
        for (ItemCursor it(first, last, n_op); it.valid() && ok; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            uint32_t sw[kScaleWords / 2] = {};
            // every wait's outcome is made warp-uniform: the TMEM stores and the
            // per-warp arrival below need the whole warp
            if (FMT == 4) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&sc_full[b], static_cast<uint32_t>(n_local / 2) & 1u, lim));
                if (!ok) break;
                load_scale_pairs(base + L.sc_off + b * kScaleSlot + r * (kScaleWords * 4), r, h, sw);
                fence_proxy_async_smem();
                mbar_arrive(&sc_empty[b]);
            }
#pragma unroll
            for (int kp = 0; kp < kXpMaxK / kAtomK / 2; ++kp, ++jp) {
                if (2 * kp >= nk) break;
                const uint32_t jr = n_local * (nk / 2) + kp;
                const int slot = jr % kRaw;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&raw_full[slot], static_cast<uint32_t>(jr / kRaw) & 1u, lim));
                if (!ok) break;
                const uint32_t raw = base + L.raw_off + slot * kRawSlot;
                uint32_t w0[16], w1[16];
                half_words<FMT>(load_half_raw2<FMT>(raw, r, 0, h, sw[2 * kp]), w0);
                half_words<FMT>(load_half_raw2<FMT>(raw, r, 1, h, sw[2 * kp + 1]), w1);
                fence_proxy_async_smem();
                mbar_arrive(&raw_empty[slot]);
                const uint32_t st = jp % kAStages;
                if (jp >= kAStages) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&a_empty[st], ((jp / kAStages) - 1) & 1u, lim));
                    if (!ok) break;
                }
                tc_fence_after_sync();
                tmem_st_x16(ta + st * kAStageCols, w0);
                tmem_st_x16(ta + st * kAStageCols + 16, w1);
                tmem_st_wait();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(at_leader(&a_full[st]));
            }
            if (!ok) break;
        }
    } else if (warp == kWaitWarp) {
        // ============================================================ MMA waiter (even CTA)
        if (leader) {
            int cur_m = -1, x_loads = 0;
            uint32_t j = 0;
            for (ItemCursor it(first, last, n_op); it.valid() && ok; it.next()) {
                const int n_local = it.item - first;
                const int b = n_local & 1;
                bool good = true;
                const bool fresh = it.m_tile != cur_m;
                if (fresh) {
                    cur_m = it.m_tile;
                    ++x_loads;
                }
                const uint32_t xpar = static_cast<uint32_t>(x_loads - 1) & 1u;
                if (lane == 0 && n_local >= 2)
                    good = mbar_wait(&acc_empty[b], static_cast<uint32_t>((n_local / 2) - 1) & 1u,
                                     lim);
                for (int kp = 0; 2 * kp < nk; ++kp, ++j) {
                    if (lane == 0) {
                        if (good && fresh) good = mbar_wait(&x_full[kp], xpar, lim);
                        if (good)
                            good = mbar_wait(&a_full[j % kAStages], (j / kAStages) & 1u, lim);
                        mma_abort[j & 1] = good ? 0u : 1u;
                    }
                    named_bar_sync(kMmaBar, 64);
                    if (__shfl_sync(0xffffffffu, good ? 1 : 0, 0) == 0) {
                        ok = false;
                        break;
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer (even CTA)
        if (leader) {
            const uint32_t idesc = idesc_f16_f32acc(2 * kTileRows, kXpBlockRows);
            constexpr uint64_t kXAtomDesc = kXAtom >> 4;
            const uint64_t bdesc0 = sw128_kmajor_desc(base + L.x_off);
            uint32_t j = 0;
            bool abort = false;
            for (ItemCursor it(first, last, n_op); it.valid() && !abort; it.next()) {
                const int n_local = it.item - first;
                const int b = n_local & 1;
                const uint32_t d = tmem + static_cast<uint32_t>(b * kXpBlockRows);
                uint64_t bdesc = bdesc0;
                for (int kp = 0; 2 * kp < nk; ++kp, ++j, bdesc += 2 * kXAtomDesc) {
                    named_bar_sync(kMmaBar, 64);
                    if (mma_abort[j & 1]) {
                        abort = true;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t at = tmem + kAccCols + (j % kAStages) * kAStageCols;
                    if (elect_one()) {
#pragma unroll
                        for (int u = 0; u < 2; ++u)
#pragma unroll
                            for (int kk = 0; kk < kAtomK / 16; ++kk)
                                tc_mma_pair_ts(d, at + 32 * u + 8 * kk,
                                               bdesc + u * kXAtomDesc + 2 * kk, idesc,
                                               (kp > 0 || u > 0 || kk > 0) ? 1u : 0u);
                        tc_commit_pair_mc(&a_empty[j % kAStages], kBoth);
                    }
                    __syncwarp();
                }
                if (abort) break;
                if (elect_one()) tc_commit_pair_mc(&acc_full[b], kBoth);
                __syncwarp();
            }
            if (abort && lane == 0) {
                tc_commit_pair_mc(drain, 1);
                mbar_wait(drain, 0, lim);
            }
            __syncwarp();
        }
    } else {
        // ============================================================ epilogue + rounding
        const int q = warp & 3;
        const int c0 = ((warp - kEpiWarp0) >> 2) * kEpiCols;
        const int row = q * 32 + lane;
        const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const int et = threadIdx.x - kEpiWarp0 * 32;
        uint32_t xbad = 0;
        int cur_m = -1, js = 0;                         // js: staging boxes consumed
        for (ItemCursor it(first, last, n_op); it.valid() && ok; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            if (it.m_tile != cur_m) {
                // First item of an activation block.  This thread has waited
                // for the accumulator of every earlier item, and each of
                // those commits follows all MMAs issued before it, so no MMA
                // still reads either CTA's resident tile.
                cur_m = it.m_tile;
                // one 128-wide K pair (atoms 2p and 2p + 1, staging boxes js ..
                // js + 3) at a time: one wait, one proxy fence and one arrival
                // on x_full[p] per pair
                for (int p = 0; 2 * p < nk && ok; ++p, js += 4) {
                    bool got = true;
#pragma unroll
                    for (int bx = 0; bx < 4; ++bx)
                        got = got && mbar_wait(&stg_full[(js + bx) % kStg],
                                               static_cast<uint32_t>((js + bx) / kStg) & 1u, lim);
                    ok = __all_sync(0xffffffffu, got);
                    if (!ok) break;
                    const uint32_t stg = base + L.stg_off;
                    xbad |= round_atom(stg + (js % kStg) * kStgBox, stg + ((js + 1) % kStg) * kStgBox,
                                       base + L.x_off + (2 * p) * kXAtom, et);
                    xbad |= round_atom(stg + ((js + 2) % kStg) * kStgBox,
                                       stg + ((js + 3) % kStg) * kStgBox,
                                       base + L.x_off + (2 * p + 1) * kXAtom, et);
                    // staging reads done (ordered before the TMA refill), resident
                    // writes ordered before the tensor core's reads
                    fence_proxy_async_smem();
#pragma unroll
                    for (int bx = 0; bx < 4; ++bx) mbar_arrive(&stg_empty[(js + bx) % kStg]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(at_leader(&x_full[p]));
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            ok = mbar_wait(&acc_full[b], static_cast<uint32_t>(n_local / 2) & 1u, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            const int m0 = it.m_tile * kXpBlockRows;
            const int o = (2 * it.op + static_cast<int>(rank)) * kTileRows + row;
            float sc = 1.f, bo = 0.f;
            if (FMT == 8 && o < N) sc = __ldg(S8 + o);
            if (bias && o < N) bo = __ldg(bias + o);
            const int mlim = min(kXpBlockRows, M - m0);
            float *yo = Y + static_cast<size_t>(m0) * N + o;
            const size_t rs = static_cast<size_t>(N);
            const uint32_t tb = tq + static_cast<uint32_t>(b * kXpBlockRows);
            int c = c0;
            for (; c + 32 <= c0 + kEpiCols; c += 32) {
                uint32_t v[32];
                tmem_ld_x32(tb + static_cast<uint32_t>(c), v);
                tmem_ld_wait();
                if (o < N) store_cols(yo + static_cast<size_t>(c) * rs, rs, v, mlim - c, sc, bo);
            }
            if (c < c0 + kEpiCols) {                    // kEpiCols an odd multiple of 16
                uint32_t v[16];
                tmem_ld_x16(tb + static_cast<uint32_t>(c), v);
                tmem_ld_wait();
                if (o < N) store_cols(yo + static_cast<size_t>(c) * rs, rs, v, mlim - c, sc, bo);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(at_leader(&acc_empty[b]));
        }
        if (__any_sync(0xffffffffu, xbad != 0) && lane == 0)
            atomicOr(&ctl->status, 1u << kStatusRange);
    }
    if (!ok) atomicOr(&ctl->status, 1u << kStatusTimeout);
    tc_fence_before_sync();
    // neither CTA releases TMEM or shared memory while the pair's MMAs may
    // still read them
    cluster_sync();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, kXpTmemCols);
    }
}

template <int FMT>
cudaError_t launch_xp_fmt(const float *X, const void *Wq, const void *S, const float *bias,
                          float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t st) {
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(xp_qgemm_kernel<FMT>, 227 * 1024, dev, attr_done)) != cudaSuccess)
        return e;
    CUtensorMap w_map, s_map, x_map;
    bool enc_ok = encode_tma_2d(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, X, K, M, 32,
                                CU_TENSOR_MAP_SWIZZLE_128B, kXpHalfRows);
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
    const int n_o = (N + kTileRows - 1) / kTileRows;
    const int n_op = (n_o + 1) / 2;
    const int n_m = (M + kXpBlockRows - 1) / kXpBlockRows;
    const int items = n_op * n_m;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kXpThreads, 1, 1);
    cfg.dynamicSmemBytes = xp_layout(FMT, K).total + 1024;
    cfg.stream = st;
    static std::atomic<int> pairs_cache[kMaxDevices];
    const int pairs = resident_pairs(xp_qgemm_kernel<FMT>, cfg, dev, pairs_cache);
    cfg.gridDim = dim3(2 * std::min(items, pairs), 1, 1);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, xp_qgemm_kernel<FMT>, w_map, s_map, x_map,
                              static_cast<const float *>(S), bias, Y, M, N, K, n_op, items, ctl);
}

}  // namespace

cudaError_t launch_xp(int fmt, const float *X, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s) {
    if (fmt == kFmtQ4) return launch_xp_fmt<kFmtQ4>(X, Wq, S, bias, Y, M, N, K, ctl, s);
    if (fmt == kFmtQ8) return launch_xp_fmt<kFmtQ8>(X, Wq, S, bias, Y, M, N, K, ctl, s);
    return launch_xp_fmt<kFmtE4M3>(X, Wq, S, bias, Y, M, N, K, ctl, s);
}

}  // namespace rtq
