// tcgen05 path for a LIST of independent projections that share a small M
// (1..128 activation rows): one persistent launch streams every projection's
// packed weights through each SM back to back.
//
// A single small-M projection moves well under a megabyte of weights, less
// than one launch's latency worth of HBM time, so its cost is its dependency
// chain, not its bytes.  Here the chains of many projections overlap: every
// CTA (one per SM) walks a list of work items -- up to a few 128-row weight
// tiles of one projection each -- while a ring of weight slots keeps the
// next tiles' codes in flight, TMEM holds a ring of accumulators so one
// tile's epilogue overlaps the next tile's MMAs, and the activation block of
// the current projection stays resident in shared memory across every item
// that reads the same activations.
//
// Tile product as in the other tcgen05 kernels (weight-stationary,
// transposed): D[o, m] = sum_k W_hat[o, k] * X[m, k] with the 128 weight rows
// as the MMA's M dimension and BNp = M rounded up to 16 activation rows as its
// N dimension; fp16 operands, fp32 accumulation in TMEM.
//
// Data movement per CTA:
//   weights  cp.async (16 bytes per thread) of one slot = 128 rows x 256
//            bytes of codes (q4: K 512, q8: K 256) plus, for q4, the rows'
//            (scale, min) words, into a ring of slots in an XOR-swizzled
//            layout: 16-byte chunk c of row r sits at chunk (c & 8) |
//            ((c & 7) ^ (r & 7)), so the dequantizers' reads of one chunk
//            over 8 consecutive rows hit 8 different bank groups.  The slot
//            completes on an mbarrier through cp.async.mbarrier.arrive.
//   activations  one bulk copy per 512-wide K chunk of the projection's fp16
//            image (written by pl_prep_kernel below in the 128-byte-swizzled
//            operand layout) into the resident activation buffer, reloaded
//            only when the (activations, K chunk) pair changes.
// Roles (21 warps):
//   warps 0-7   dequantizers: thread (r, h) converts K values [32h, 32h+32) of
//               every 64-wide K step of row r into TMEM lane r of the step's A
//               stage (tcgen05.st), as in the activation-resident kernel.
//   warp 8      MMA issuer, fed through named barrier 1 by
//   warp 9      the MMA waiter, which performs all of the issuer's waits.
//   warps 10-17 epilogue: TMEM -> registers (q8 row scale) -> fp32 Y.
//   warps 18-19 weight producers (cp.async).
//   warp 20     activation loader (one thread, bulk copies).
// Work items longer than one 512-wide K chunk (K > 512) run chunk by chunk
// over all their tiles (each tile in its own accumulator), so one resident
// activation chunk serves every tile of the item.
//
// Work distribution (host, launch_pl): items are cut from the projections
// (at most 4 tiles, or as many as the accumulator ring holds when K > 512),
// assigned largest first to the least loaded CTA, and each CTA's items are
// ordered by their activation buffer so that the resident block is reloaded
// as rarely as possible.  Every tile is computed by one CTA from start to
// end, so results do not depend on the assignment.
//
// Every mbarrier wait is bounded; a wait that gives up latches
// RT_ERR_DEVICE_TIMEOUT and the CTA winds down: copies it issued complete,
// MMAs it issued drain, TMEM is released.
#include <algorithm>
#include <numeric>
#include <vector>

#include "kernels.cuh"
#include "pl.cuh"
#include "tmapipe.cuh"

namespace rtq {
namespace {

constexpr int kDeqWarps = 8;
constexpr int kIssuerWarp = 8;
constexpr int kWaiterWarp = 9;
constexpr int kEpiWarp0 = 10;
constexpr int kEpiWarps = 8;
constexpr int kProdWarp0 = 18;
constexpr int kProdWarps = 2;
constexpr int kXWarp = 20;
constexpr int kPlThreads = (kXWarp + 1) * 32;        // 672
constexpr int kProdThreads = kProdWarps * 32;        // 64
constexpr int kEpiThreads = kEpiWarps * 32;          // 256
constexpr uint32_t kMmaBar = 1;                      // named barrier: waiter <-> issuer
constexpr uint32_t kEpiBar = 2;                      // named barrier: the epilogue warps
constexpr int kSlotBytes = 32 * 1024;                // 128 rows x 256 bytes of codes
constexpr int kScaleBytes = 8 * 1024;                // 128 rows x 16 (scale, min) words
constexpr int kMaxSlots = 4;
constexpr int kAStages = 4;
constexpr uint32_t kAStageCols = 32;
constexpr uint32_t kAOff = 384;                      // A stages at TMEM columns [384, 512)
constexpr int kXChunk = 512;                         // K of one resident activation chunk

// K covered by one weight slot (256 bytes of codes per row).
__host__ __device__ constexpr int slot_k(int fmt) { return fmt == 4 ? 512 : 256; }

struct PlLayout {
    int x_off, w_off, s_off, bar_off, total;
};

__host__ __device__ inline PlLayout pl_layout(int bnp, int nslots) {
    PlLayout L;
    L.x_off = 0;
    L.w_off = bnp * kXChunk * 2;
    L.s_off = L.w_off + nslots * kSlotBytes;
    L.bar_off = L.s_off + nslots * kScaleBytes;
    // slot full/empty, A full/empty, x full/empty, acc full/empty, drain, then
    // 8 words: TMEM address, 2 issuer abort flags, the epilogue's flags
    L.total = L.bar_off + (2 * kMaxSlots + 2 * kAStages + 2 + 2 * kPlMaxAcc + 1) * 8 + 32;
    return L;
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Arrives on `bar` once every cp.async this thread issued so far has landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Physical 16-byte chunk of logical chunk c (0..15) of slot row r.
__device__ __forceinline__ int wswz(int c, int r) { return (c & 8) | ((c & 7) ^ (r & 7)); }
// Physical 16-byte chunk of logical scale chunk c (0..3) of row r.
__device__ __forceinline__ int sswz(int c, int r) { return c ^ ((r >> 1) & 3); }

// The walk every role takes through a CTA's items: item (one K chunk of a
// few tiles) -> tile -> weight slot -> 64-wide K step.  Each role advances it
// at its own grain.
struct Item {
    const PlProj *p;
    int tile0, ntiles, chunk, nchunks;
};

__device__ __forceinline__ Item item_at(const PlParams &P, int i) {
    const PlItem &it = P.items[i];
    Item r;
    r.p = &P.proj[it.proj];
    r.tile0 = static_cast<int>(it.tile0);
    r.ntiles = it.ntiles;
    r.chunk = it.chunk;
    r.nchunks = (r.p->K + kXChunk - 1) / kXChunk;
    return r;
}

// K range [k0, k0 + len) of slot w of chunk c; 0 if the slot lies past K.
__device__ __forceinline__ int slot_len(const PlProj &p, int c, int w, int &k0) {
    k0 = c * kXChunk + w * slot_k(p.fmt);
    return max(0, min(slot_k(p.fmt), p.K - k0));
}

__device__ __forceinline__ int slots_in_chunk(const PlProj &p, int c) {
    const int len = min(kXChunk, p.K - c * kXChunk);
    return (len + slot_k(p.fmt) - 1) / slot_k(p.fmt);
}

template <int FMT>
__device__ __forceinline__ void dequant_slot(uint32_t wslot, uint32_t sslot, int r, int h, int s,
                                             uint32_t (&w)[16]) {
    HalfRaw R;
    if (FMT == 4) {
        R.p0 = lds_v4(wslot + r * 256 + wswz(2 * s + h, r) * 16);
        R.p1 = make_uint4(0, 0, 0, 0);
        // (scale, min) word 2s + h of the row: chunk s >> 1, word (2s + h) & 3
        const uint4 sc = lds_v4(sslot + r * 64 + sswz(s >> 1, r) * 16);
        const int wi = (2 * s + h) & 3;
        R.smw = wi == 0 ? sc.x : wi == 1 ? sc.y : wi == 2 ? sc.z : sc.w;
        half_words<4>(R, w);
    } else {   // q8 and e4m3: one byte per weight
        R.p0 = lds_v4(wslot + r * 256 + wswz(4 * s + 2 * h, r) * 16);
        R.p1 = lds_v4(wslot + r * 256 + wswz(4 * s + 2 * h + 1, r) * 16);
        R.smw = 0;
        half_words<FMT>(R, w);
    }
}

__global__ void __launch_bounds__(kPlThreads, 1)
    pl_qgemm_kernel(const __grid_constant__ PlParams P, DevCtl *ctl) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const int BNp = P.bnp, M = P.M, NS = P.nslots, R = P.nacc;
    const PlLayout L = pl_layout(BNp, NS);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *slot_full = bars;
    uint64_t *slot_empty = slot_full + kMaxSlots;
    uint64_t *a_full = slot_empty + kMaxSlots;
    uint64_t *a_empty = a_full + kAStages;
    uint64_t *x_full = a_empty + kAStages;
    uint64_t *x_empty = x_full + 1;
    uint64_t *acc_full = x_empty + 1;
    uint64_t *acc_empty = acc_full + kPlMaxAcc;
    uint64_t *drain = acc_empty + kPlMaxAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *mma_abort = tmem_slot + 1;       // waiter -> issuer, per step parity
    const unsigned long long *lim = &ctl->wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i_first = P.cta_items[blockIdx.x], i_last = P.cta_items[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSlots; ++s) {
            mbar_init(&slot_full[s], kProdThreads);
            mbar_init(&slot_empty[s], kDeqWarps * 32);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], kDeqWarps * 32);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(x_full, 1);
        mbar_init(x_empty, 1);
        for (int b = 0; b < kPlMaxAcc; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiThreads);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // The next launch in the stream may start its own weight prefetch now.
    pdl_launch_dependents();
    bool ok = true;

    if (warp >= kProdWarp0 && warp < kProdWarp0 + kProdWarps) {
        // ======================================================= weight producers
        // Packed weights do not depend on the previous kernel in the stream.
        // (Test hook: with `inject`, thread 0 leaves out its arrival on the
        // first slot, so the dequantizers' wait for it runs out.)
        const int t = threadIdx.x - kProdWarp0 * 32;
        int j = 0;
        for (int i = i_first; i < i_last && ok; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = *it.p;
            const int fmt = p.fmt, c = it.chunk;
            const size_t row_stride = fmt == 4 ? static_cast<size_t>(p.K / 2) : static_cast<size_t>(p.K);
            const int nw = slots_in_chunk(p, c);
            for (int tt = 0; tt < it.ntiles && ok; ++tt) {
                const int o0 = (it.tile0 + tt) * 128;
                const int rows = min(128, p.N - o0);
                for (int w = 0; w < nw; ++w, ++j) {
                    const int slot = j % NS;
                    if (j >= NS &&
                        !mbar_wait(&slot_empty[slot], static_cast<uint32_t>((j / NS) - 1) & 1u, lim)) {
                        ok = false;
                        break;
                    }
                    int k0;
                    const int klen = slot_len(p, c, w, k0);
                    const int row_chunks = (fmt == 4 ? klen / 2 : klen) / 16;
                    const uint8_t *src = static_cast<const uint8_t *>(p.Wq) +
                                         static_cast<size_t>(o0) * row_stride + (fmt == 4 ? k0 / 2 : k0);
                    const uint32_t dst = base + L.w_off + slot * kSlotBytes;
                    for (int e = t; e < 128 * 16; e += kProdThreads) {
                        const int r = e >> 4, ch = e & 15;
                        if (r < rows && ch < row_chunks)
                            cp_async_16(dst + r * 256 + wswz(ch, r) * 16,
                                        src + static_cast<size_t>(r) * row_stride + ch * 16);
                    }
                    if (fmt == 4) {
                        // (scale, min) words of the slot's groups: klen / 32
                        // words per row, 16-byte chunks of 4 words
                        const int schunks = klen / 128;
                        const uint8_t *ssrc = static_cast<const uint8_t *>(p.S) +
                                              static_cast<size_t>(o0) * (p.K / 32) * 4 + (k0 / 32) * 4;
                        const uint32_t sdst = base + L.s_off + slot * kScaleBytes;
                        for (int e = t; e < 128 * 4; e += kProdThreads) {
                            const int r = e >> 2, ch = e & 3;
                            if (r < rows && ch < schunks)
                                cp_async_16(sdst + r * 64 + sswz(ch, r) * 16,
                                            ssrc + static_cast<size_t>(r) * (p.K / 32) * 4 + ch * 16);
                        }
                    }
                    if (!(j == 0 && t == 0 && ctl->inject)) cp_async_arrive(&slot_full[slot]);
                }
            }
        }
        cp_async_wait_all();   // every copy this thread issued has landed
    } else if (warp == kXWarp) {
        // ======================================================= activation loader
        if (lane == 0) {
            pdl_wait_prior_grid();     // the fp16 images come from the preceding pre-pass
            int cur_x = -1, cur_c = -1, nx = 0;
            for (int i = i_first; i < i_last && ok; ++i) {
                const Item it = item_at(P, i);
                const PlProj &p = *it.p;
                const int c = it.chunk;
                if (p.xid == cur_x && c == cur_c) continue;
                if (nx > 0 && !mbar_wait(x_empty, static_cast<uint32_t>(nx - 1) & 1u, lim)) {
                    ok = false;
                    break;
                }
                const int atoms = (min(kXChunk, p.K - c * kXChunk)) / 64;
                const uint32_t bytes = static_cast<uint32_t>(atoms * BNp * 128);
                mbar_expect_tx(x_full, bytes);
                bulk_load(base + L.x_off, p.Xh + static_cast<size_t>(c) * BNp * 1024, bytes, x_full);
                cur_x = p.xid;
                cur_c = c;
                ++nx;
            }
            if (nx > 0) mbar_wait(x_full, static_cast<uint32_t>(nx - 1) & 1u, lim);
        }
        __syncwarp();
    } else if (warp < kDeqWarps) {
        // ======================================================= dequantizers
        const int h = warp >> 2;
        const int r = threadIdx.x & 127;
        const uint32_t ta = tmem + kAOff + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                            static_cast<uint32_t>(16 * h);
        int j = 0, ja = 0;
        for (int i = i_first; i < i_last && ok; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = *it.p;
            const int c = it.chunk;
            const int nw = slots_in_chunk(p, c);
            for (int tt = 0; tt < it.ntiles && ok; ++tt) {
                for (int w = 0; w < nw; ++w, ++j) {
                    const int slot = j % NS;
                    if (!mbar_wait(&slot_full[slot], static_cast<uint32_t>(j / NS) & 1u, lim)) {
                        ok = false;
                        break;
                    }
                    int k0;
                    const int nsteps = slot_len(p, c, w, k0) / 64;
                    const uint32_t wslot = base + L.w_off + slot * kSlotBytes;
                    const uint32_t sslot = base + L.s_off + slot * kScaleBytes;
                    for (int s = 0; s < nsteps; ++s, ++ja) {
                        uint32_t wv[16];
                        if (p.fmt == kFmtQ4)
                            dequant_slot<kFmtQ4>(wslot, sslot, r, h, s, wv);
                        else if (p.fmt == kFmtQ8)
                            dequant_slot<kFmtQ8>(wslot, sslot, r, h, s, wv);
                        else
                            dequant_slot<kFmtE4M3>(wslot, sslot, r, h, s, wv);
                        const int st = ja % kAStages;
                        if (ja >= kAStages &&
                            !mbar_wait(&a_empty[st], static_cast<uint32_t>((ja / kAStages) - 1) & 1u,
                                       lim)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        tmem_st_x16(ta + static_cast<uint32_t>(st) * kAStageCols, wv);
                        tmem_st_wait();
                        tc_fence_before_sync();
                        mbar_arrive(&a_full[st]);
                    }
                    if (!ok) break;
                    // every read of the slot has been consumed by a store above
                    mbar_arrive(&slot_empty[slot]);
                }
            }
        }
    } else if (warp == kWaiterWarp) {
        // ======================================================= MMA waiter
        // All waits of the issuer, handed over per K step through named
        // barrier kMmaBar (a thread that waits on an mbarrier right after a
        // tcgen05.commit stalls until its MMAs drain, so the issuer never waits).
        int cur_x = -1, cur_c = -1, nx = 0, ja = 0, ntile = 0;
        for (int i = i_first; i < i_last && ok; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = *it.p;
            const int c = it.chunk;
            bool good = true;
            const bool fresh = !(p.xid == cur_x && c == cur_c);
            if (fresh) {
                cur_x = p.xid;
                cur_c = c;
                ++nx;
            }
            const int nw = slots_in_chunk(p, c);
            for (int tt = 0; tt < it.ntiles && ok; ++tt) {
                const int n_acc = ntile + tt;                 // accumulator of this tile
                for (int w = 0; w < nw && ok; ++w) {
                    int k0;
                    const int nsteps = slot_len(p, c, w, k0) / 64;
                    for (int s = 0; s < nsteps; ++s, ++ja) {
                        if (lane == 0) {
                            if (good && fresh && tt == 0 && w == 0 && s == 0)
                                good = mbar_wait(x_full, static_cast<uint32_t>(nx - 1) & 1u, lim);
                            if (good && w == 0 && s == 0 && n_acc >= R)
                                good = mbar_wait(&acc_empty[n_acc % R],
                                                 static_cast<uint32_t>((n_acc / R) - 1) & 1u, lim);
                            if (good)
                                good = mbar_wait(&a_full[ja % kAStages],
                                                 static_cast<uint32_t>(ja / kAStages) & 1u, lim);
                            mma_abort[ja & 1] = good ? 0u : 1u;
                        }
                        named_bar_sync(kMmaBar, 64);
                        if (__shfl_sync(0xffffffffu, good ? 1 : 0, 0) == 0) {
                            ok = false;
                            break;
                        }
                    }
                }
            }
            ntile += it.ntiles;
        }
    } else if (warp == kIssuerWarp) {
        // ======================================================= MMA issuer
        const uint32_t idesc = idesc_f16_f32acc(128, BNp);
        const uint64_t xdesc0 = sw128_kmajor_desc(base + L.x_off);
        const uint64_t atom_desc = static_cast<uint64_t>(BNp * 128) >> 4;
        int ja = 0, ntile = 0;
        bool abort = false;
        for (int i = i_first; i < i_last && !abort; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = *it.p;
            const int c = it.chunk;
            const int nw = slots_in_chunk(p, c);
            for (int tt = 0; tt < it.ntiles && !abort; ++tt) {
                const int n_acc = ntile + tt;
                const uint32_t d = tmem + static_cast<uint32_t>((n_acc % R) * BNp);
                for (int w = 0; w < nw && !abort; ++w) {
                    int k0;
                    const int nsteps = slot_len(p, c, w, k0) / 64;
                    const int atom0 = (k0 - c * kXChunk) / 64;
                    for (int s = 0; s < nsteps; ++s, ++ja) {
                        named_bar_sync(kMmaBar, 64);
                        if (mma_abort[ja & 1]) {
                            abort = true;
                            break;
                        }
                        if (lane == 0) {
                            tc_fence_after_sync();
                            const uint32_t a =
                                tmem + kAOff + static_cast<uint32_t>(ja % kAStages) * kAStageCols;
                            const uint64_t bdesc = xdesc0 + static_cast<uint64_t>(atom0 + s) * atom_desc;
                            const bool first = w == 0 && s == 0;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                tc_mma_f16kind_ts(d, a + 8 * kk, bdesc + 2 * kk, idesc,
                                                  (first && kk == 0) ? 0u : 1u);
                            tc_commit(&a_empty[ja % kAStages]);
                        }
                    }
                }
                if (!abort && lane == 0) tc_commit(&acc_full[n_acc % R]);
            }
            // release the activation chunk once its MMAs complete if the next
            // item reads a different (activations, chunk)
            if (!abort && lane == 0 && i + 1 < i_last) {
                const PlItem &nx = P.items[i + 1];
                if (!(P.proj[nx.proj].xid == p.xid && nx.chunk == c)) tc_commit(x_empty);
            }
            ntile += it.ntiles;
        }
        if (abort && lane == 0) {
            // MMAs already issued may still read shared memory and write
            // TMEM: wait (bounded) for them before the CTA releases either
            tc_commit(drain);
            mbar_wait(drain, 0, lim);
        }
        __syncwarp();
    } else {
        // ======================================================= epilogue
        pdl_wait_prior_grid();         // Y may be read or written by earlier kernels
        const int et = threadIdx.x - kEpiWarp0 * 32;   // 0..255
        const int q = warp & 3;
        const int half = (warp - kEpiWarp0) >> 2;
        const int cols = BNp / 2;                      // a multiple of 8
        const int c0 = half * cols;
        const int row = q * 32 + lane;                 // TMEM lane = weight row in the tile
        const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
        // Thread 0 of the epilogue waits for each accumulator and shares the
        // outcome through named barrier kEpiBar, so the eight warps always
        // take the same branch and meet at the same barriers.
        volatile uint32_t *last_flag = tmem_slot + 3;
        volatile uint32_t *full_flag = tmem_slot + 4;       // two, by tile parity
        int ntile = 0;
        for (int i = i_first; i < i_last && ok; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = *it.p;
            const bool split = it.nchunks > 1;
            for (int tt = 0; tt < it.ntiles && ok; ++tt, ++ntile) {
                const int slot = ntile % R;
                if (et == 0)
                    full_flag[ntile & 1] =
                        mbar_wait(&acc_full[slot], static_cast<uint32_t>(ntile / R) & 1u, lim) ? 1u
                                                                                                : 0u;
                named_bar_sync(kEpiBar, kEpiThreads);
                ok = full_flag[ntile & 1] != 0;
                if (!ok) break;
                tc_fence_after_sync();
                const int tile = it.tile0 + tt;
                const int o = tile * 128 + row;
                const uint32_t tacc = tq + static_cast<uint32_t>(slot * BNp + c0);
                if (!split) {
                    float sc = 1.f, b = 0.f;
                    if (p.fmt == 8 && o < p.N) sc = __ldg(static_cast<const float *>(p.S) + o);
                    if (p.bias && o < p.N) b = __ldg(p.bias + o);
                    float *yo = p.Y + o;
                    const size_t rs = static_cast<size_t>(p.N);
                    for (int cc = 0; cc < cols; cc += 8) {
                        uint32_t v[8];
                        tmem_ld_x8(tacc + static_cast<uint32_t>(cc), v);
                        tmem_ld_wait();
                        if (o < p.N) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int m = c0 + cc + e;
                                if (m < M) yo[static_cast<size_t>(m) * rs] = fmaf(__uint_as_float(v[e]), sc, b);
                            }
                        }
                    }
                    tc_fence_before_sync();
                    mbar_arrive(&acc_empty[slot]);
                    continue;
                }
                // Split tile: this chunk's partial goes to its slot of the
                // partials, column-major ([m][row]) so a warp writes 128
                // contiguous bytes per column; the accumulator is free then.
                const int st = p.sbase + tile;
                float *part = P.partials +
                              static_cast<size_t>(st * P.max_chunks + it.chunk) * BNp * 128;
                for (int cc = 0; cc < cols; cc += 8) {
                    uint32_t v[8];
                    tmem_ld_x8(tacc + static_cast<uint32_t>(cc), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        __stcg(part + static_cast<size_t>(c0 + cc + e) * 128 + row, __uint_as_float(v[e]));
                }
                tc_fence_before_sync();
                mbar_arrive(&acc_empty[slot]);
                // The last chunk to finish sums the partials in chunk order
                // (the same order whichever CTA it is) and writes Y.
                __threadfence();
                named_bar_sync(kEpiBar, kEpiThreads);
                if (et == 0) {
                    const unsigned done = atomicAdd(P.counters + st, 1u);
                    *last_flag = (done == static_cast<unsigned>(it.nchunks - 1)) ? 1u : 0u;
                }
                named_bar_sync(kEpiBar, kEpiThreads);
                if (*last_flag) {
                    __threadfence();
                    if (o < p.N) {
                        const float sc = p.fmt == 8 ? __ldg(static_cast<const float *>(p.S) + o) : 1.f;
                        const float b = p.bias ? __ldg(p.bias + o) : 0.f;
                        const float *p0 = P.partials + static_cast<size_t>(st * P.max_chunks) * BNp * 128;
                        for (int m = c0; m < c0 + cols && m < M; ++m) {
                            float acc = __ldcg(p0 + static_cast<size_t>(m) * 128 + row);
                            for (int ch = 1; ch < it.nchunks; ++ch)
                                acc += __ldcg(p0 + (static_cast<size_t>(ch) * BNp + m) * 128 + row);
                            p.Y[static_cast<size_t>(m) * p.N + o] = fmaf(acc, sc, b);
                        }
                    }
                    if (et == 0) P.counters[st] = 0u;      // ready for the next launch
                }
                named_bar_sync(kEpiBar, kEpiThreads);      // last_flag is read by all
            }
        }
    }
    if (!ok) atomicOr(&ctl->status, 1u << kStatusTimeout);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------ pre-pass
// Converts each distinct activation block X [M, K] fp32 once into the fp16
// image the list kernel loads: [K/64 atoms][BNp rows][128 bytes], 16-byte
// chunk j of row m at chunk j ^ (m & 7) (the 128-byte swizzle), pairs within
// every chunk in the operand order of dequant.cuh, rows M..BNp-1 zero.  One
// 512-wide K chunk is then one contiguous range.  An activation that is not
// a finite fp16 value after rounding latches kStatusRange.
__global__ void __launch_bounds__(256)
    pl_prep_kernel(const __grid_constant__ PlPrep P, DevCtl *ctl) {
    pdl_wait_prior_grid();
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int i = threadIdx.x; i < P.n_counters; i += blockDim.x) P.counters[i] = 0u;
    const PlPrepImage &im = P.img[blockIdx.y];
    const int BNp = P.bnp, M = P.M, K = im.K;
    const int64_t pieces = static_cast<int64_t>(K / 8) * BNp;   // 16-byte output pieces
    uint32_t bad = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < pieces;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int j = static_cast<int>(i & 7);
        const int64_t am = i >> 3;                  // atom * BNp + row
        const int m = static_cast<int>(am % BNp);
        const int a = static_cast<int>(am / BNp);
        uint4 out = make_uint4(0, 0, 0, 0);
        if (m < M) {
            const float4 *src =
                reinterpret_cast<const float4 *>(im.X + static_cast<size_t>(m) * K + a * 64 + j * 8);
            const uint2 lo = x4_f16(__ldg(src)), hi = x4_f16(__ldg(src + 1));
            bad |= f16x2_nonfinite(lo) | f16x2_nonfinite(hi);
            out = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        uint8_t *dst = im.Xh + (static_cast<size_t>(a) * BNp + m) * 128 + ((j ^ (m & 7)) << 4);
        *reinterpret_cast<uint4 *>(dst) = out;
    }
    if (__any_sync(0xffffffffu, bad != 0) && (threadIdx.x & 31) == 0)
        atomicOr(&ctl->status, 1u << kStatusRange);
    pdl_launch_dependents();
}

cudaError_t launch_pl_prep(const PlPrep &prep, int n_images, int64_t max_k, DevCtl *ctl,
                           cudaStream_t s) {
    if (n_images < 1) return cudaSuccess;
    const int64_t pieces = max_k / 8 * prep.bnp;
    const unsigned gx = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(
        (pieces + 255) / 256, std::max<int64_t>(1, 296 / n_images))));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gx, static_cast<unsigned>(n_images), 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, pl_prep_kernel, prep, ctl);
}

cudaError_t launch_pl(const PlParams &P, int n_ctas, DevCtl *ctl, cudaStream_t s) {
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(pl_qgemm_kernel, 227 * 1024, dev, attr_done)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_ctas), 1, 1);
    cfg.blockDim = dim3(kPlThreads, 1, 1);
    cfg.dynamicSmemBytes = pl_layout(P.bnp, P.nslots).total + 1024;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, pl_qgemm_kernel, P, ctl);
}

}  // namespace

int pl_bnp(int M) { return std::max(16, (M + 15) / 16 * 16); }

int pl_nacc(int bnp) { return std::min(kPlMaxAcc, static_cast<int>(kAOff) / bnp); }

int pl_nslots(int bnp) {
    const int avail = 227 * 1024 - 1024 - bnp * kXChunk * 2 - 512;
    return std::max(2, std::min(kMaxSlots, avail / (kSlotBytes + kScaleBytes)));
}

bool pl_supported(int fmt, int M, int K) {
    // q4 (scale, min) rows are 16-byte cp.async copies: K/8 bytes a multiple of 16
    return M >= 1 && M <= 128 && (fmt == 4 ? K % 128 == 0 : K % 64 == 0);
}

namespace {

int64_t pl_image_bytes(int M, int K) { return static_cast<int64_t>(pl_bnp(M)) * K * 2; }

// Workspace of a list call: the distinct activation images ((X, K) -> image
// index, in order of first appearance), then the partial tiles and counters
// of the projections with K > 512 ("split" tiles, one partial per 512-wide K
// chunk).
struct Plan {
    std::vector<int> xid;            // per projection
    std::vector<int> sbase;          // per projection: first split-tile index, or -1
    std::vector<const float *> X;    // per image
    std::vector<int> K;
    std::vector<size_t> off;
    int n_split = 0, max_chunks = 1;
    size_t partials_off = 0, counters_off = 0, bytes = 0;
};

constexpr size_t align256(size_t b) { return (b + 255) / 256 * 256; }

Plan plan_list(const PlInput *in, int count, int M) {
    Plan pl;
    pl.xid.resize(count);
    pl.sbase.assign(count, -1);
    size_t img = 0;
    for (int i = 0; i < count; ++i) {
        int found = -1;
        for (size_t j = 0; j < pl.X.size(); ++j)
            if (pl.X[j] == in[i].X && pl.K[j] == in[i].K) found = static_cast<int>(j);
        if (found < 0) {
            found = static_cast<int>(pl.X.size());
            pl.X.push_back(in[i].X);
            pl.K.push_back(in[i].K);
            pl.off.push_back(img);
            img += align256(static_cast<size_t>(pl_image_bytes(M, in[i].K)));
        }
        pl.xid[i] = found;
        const int nchunks = (in[i].K + kXChunk - 1) / kXChunk;
        if (nchunks > 1) {
            pl.sbase[i] = pl.n_split;
            pl.n_split += (in[i].N + 127) / 128;
            pl.max_chunks = std::max(pl.max_chunks, nchunks);
        }
    }
    pl.partials_off = img;
    const size_t part = static_cast<size_t>(pl.n_split) * pl.max_chunks * pl_bnp(M) * 128 * 4;
    pl.counters_off = align256(pl.partials_off + part);
    pl.bytes = align256(pl.counters_off + static_cast<size_t>(pl.n_split) * 4);
    return pl;
}

// Tiles per work item: up to about 160 KB of packed weights (four q4 tiles
// of a 512-wide chunk, two q8 or e4m3 tiles), so that the items assigned to
// one CTA can be balanced closely.
int tiles_per_item(const PlInput &q) {
    const int klen = std::min(q.K, kXChunk);
    const double tile = 128.0 * klen * (q.fmt == 4 ? 0.625 : 1.0);
    return std::max(1, std::min(4, static_cast<int>(160.0 * 1024 / tile)));
}

}  // namespace

size_t pl_workspace_bytes(const PlInput *in, int count, int M) {
    return plan_list(in, count, M).bytes;
}

cudaError_t launch_pl_batch(const PlInput *in, int count, int M, void *ws, DevCtl *ctl,
                            cudaStream_t s) {
    if (count < 1) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    sms = std::min(sms, kPlMaxCtas);
    const int bnp = pl_bnp(M), nacc = pl_nacc(bnp), nslots = pl_nslots(bnp);
    const Plan pl = plan_list(in, count, M);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    unsigned *counters = reinterpret_cast<unsigned *>(wsb + pl.counters_off);

    // 1. every distinct activation block once into its fp16 image; the first
    // pre-pass launch also zeroes the split tiles' counters
    for (size_t i0 = 0; i0 < pl.X.size(); i0 += kPlMaxProj) {
        thread_local PlPrep prep;   // large: kept off the stack; a launch copies it
        prep.M = M;
        prep.bnp = bnp;
        prep.counters = counters;
        prep.n_counters = i0 == 0 ? pl.n_split : 0;
        const int n = static_cast<int>(std::min<size_t>(kPlMaxProj, pl.X.size() - i0));
        int max_k = 0;
        for (int j = 0; j < n; ++j) {
            prep.img[j] = {pl.X[i0 + j], wsb + pl.off[i0 + j], pl.K[i0 + j], 0};
            max_k = std::max(max_k, pl.K[i0 + j]);
        }
        if ((e = launch_pl_prep(prep, n, max_k, ctl, s)) != cudaSuccess) return e;
    }

    // 2. projections ordered by activation image (stable), launches of at most
    // kPlMaxProj projections and kPlMaxItems items
    std::vector<int> order(count);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return pl.xid[a] < pl.xid[b]; });
    thread_local PlParams P;     // large: kept off the stack; a launch copies it
    size_t pos = 0;
    while (pos < order.size()) {
        std::vector<PlItem> items;
        std::vector<double> cost;
        int np = 0;
        for (; pos < order.size() && np < kPlMaxProj; ++np, ++pos) {
            const int src = order[pos];
            const PlInput &q = in[src];
            const int tiles = (q.N + 127) / 128;
            const int nchunks = (q.K + kXChunk - 1) / kXChunk;
            const int per = tiles_per_item(q);
            const int n_items = nchunks * ((tiles + per - 1) / per);
            if (np > 0 && items.size() + n_items > static_cast<size_t>(kPlMaxItems)) break;
            P.proj[np] = {wsb + pl.off[pl.xid[src]], q.Wq, q.S, q.bias, q.Y, q.N, q.K, q.fmt,
                          pl.xid[src], pl.sbase[src]};
            for (int c = 0; c < nchunks; ++c) {
                const int klen = std::min(kXChunk, q.K - c * kXChunk);
                for (int t = 0; t < tiles; t += per) {
                    const int nt = std::min(per, tiles - t);
                    items.push_back({static_cast<uint32_t>(t), static_cast<uint16_t>(np),
                                     static_cast<uint8_t>(nt), static_cast<uint8_t>(c)});
                    const int rows = std::min(nt * 128, q.N - t * 128);
                    cost.push_back(static_cast<double>(rows) * klen * (q.fmt == 4 ? 0.625 : 1.0));
                }
            }
        }
        // largest item first onto the least loaded CTA
        const int n_items = static_cast<int>(items.size());
        const int G = std::min(sms, n_items);
        std::vector<int> by_cost(n_items);
        std::iota(by_cost.begin(), by_cost.end(), 0);
        std::stable_sort(by_cost.begin(), by_cost.end(),
                         [&](int a, int b) { return cost[a] > cost[b]; });
        std::vector<double> load(G, 0.0);
        std::vector<std::vector<int>> mine(G);
        for (int it : by_cost) {
            const int b = static_cast<int>(std::min_element(load.begin(), load.end()) - load.begin());
            load[b] += cost[it];
            mine[b].push_back(it);
        }
        // within a CTA: items of one activation chunk together, in list order
        int k = 0;
        for (int b = 0; b < G; ++b) {
            std::sort(mine[b].begin(), mine[b].end(), [&](int a, int c) {
                const PlItem &x = items[a], &y = items[c];
                if (P.proj[x.proj].xid != P.proj[y.proj].xid)
                    return P.proj[x.proj].xid < P.proj[y.proj].xid;
                if (x.chunk != y.chunk) return x.chunk < y.chunk;
                if (x.proj != y.proj) return x.proj < y.proj;
                return x.tile0 < y.tile0;
            });
            P.cta_items[b] = k;
            for (int it : mine[b]) P.items[k++] = items[it];
        }
        P.cta_items[G] = k;
        P.M = M;
        P.bnp = bnp;
        P.nslots = nslots;
        P.nacc = nacc;
        P.partials = reinterpret_cast<float *>(wsb + pl.partials_off);
        P.counters = counters;
        P.max_chunks = pl.max_chunks;
        P.pad = 0;
        if ((e = launch_pl(P, G, ctl, s)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace rtq
