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
//   weights  TMA: one slot = 128 rows x 256 bytes of codes (q4: K 512, q8:
//            K 256) as two boxes of 128 rows x 128 bytes from the
//            projection's [N, row bytes] tensor map, plus, for q4, one box of
//            the rows' 16 (scale, min) words.  The codes land 128-byte
//            swizzled (16-byte chunk c of row r at chunk c ^ (r & 7)), the
//            words 64-byte swizzled (chunk c at c ^ ((r >> 1) & 3)), so the
//            dequantizers' reads of one chunk over 8 consecutive rows hit 8
//            different bank groups.  The tensor maps travel in the kernel's
//            parameters, encoded on the host once per weight and thread.
//            (A slot issued as 16-byte cp.async copies instead costs one
//            instruction per 16 bytes on the SM's load/store path and paced
//            the whole pipeline; a TMA box costs one.)
//   activations  the projection's fp16 image (written by pl_prep_kernel below
//            in the 128-byte-swizzled operand layout), one 512-wide K chunk
//            at a time, into a resident buffer of two halves (K atoms 0-3 and
//            4-7 of the chunk, one bulk copy each).  A half is reloaded only
//            when the (activations, K chunk) pair changes, and only once the
//            MMAs of its previous use have completed: the next chunk's first
//            half streams in while the current chunk's second half is used.
// A stages: the MMAs read the dequantized weights from TMEM, one stage = two
// 64-wide K steps (64 columns) in a ring of four at columns [256, 512), in
// the operand order of dequant.cuh (pairs (k + t, k + t + 4) in every 8
// K values), which the activation image follows too.
// Roles (20 warps):
//   warps 0-7   dequantizers: thread (r, h) converts step h of each stage of
//               row r (64 K values) into TMEM lane r of the stage: it loads
//               all its bytes of a weight slot into registers at once,
//               releases the slot, then converts and stores stage by stage.
//   warp 8      MMA issuer, fed through named barrier 1 by
//   warp 9      the MMA waiter, which performs all of the issuer's waits.
//   warps 10-17 epilogue: TMEM -> registers (q8 row scale) -> fp32 Y.
//   warp 18     weight producer (one thread, TMA).
//   warp 19     activation loader (one thread, bulk copies).
// A tile with K > 512 is one work item that runs chunk by chunk, its
// accumulator kept in TMEM across the chunks: no partial sums leave the SM.
// (Splitting K over CTAs, with fp32 partials that the last chunk to finish
// summed, cost more than half the time of a K = 2048 list: the partial
// stores, fences and the dependent reduction loads.)
//
// Work distribution (host, launch_pl_batch): items (up to four tiles of K <=
// 512, about 80 KB of packed weights; one tile when K > 512) are sorted by
// (activation image, projection, tile) and the sorted sequence is cut into
// one contiguous run per CTA with about equal bytes, so a CTA switches its
// activation image rarely.  Every tile is computed by one CTA from start to
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
constexpr int kProdWarp = 18;
constexpr int kXWarp = 19;
constexpr int kPlThreads = (kXWarp + 1) * 32;        // 640
constexpr int kEpiThreads = kEpiWarps * 32;          // 256
constexpr uint32_t kMmaBar = 1;                      // named barrier: waiter <-> issuer
constexpr uint32_t kEpiBar = 2;                      // named barrier: the epilogue warps
constexpr int kSlotBytes = 32 * 1024;                // 128 rows x 256 bytes of codes
constexpr int kBoxBytes = 16 * 1024;                 // one TMA box: 128 rows x 128 bytes
constexpr int kScaleBytes = 8 * 1024;                // 128 rows x 16 (scale, min) words
constexpr int kMaxSlots = 4;
constexpr int kAStages = 4;                          // a power of two
constexpr uint32_t kAStageCols = 64;                 // two 64-wide K steps
constexpr uint32_t kAOff = 256;                      // A stages at TMEM columns [256, 512)
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
    // slot full/empty, A full/empty, 2 x full/empty, acc full/empty, drain,
    // then 8 words: TMEM address, 2 issuer abort flags, the epilogue's flags
    L.total = L.bar_off + (2 * kMaxSlots + 2 * kAStages + 4 + 2 * kPlMaxAcc + 1) * 8 + 32;
    return L;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Shared address of 16-byte chunk c (0..15) of row r of a weight slot: box
// c / 8, 128-byte swizzle within it.
__device__ __forceinline__ uint32_t wchunk(uint32_t slot, int c, int r) {
    return slot + (static_cast<uint32_t>(c >> 3) << 14) + static_cast<uint32_t>(r * 128) +
           (static_cast<uint32_t>((c & 7) ^ (r & 7)) << 4);
}
// Physical 16-byte chunk of logical scale chunk c (0..3) of row r.
__device__ __forceinline__ int sswz(int c, int r) { return c ^ ((r >> 1) & 3); }

// The walk every role takes through a CTA's items: item -> 512-wide K chunk
// -> tile -> weight slot -> stage.  Each role advances it at its own grain.  The projection's fields are copied into registers once
// per item: read through a pointer into the parameter space they would be
// loaded again after every asm statement that clobbers memory (the barrier
// waits and arrivals), a few hundred cycles each.
struct Item {
    PlProj p;
    int proj, tile0, ntiles, nchunks;
};

__device__ __forceinline__ Item item_at(const PlParams &P, int i) {
    const PlItem it = P.items[i];
    Item r;
    r.p = P.proj[it.proj];
    r.proj = it.proj;
    r.tile0 = static_cast<int>(it.tile0);
    r.ntiles = it.ntiles;
    r.nchunks = (r.p.K + kXChunk - 1) / kXChunk;
    return r;
}

// K range [k0, k0 + len) of slot w of chunk c; 0 if the slot lies past K.
__device__ __forceinline__ int slot_len(const PlProj &p, int c, int w, int &k0) {
    k0 = c * kXChunk + w * slot_k(p.fmt);
    return max(0, min(slot_k(p.fmt), p.K - k0));
}

// 64-wide K atoms of chunk c (8 except in a last, shorter chunk).
__device__ __forceinline__ int chunk_atoms(const PlProj &p, int c) { return min(8, (p.K - c * kXChunk) / 64); }

__device__ __forceinline__ int slots_in_chunk(const PlProj &p, int c) {
    const int len = min(kXChunk, p.K - c * kXChunk);
    return (len + slot_k(p.fmt) - 1) / slot_k(p.fmt);
}

// ------------------------------------------------------------ dequantization
__device__ __forceinline__ void put4(uint32_t (&w)[16], int i, uint4 v) {
    w[i] = v.x;
    w[i + 1] = v.y;
    w[i + 2] = v.z;
    w[i + 3] = v.w;
}

// Half h of 32 K values (h = 0: K 0..31 of the step, 1: K 32..63) of one
// thread's step -> 16 operand words.  q4: r0 = the 16 bytes of codes, sw =
// the group's (scale, min) word; q8 / e4m3: r0, r1 = the 32 bytes of codes.
template <int FMT>
__device__ __forceinline__ void convert_half(uint4 r0, uint4 r1, uint32_t sw, uint32_t (&w)[16]) {
    if (FMT == kFmtQ4) {
        uint32_t s2, m2;
        q4_scale_min_f16x2(sw, s2, m2);
        put4(w, 0, q4_word_f16(r0.x, s2, m2));
        put4(w, 4, q4_word_f16(r0.y, s2, m2));
        put4(w, 8, q4_word_f16(r0.z, s2, m2));
        put4(w, 12, q4_word_f16(r0.w, s2, m2));
    } else if (FMT == kFmtQ8) {
        put4(w, 0, q8_words_f16(r0.x, r0.y));
        put4(w, 4, q8_words_f16(r0.z, r0.w));
        put4(w, 8, q8_words_f16(r1.x, r1.y));
        put4(w, 12, q8_words_f16(r1.z, r1.w));
    } else {
        put4(w, 0, e4m3_words_f16(r0.x, r0.y));
        put4(w, 4, e4m3_words_f16(r0.z, r0.w));
        put4(w, 8, e4m3_words_f16(r1.x, r1.y));
        put4(w, 12, e4m3_words_f16(r1.z, r1.w));
    }
}

// Up to kRound stages of one weight slot for thread (r, h) (two for q4, one
// for the one-byte formats, whose steps hold twice the bytes): its steps
// s = s0 + 2i + h below nsteps.  Their bytes are loaded first (the slot is
// released after the slot's last loads); then, per stage, the thread waits
// for the stage to be free, converts its step and stores it (32 columns at
// offset 32h), and every thread arrives.  Returns false if a wait ran out.
template <int FMT>
__device__ __forceinline__ bool dequant_pair(uint32_t wslot, uint32_t sslot, int r, int h, int s0,
                                             int nsteps, uint32_t ta, int &ja, uint64_t *slot_empty,
                                             uint64_t *a_full, uint64_t *a_empty,
                                             const unsigned long long *lim) {
    constexpr int kRaw = FMT == kFmtQ4 ? 2 : 4;     // 16-byte pieces per step
    constexpr int kRound = FMT == kFmtQ4 ? 2 : 1;   // stages per round
    uint4 raw[kRound][kRaw];
    uint2 sc[kRound];
#pragma unroll
    for (int i = 0; i < kRound; ++i) {
        const int s = s0 + 2 * i + h;
        if (s < nsteps) {
#pragma unroll
            for (int q = 0; q < kRaw; ++q) raw[i][q] = lds_v4(wchunk(wslot, kRaw * s + q, r));
            // q4: groups 2s, 2s + 1 = words 4 (s >> 1) + 2h, + 1 of the row
            if (FMT == kFmtQ4) sc[i] = lds_v2(sslot + r * 64 + sswz(s >> 1, r) * 16 + 8 * h);
        }
    }
    if (s0 + 2 * kRound >= nsteps) mbar_arrive(slot_empty);   // every read of the slot has returned
#pragma unroll
    for (int i = 0; i < kRound; ++i) {
        const int s = s0 + 2 * i + h;
        if (s0 + 2 * i >= nsteps) break;
        const int st = ja % kAStages;
        if (ja >= kAStages &&
            !mbar_wait(&a_empty[st], static_cast<uint32_t>((ja / kAStages) - 1) & 1u, lim))
            return false;
        tc_fence_after_sync();
        if (s < nsteps) {
            const uint32_t t = ta + static_cast<uint32_t>(st) * kAStageCols;
            uint32_t w[16];
            if (FMT == kFmtQ4) {
                convert_half<FMT>(raw[i][0], raw[i][0], sc[i].x, w);
                tmem_st_x16(t, w);
                convert_half<FMT>(raw[i][1], raw[i][1], sc[i].y, w);
                tmem_st_x16(t + 16, w);
            } else {
                convert_half<FMT>(raw[i][0], raw[i][1], 0u, w);
                tmem_st_x16(t, w);
                convert_half<FMT>(raw[i][2], raw[i][3], 0u, w);
                tmem_st_x16(t + 16, w);
            }
            tmem_st_wait();
        }
        tc_fence_before_sync();
        mbar_arrive(&a_full[st]);
        ++ja;
    }
    return true;
}

// A whole weight slot (nsteps 64-wide steps) for thread (r, h).
template <int FMT>
__device__ __forceinline__ bool dequant_slot(uint32_t wslot, uint32_t sslot, int r, int h, int nsteps,
                                             uint32_t ta, int &ja, uint64_t *slot_empty,
                                             uint64_t *a_full, uint64_t *a_empty,
                                             const unsigned long long *lim) {
    for (int s0 = 0; s0 < nsteps; s0 += FMT == kFmtQ4 ? 4 : 2)
        if (!dequant_pair<FMT>(wslot, sslot, r, h, s0, nsteps, ta, ja, slot_empty, a_full, a_empty, lim))
            return false;
    return true;
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
    uint64_t *x_full = a_empty + kAStages;             // two: the halves of the buffer
    uint64_t *x_empty = x_full + 2;
    uint64_t *acc_full = x_empty + 2;
    uint64_t *acc_empty = acc_full + kPlMaxAcc;
    uint64_t *drain = acc_empty + kPlMaxAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *mma_abort = tmem_slot + 1;       // waiter -> issuer, per step parity
    const unsigned long long *lim = &ctl->wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i_first = P.cta_items[blockIdx.x], i_last = P.cta_items[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSlots; ++s) {
            mbar_init(&slot_full[s], 1);
            mbar_init(&slot_empty[s], kDeqWarps * 32);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], kDeqWarps * 32);
            mbar_init(&a_empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&x_full[h], 1);
            mbar_init(&x_empty[h], 1);
        }
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

    if (warp == kProdWarp) {
        // ======================================================= weight producer
        // Packed weights do not depend on the previous kernel in the stream.
        // (Test hook: with `inject`, the first slot is never loaded, so the
        // dequantizers' wait for it runs out.)
        if (lane == 0) {
            for (int i = i_first, last = -1; i < i_last; ++i) {
                const int pj = P.items[i].proj;
                if (pj == last) continue;
                last = pj;
                prefetch_tensormap(&P.wmap[pj]);
                if (P.proj[pj].fmt == kFmtQ4) prefetch_tensormap(&P.smap[pj]);
            }
            int j = 0;
            bool skipped0 = false;
            for (int i = i_first; i < i_last && ok; ++i) {
                const Item it = item_at(P, i);
                const PlProj &p = it.p;
                const CUtensorMap *wm = &P.wmap[it.proj];
                const CUtensorMap *sm = &P.smap[it.proj];
                const int fmt = p.fmt;
                for (int c = 0; c < it.nchunks && ok; ++c) {
                    const int nw = slots_in_chunk(p, c);
                    for (int tt = 0; tt < it.ntiles && ok; ++tt) {
                        const int o0 = (it.tile0 + tt) * 128;
                        for (int w = 0; w < nw; ++w, ++j) {
                            const int slot = j % NS;
                            if (j >= NS &&
                                !mbar_wait(&slot_empty[slot], static_cast<uint32_t>((j / NS) - 1) & 1u, lim)) {
                                ok = false;
                                break;
                            }
                            if (j == 0 && ctl->inject) {
                                skipped0 = true;
                                continue;
                            }
                            int k0;
                            const int klen = slot_len(p, c, w, k0);
                            const int row_bytes = fmt == kFmtQ4 ? klen / 2 : klen;   // 64..256
                            const int x = fmt == kFmtQ4 ? k0 / 2 : k0;              // multiple of 256
                            const uint32_t dst = base + L.w_off + slot * kSlotBytes;
                            // a box's bytes count in full, rows past N and
                            // columns past the row included (TMA fills zeros)
                            const int boxes = row_bytes > 128 ? 2 : 1;
                            mbar_expect_tx(&slot_full[slot],
                                           static_cast<uint32_t>(boxes * kBoxBytes +
                                                                 (fmt == kFmtQ4 ? kScaleBytes : 0)));
                            tma_load_2d(dst, wm, x, o0, &slot_full[slot]);
                            if (boxes == 2) tma_load_2d(dst + kBoxBytes, wm, x + 128, o0, &slot_full[slot]);
                            if (fmt == kFmtQ4)
                                tma_load_2d(base + L.s_off + slot * kScaleBytes, sm, k0 / 32, o0,
                                            &slot_full[slot]);
                        }
                    }
                }
            }
            // Every load issued has landed before the CTA may exit: slots
            // before the last NS were reused, so they have been consumed.
            for (int jj = max(0, j - NS); jj < j; ++jj)
                if (!(jj == 0 && skipped0))
                    mbar_wait(&slot_full[jj % NS], static_cast<uint32_t>(jj / NS) & 1u, lim);
        }
        __syncwarp();
    } else if (warp == kXWarp) {
        // ======================================================= activation loader
        // One use of the resident buffer = one (activation image, K chunk)
        // over consecutive chunks of the walk.  Each half (atoms 0-3, 4-7 of
        // the chunk) is refilled once the MMAs of the previous use of that
        // half have completed, so a chunk's first half loads while the
        // previous chunk's second half is still being multiplied.
        if (lane == 0) {
            pdl_wait_prior_grid();     // the fp16 images come from the preceding pre-pass
            int cur_x = -1, cur_c = -1, loads0 = 0, loads1 = 0;
            for (int i = i_first; i < i_last && ok; ++i) {
                const Item it = item_at(P, i);
                const PlProj &p = it.p;
                for (int c = 0; c < it.nchunks && ok; ++c) {
                    if (p.xid == cur_x && c == cur_c) continue;
                    cur_x = p.xid;
                    cur_c = c;
                    const int atoms = chunk_atoms(p, c);
                    for (int h = 0; h < (atoms > 4 ? 2 : 1); ++h) {
                        const int nl = h ? loads1 : loads0;
                        if (nl > 0 && !mbar_wait(&x_empty[h], static_cast<uint32_t>(nl - 1) & 1u, lim)) {
                            ok = false;
                            break;
                        }
                        const int na = min(4, atoms - 4 * h);
                        const uint32_t bytes = static_cast<uint32_t>(na * BNp * 128);
                        mbar_expect_tx(&x_full[h], bytes);
                        bulk_load(base + L.x_off + static_cast<uint32_t>(h * 4 * BNp * 128),
                                  p.Xh + static_cast<size_t>(c * 8 + 4 * h) * BNp * 128, bytes, &x_full[h]);
                        if (h) ++loads1; else ++loads0;
                    }
                }
            }
            if (loads0 > 0) mbar_wait(&x_full[0], static_cast<uint32_t>(loads0 - 1) & 1u, lim);
            if (loads1 > 0) mbar_wait(&x_full[1], static_cast<uint32_t>(loads1 - 1) & 1u, lim);
        }
        __syncwarp();
    } else if (warp < kDeqWarps) {
        // ======================================================= dequantizers
        const int h = warp >> 2;
        const int r = threadIdx.x & 127;
        const uint32_t ta = tmem + kAOff + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                            static_cast<uint32_t>(32 * h);
        int j = 0, ja = 0;
        for (int i = i_first; i < i_last && ok; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = it.p;
            for (int c = 0; c < it.nchunks && ok; ++c) {
                const int nw = slots_in_chunk(p, c);
                for (int tt = 0; tt < it.ntiles && ok; ++tt) {
                    for (int w = 0; w < nw && ok; ++w, ++j) {
                        const int slot = j % NS;
                        if (!mbar_wait(&slot_full[slot], static_cast<uint32_t>(j / NS) & 1u, lim)) {
                            ok = false;
                            break;
                        }
                        int k0;
                        const int nsteps = slot_len(p, c, w, k0) / 64;
                        const uint32_t wslot = base + L.w_off + slot * kSlotBytes;
                        const uint32_t sslot = base + L.s_off + slot * kScaleBytes;
                        if (p.fmt == kFmtQ4)
                            ok = dequant_slot<kFmtQ4>(wslot, sslot, r, h, nsteps, ta, ja, &slot_empty[slot],
                                                      a_full, a_empty, lim);
                        else if (p.fmt == kFmtQ8)
                            ok = dequant_slot<kFmtQ8>(wslot, sslot, r, h, nsteps, ta, ja, &slot_empty[slot],
                                                      a_full, a_empty, lim);
                        else
                            ok = dequant_slot<kFmtE4M3>(wslot, sslot, r, h, nsteps, ta, ja,
                                                        &slot_empty[slot], a_full, a_empty, lim);
                    }
                }
            }
        }
    } else if (warp == kWaiterWarp) {
        // ======================================================= MMA waiter
        // All waits of the issuer, handed over per stage through named
        // barrier kMmaBar (a thread that waits on an mbarrier right after a
        // tcgen05.commit stalls until its MMAs drain, so the issuer never waits).
        // loads of each half so far, and whether this use's stages have
        // reached each half (scalars: an indexed array would live in memory)
        int cur_x = -1, cur_c = -1, ja = 0, ntile = 0, loads0 = 0, loads1 = 0;
        bool seen0 = false, seen1 = false;
        bool good = true;
        for (int i = i_first; i < i_last && ok; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = it.p;
            for (int c = 0; c < it.nchunks && ok; ++c) {
                if (!(p.xid == cur_x && c == cur_c)) {
                    cur_x = p.xid;
                    cur_c = c;
                    ++loads0;
                    if (chunk_atoms(p, c) > 4) ++loads1;
                    seen0 = seen1 = false;
                }
                const int nw = slots_in_chunk(p, c);
                for (int tt = 0; tt < it.ntiles && ok; ++tt) {
                    const int n_acc = ntile + tt;                 // accumulator of this tile
                    for (int w = 0; w < nw && ok; ++w) {
                        int k0;
                        const int nsteps = slot_len(p, c, w, k0) / 64;
                        const int atom0 = (k0 - c * kXChunk) / 64;
                        for (int s = 0; 2 * s < nsteps; ++s, ++ja) {
                            const int hx = atom0 + 2 * s >= 4 ? 1 : 0;
                            const bool first_touch = hx ? !seen1 : !seen0;
                            if (lane == 0) {
                                if (good && first_touch)
                                    good = mbar_wait(&x_full[hx],
                                                     static_cast<uint32_t>((hx ? loads1 : loads0) - 1) & 1u, lim);
                                if (good && c == 0 && w == 0 && s == 0 && n_acc >= R)
                                    good = mbar_wait(&acc_empty[n_acc % R],
                                                     static_cast<uint32_t>((n_acc / R) - 1) & 1u, lim);
                                if (good)
                                    good = mbar_wait(&a_full[ja % kAStages],
                                                     static_cast<uint32_t>(ja / kAStages) & 1u, lim);
                                mma_abort[ja & 1] = good ? 0u : 1u;
                            }
                            seen0 = seen0 || hx == 0;
                            seen1 = seen1 || hx == 1;
                            named_bar_sync(kMmaBar, 64);
                            if (__shfl_sync(0xffffffffu, good ? 1 : 0, 0) == 0) {
                                ok = false;
                                break;
                            }
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
            const PlProj &p = it.p;
            // does the next item start a different use of the X buffer?
            bool next_same_x = false;
            if (i + 1 < i_last) {
                const PlItem &nx = P.items[i + 1];
                next_same_x = P.proj[nx.proj].xid == p.xid;
            }
            for (int c = 0; c < it.nchunks && !abort; ++c) {
                const int nw = slots_in_chunk(p, c);
                // this (item, chunk) ends its use of the X buffer, and another use follows
                const bool use_ends = c + 1 < it.nchunks || (i + 1 < i_last && !(next_same_x && c == 0));
                for (int tt = 0; tt < it.ntiles && !abort; ++tt) {
                    const int n_acc = ntile + tt;
                    const uint32_t d = tmem + static_cast<uint32_t>((n_acc % R) * BNp);
                    const bool release = use_ends && tt + 1 == it.ntiles;
                    for (int w = 0; w < nw && !abort; ++w) {
                        int k0;
                        const int nsteps = slot_len(p, c, w, k0) / 64;
                        const int atom0 = (k0 - c * kXChunk) / 64;
                        for (int s = 0; 2 * s < nsteps; ++s, ++ja) {
                            named_bar_sync(kMmaBar, 64);
                            if (mma_abort[ja & 1]) {
                                abort = true;
                                break;
                            }
                            // the whole warp walks the loop; one elected lane issues
                            tc_fence_after_sync();
                            const int st = ja & (kAStages - 1);
                            const uint32_t a = tmem + kAOff + static_cast<uint32_t>(st) * kAStageCols;
                            const int atom = atom0 + 2 * s;
                            const uint64_t b0 = xdesc0 + static_cast<uint64_t>(atom) * atom_desc;
                            const uint32_t acc0 = (c == 0 && w == 0 && s == 0) ? 0u : 1u;
                            const bool two = 2 * s + 1 < nsteps;
                            // last stage on this half of the buffer in the use: the
                            // next stage is in the other half, or the tile ends
                            const int hx = atom >= 4 ? 1 : 0;
                            const bool tile_end = 2 * s + 2 >= nsteps && w + 1 == nw;
                            const int next_atom = 2 * s + 2 < nsteps ? atom + 2 : (w + 1) * slot_k(p.fmt) / 64;
                            const bool half_end = tile_end || (next_atom >= 4 ? 1 : 0) != hx;
                            if (elect_one()) {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    tc_mma_f16kind_ts(d, a + 8 * kk, b0 + 2 * kk, idesc, kk == 0 ? acc0 : 1u);
                                if (two) {
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        tc_mma_f16kind_ts(d, a + 32 + 8 * kk, b0 + atom_desc + 2 * kk, idesc, 1u);
                                }
                                tc_commit(&a_empty[st]);
                                if (release && half_end) tc_commit(&x_empty[hx]);
                            }
                            __syncwarp();
                        }
                    }
                    if (!abort && c + 1 == it.nchunks && elect_one()) tc_commit(&acc_full[n_acc % R]);
                    __syncwarp();
                }
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
        volatile uint32_t *full_flag = tmem_slot + 4;       // two, by tile parity
        int ntile = 0;
        for (int i = i_first; i < i_last && ok; ++i) {
            const Item it = item_at(P, i);
            const PlProj &p = it.p;
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
                const int o = (it.tile0 + tt) * 128 + row;
                const uint32_t tacc = tq + static_cast<uint32_t>(slot * BNp + c0);
                float sc = 1.f, b = 0.f;
                if (p.fmt == kFmtQ8 && o < p.N) sc = __ldg(static_cast<const float *>(p.S) + o);
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
// chunk j of row m at chunk j ^ (m & 7) (the 128-byte swizzle), the 8 values
// of every chunk in the operand order of dequant.cuh, rows M..BNp-1 zero.
// One 512-wide K chunk is then one contiguous range.  An activation that is
// not a finite fp16 value after rounding latches kStatusRange.
__global__ void __launch_bounds__(256)
    pl_prep_kernel(const __grid_constant__ PlPrep P, DevCtl *ctl) {
    // The list launch that follows may start right away: its weight copies
    // do not depend on this kernel, and it reads the images only after its
    // own wait for this grid's completion.
    pdl_launch_dependents();
    pdl_wait_prior_grid();
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
            out = x8_f16(__ldg(src), __ldg(src + 1));
            bad |= f16x2_nonfinite(make_uint2(out.x, out.y)) | f16x2_nonfinite(make_uint2(out.z, out.w));
        }
        uint8_t *dst = im.Xh + (static_cast<size_t>(a) * BNp + m) * 128 + ((j ^ (m & 7)) << 4);
        *reinterpret_cast<uint4 *>(dst) = out;
    }
    if (__any_sync(0xffffffffu, bad != 0) && (threadIdx.x & 31) == 0)
        atomicOr(&ctl->status, 1u << kStatusRange);
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

namespace {

// Tiles per work item: up to about 80 KB of packed weights (two q4 tiles of
// K = 512, one q8 or e4m3 tile), small against a CTA's share of a list so
// that the runs cut from the sorted items come out nearly equal.  With
// K > 512 an item is one tile: its accumulator stays in TMEM over all chunks.
int tiles_per_item(int fmt, int K) {
    if (K > kXChunk) return 1;
    const double tile = 128.0 * K * (fmt == 4 ? 0.625 : 1.0);
    return std::max(1, std::min(4, static_cast<int>(80.0 * 1024 / tile)));
}

int64_t items_of(int fmt, int64_t N, int K) {
    const int64_t tiles = (N + 127) / 128;
    const int per = tiles_per_item(fmt, K);
    return (tiles + per - 1) / per;
}

}  // namespace

bool pl_supported(int fmt, int M, int64_t N, int K) {
    // TMA boxes: the rows of codes and of q4 (scale, min) words (K/8 bytes)
    // must be multiples of 16 bytes; one projection's items fit one launch
    return M >= 1 && M <= 128 && N >= 1 && (fmt == 4 ? K % 128 == 0 : K % 64 == 0) &&
           items_of(fmt, N, K) <= kPlMaxItems;
}

namespace {

int64_t pl_image_bytes(int M, int K) { return static_cast<int64_t>(pl_bnp(M)) * K * 2; }

// Workspace of a list call: the distinct activation images ((X, K) -> image
// index, in order of first appearance).
struct Plan {
    std::vector<int> xid;            // per projection
    std::vector<const float *> X;    // per image
    std::vector<int> K;
    std::vector<size_t> off;
    size_t bytes = 0;
};

constexpr size_t align256(size_t b) { return (b + 255) / 256 * 256; }

Plan plan_list(const PlInput *in, int count, int M) {
    Plan pl;
    pl.xid.resize(count);
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
    }
    pl.bytes = img;
    return pl;
}

// Tensor maps of the packed weights, cached per thread by (pointer, shape,
// kind) in a small direct-mapped table, so that a list call encodes only the
// weights it has not seen lately.  kind 0: codes, kind 1: q4 (scale, min)
// words.
bool weight_map(CUtensorMap *out, int kind, int fmt, const void *ptr, int64_t N, int K) {
    struct Entry {
        CUtensorMap map;
        const void *ptr;
        int64_t N;
        int K, key;
    };
    constexpr int kEntries = 256;
    thread_local Entry cache[kEntries] = {};
    const int key = kind * 16 + fmt;
    const uintptr_t h = (reinterpret_cast<uintptr_t>(ptr) >> 8) ^ static_cast<uintptr_t>(N * 31 + K) ^
                        static_cast<uintptr_t>(key);
    Entry &e = cache[(h ^ (h >> 9)) % kEntries];
    if (e.ptr == ptr && e.N == N && e.K == K && e.key == key) {
        *out = e.map;
        return true;
    }
    bool ok;
    if (kind == 0)
        ok = encode_tma_2d(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ptr,
                           static_cast<uint64_t>(fmt == 4 ? K / 2 : K), static_cast<uint64_t>(N), 128,
                           CU_TENSOR_MAP_SWIZZLE_128B, 128);
    else
        ok = encode_tma_2d(out, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, ptr, static_cast<uint64_t>(K / 32),
                           static_cast<uint64_t>(N), 16, CU_TENSOR_MAP_SWIZZLE_64B, 128);
    if (ok) {
        e.map = *out;
        e.ptr = ptr;
        e.N = N;
        e.K = K;
        e.key = key;
    }
    return ok;
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

    // 1. every distinct activation block once into its fp16 image
    for (size_t i0 = 0; i0 < pl.X.size(); i0 += kPlMaxProj) {
        thread_local PlPrep prep;   // large: kept off the stack; a launch copies it
        prep.M = M;
        prep.bnp = bnp;
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
            const int per = tiles_per_item(q.fmt, q.K);
            const int n_items = (tiles + per - 1) / per;
            if (n_items > kPlMaxItems) return cudaErrorInvalidValue;   // not pl_supported
            if (np > 0 && items.size() + n_items > static_cast<size_t>(kPlMaxItems)) break;
            if (!weight_map(&P.wmap[np], 0, q.fmt, q.Wq, q.N, q.K) ||
                (q.fmt == 4 && !weight_map(&P.smap[np], 1, q.fmt, q.S, q.N, q.K)))
                return cudaErrorInvalidValue;
            P.proj[np] = {wsb + pl.off[pl.xid[src]], q.Wq, q.S, q.bias, q.Y, q.N, q.K, q.fmt,
                          pl.xid[src], 0};
            for (int t = 0; t < tiles; t += per) {
                const int nt = std::min(per, tiles - t);
                items.push_back({static_cast<uint32_t>(t), static_cast<uint16_t>(np),
                                 static_cast<uint8_t>(nt), 0});
                const int rows = std::min(nt * 128, q.N - t * 128);
                cost.push_back(static_cast<double>(rows) * q.K * (q.fmt == 4 ? 0.625 : 1.0));
            }
        }
        // items in (activation image, projection, tile) order, cut into G
        // contiguous runs of about equal bytes
        const int n_items = static_cast<int>(items.size());
        const int G = std::min(sms, n_items);
        std::vector<int> order_it(n_items);
        std::iota(order_it.begin(), order_it.end(), 0);
        std::stable_sort(order_it.begin(), order_it.end(), [&](int a, int c) {
            const PlItem &x = items[a], &y = items[c];
            if (P.proj[x.proj].xid != P.proj[y.proj].xid) return P.proj[x.proj].xid < P.proj[y.proj].xid;
            if (x.proj != y.proj) return x.proj < y.proj;
            return x.tile0 < y.tile0;
        });
        double total = 0.0;
        for (double c : cost) total += c;
        int k = 0;
        double done = 0.0;
        for (int b = 0; b < G; ++b) {
            P.cta_items[b] = k;
            const double target = total * (b + 1) / G;
            // at least one item, and one left for every later CTA; an item
            // joins this run if its midpoint lies before the target
            const int last = n_items - (G - 1 - b);
            do {
                done += cost[order_it[k]];
                P.items[k] = items[order_it[k]];
                ++k;
            } while (k < last && done + 0.5 * cost[order_it[k]] < target);
        }
        P.cta_items[G] = k;
        P.M = M;
        P.bnp = bnp;
        P.nslots = nslots;
        P.nacc = nacc;
        if ((e = launch_pl(P, G, ctl, s)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace rtq
