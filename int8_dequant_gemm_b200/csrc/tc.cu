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
// Operands are fp16 (q4 weights: the exact code*scale+min rounded once by
// fma.rn.f16x2; q8 codes exact; activations rounded to nearest-even) in
// tcgen05.mma kind::f16.  fp16 keeps 11 significant bits, at the price of the
// fp16 range: an activation that rounds to infinity (|x| >= 65520) or is not
// finite makes its outputs infinite or NaN, and the epilogue latches
// kStatusRange in the device control block for any output that is not finite
// (finite fp16 operands cannot overflow an fp32 sum of K <= 2^20 products).  Within every
// 8-element K chunk k .. k+7 both operands store the pairs
// (k + t, k + t + 4), t = 0..3 (see dequant.cuh).
//
// One CTA = 8 converter warps + 1 MMA warp.  Per 64-wide K step the converter
// warps
//   - issue every global load of the step at once -- the packed weight slice
//     (q4: 32 B of codes + one (scale, min) word per group and row; q8: 64 B
//     of codes per row) and the fp32 activation slice, 16 threads per row in
//     contiguous 16-byte pieces -- one step ahead of
//     the step they convert, so a step's loads are in flight while the
//     previous one is converted (register double buffering);
//   - dequantize / round in registers and store 16-bit operands into the A
//     (weights) and B (activations) stages,
// both in the K-major 128-byte-swizzle layout the MMA descriptors describe,
// then fence the generic->async proxy and arrive on the stage's `full`
// mbarrier.  One thread of the MMA warp waits on `full`, issues four
// tcgen05.mma (K = 16 each) and commits to the stage's `empty` mbarrier, which
// hands the stage back to the converters once the tensor core has read it.
// After the last K step a final commit releases the epilogue: the converter
// warps read TMEM (32x32b loads, one weight row per thread), apply the q8 row
// scale in fp32 and store fp32 Y with 128-byte coalesced rows.  Tiles of up to
// 128 activation rows leave room for two CTAs per SM, so one CTA's epilogue
// overlaps the other's main loop.
//
// Every mbarrier wait is bounded; a wait that gives up latches
// RT_ERR_DEVICE_TIMEOUT in the device status word and the CTA winds down: the
// MMA thread waits (bounded) for the MMAs it issued before TMEM is released,
// and with split K no CTA of the cluster stores a tile that any of its CTAs
// failed to finish.
//
// The same tile code also runs as a grouped launch (tc_group_kernel): up to
// four independent projections with one activation tile each, e.g. a block's
// qkvg, wo, w13 and w2 at M = 80.  Each CTA takes a weight tile of one of
// them, so the four dependency chains of load -> MMA -> reduction -> store
// overlap in one launch instead of following one another.
#include <algorithm>

#include "dequant.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rtq {
namespace {

constexpr int kTileO = 128;                      // weight rows per tile (MMA M)
constexpr int kTileK = 64;                       // K per stage: one 128-byte 16-bit row
constexpr int kConvWarps = 8;
constexpr int kConvThreads = kConvWarps * 32;    // 256
constexpr int kTcThreads = kConvThreads + 32;    // + MMA warp
constexpr int kAStageBytes = kTileO * 128;       // 16 KB
constexpr int kMaxSmem = 227 * 1024;
constexpr int kTwoCtaSmem = 110 * 1024;          // budget that lets two CTAs share an SM
constexpr int kSmemPerSm = 228 * 1024;           // shared memory of one SM
constexpr int kSmemReserve = 1024;               // the runtime's reservation per CTA

__host__ __device__ inline int tc_stage_bytes(int bn) { return kAStageBytes + bn * 128; }

// The stage ring, which with split K is reused for the CTA's fp32 partial
// tile (BN columns of 128 rows).
__host__ __device__ inline int tc_region_bytes(int bn, int stages, int ksplit) {
    const int ring = stages * tc_stage_bytes(bn);
    const int part = ksplit > 1 ? bn * kTileO * 4 : 0;
    return ((ring > part ? ring : part) + 1023) / 1024 * 1024;
}

__host__ __device__ inline int tc_smem_bytes(int bn, int stages, int ksplit) {
    // full/empty per stage, done, drain, TMEM address + CTA-ok flag
    return 1024 + tc_region_bytes(bn, stages, ksplit) + (2 * stages + 2) * 8 + 16;
}

__host__ __device__ inline uint32_t tmem_cols_for(int bn) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(bn)) c <<= 1;
    return c;
}

// Dynamic shared memory of a launch, raised where needed so that no more CTAs
// fit on an SM than its 512 TMEM columns serve.  tcgen05.alloc blocks until
// columns are free, and a CTA holding columns may wait in a cluster barrier
// for a peer that is blocked in its allocation on another SM, so residency
// must never ask for more columns than an SM has.  (Registers already hold
// the kernel to two CTAs per SM; this keeps the guarantee independent of
// register allocation.)
inline int tc_launch_smem(int bn, int stages, int ksplit) {
    const int need = tc_smem_bytes(bn, stages, ksplit);
    const int max_ctas = 512 / static_cast<int>(tmem_cols_for(bn));
    const int floor_bytes = kSmemPerSm / (max_ctas + 1) - kSmemReserve + 1;
    return std::max(need, (floor_bytes + 127) / 128 * 128);
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// Per-thread constants of the converter role.
//   A (weights): thread t owns row t/2 of the 128-row tile and half h = t&1 of
//   its 64-element K slice (q4: one group of 32 codes; q8: 32 codes).
//   B (activations): 16 threads cover one row's 64 fp32 (256 contiguous
//   bytes) as 16-byte pieces; thread t owns piece p = t&15 of rows
//   t/16 + 16*i, i < PIECES.
struct ConvThread {
    int t, ra, h, p, rb0;
    uint32_t a_off[4];   // smem byte offsets of the thread's 4 A chunks
    uint32_t b_off0;     // smem byte offset of its first B piece (+2048 per i)
};

__device__ __forceinline__ ConvThread conv_thread(int t) {
    ConvThread c;
    c.t = t;
    c.ra = t >> 1;
    c.h = t & 1;
    for (int j = 0; j < 4; ++j) c.a_off[j] = swz(c.ra, 4 * c.h + j);
    c.p = t & 15;
    c.rb0 = t >> 4;
    c.b_off0 = swz(c.rb0, c.p >> 1) + (c.p & 1) * 8;
    return c;
}

// Registers holding one K step's raw data for one converter thread.
//   A: q4 -> a0 = 16 B of codes, a1.x = the group's (scale, min);
//      q8 -> a0, a1 = 32 B of codes.
//   B: PIECES float4 of activations.
template <int PIECES>
struct StageRegs {
    uint4 a0, a1;
    float4 b[PIECES];
};

template <int FMT, int PIECES>
__device__ __forceinline__ void load_stage(StageRegs<PIECES> &R, const ConvThread &c,
                                           const float *__restrict__ X,
                                           const void *__restrict__ Wq,
                                           const void *__restrict__ S, int o0, int m0, int k0,
                                           int M, int N, int K, int BN) {
    const int o = o0 + c.ra;
    R.a0 = make_uint4(0, 0, 0, 0);
    R.a1 = make_uint4(0, 0, 0, 0);
    if (o < N) {
        if (FMT == 4) {
            R.a0 = ldg_nc_v4(static_cast<const uint8_t *>(Wq) + static_cast<size_t>(o) * (K / 2) +
                             k0 / 2 + c.h * 16);
            R.a1.x = ldg_nc_u32(static_cast<const uint32_t *>(S) +
                                static_cast<size_t>(o) * (K / 32) + k0 / 32 + c.h);
        } else {
            const int8_t *src =
                static_cast<const int8_t *>(Wq) + static_cast<size_t>(o) * K + k0 + c.h * 32;
            R.a0 = ldg_nc_v4(src);
            R.a1 = ldg_nc_v4(src + 16);
        }
    }
    const float *xb = X + static_cast<size_t>(m0 + c.rb0) * K + k0 + c.p * 4;
#pragma unroll
    for (int i = 0; i < PIECES; ++i) {
        const int rr = c.rb0 + 16 * i;
        R.b[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (rr < BN && m0 + rr < M) R.b[i] = ldg_f4(xb + static_cast<size_t>(16 * i) * K);
    }
}

__device__ __forceinline__ void sts_v2(uint32_t saddr, uint2 v) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(saddr), "r"(v.x), "r"(v.y) : "memory");
}

// Converts one K step held in R and stores it into the stage at sA (weights)
// and sB (activations).
template <int FMT, int PIECES>
__device__ __forceinline__ void store_stage(const StageRegs<PIECES> &R, const ConvThread &c,
                                            uint32_t sA, uint32_t sB, int BN) {
    if (FMT == 4) {
        uint32_t s2, m2;
        q4_scale_min_f16x2(R.a1.x, s2, m2);
        sts_v4(sA + c.a_off[0], q4_word_f16(R.a0.x, s2, m2));
        sts_v4(sA + c.a_off[1], q4_word_f16(R.a0.y, s2, m2));
        sts_v4(sA + c.a_off[2], q4_word_f16(R.a0.z, s2, m2));
        sts_v4(sA + c.a_off[3], q4_word_f16(R.a0.w, s2, m2));
    } else if (FMT == 8) {
        sts_v4(sA + c.a_off[0], q8_words_f16(R.a0.x, R.a0.y));
        sts_v4(sA + c.a_off[1], q8_words_f16(R.a0.z, R.a0.w));
        sts_v4(sA + c.a_off[2], q8_words_f16(R.a1.x, R.a1.y));
        sts_v4(sA + c.a_off[3], q8_words_f16(R.a1.z, R.a1.w));
    } else {   // e4m3: one byte per weight like q8, no scale
        sts_v4(sA + c.a_off[0], e4m3_words_f16(R.a0.x, R.a0.y));
        sts_v4(sA + c.a_off[1], e4m3_words_f16(R.a0.z, R.a0.w));
        sts_v4(sA + c.a_off[2], e4m3_words_f16(R.a1.x, R.a1.y));
        sts_v4(sA + c.a_off[3], e4m3_words_f16(R.a1.z, R.a1.w));
    }
    // A chunk's 8 activations are split between lanes p (even: k .. k+3) and
    // p + 1 (odd: k+4 .. k+7); each lane takes two values from its partner and
    // writes its half of the chunk's pairs (k + t, k + t + 4): t = 0, 1 from
    // the even lane, t = 2, 3 from the odd one.
    const bool odd = (c.p & 1) != 0;
#pragma unroll
    for (int i = 0; i < PIECES; ++i) {
        const float4 a = R.b[i];
        const float s0 = __shfl_xor_sync(0xffffffffu, odd ? a.x : a.z, 1);
        const float s1 = __shfl_xor_sync(0xffffffffu, odd ? a.y : a.w, 1);
        const uint2 v = odd ? make_uint2(pack_f16x2(s0, a.z), pack_f16x2(s1, a.w))
                            : make_uint2(pack_f16x2(a.x, s0), pack_f16x2(a.y, s1));
        if (c.rb0 + 16 * i < BN) sts_v2(sB + c.b_off0 + 2048u * i, v);
    }
}

// True for an infinite or NaN fp32 value.
__device__ __forceinline__ bool nonfinite(float v) {
    return (__float_as_uint(v) & 0x7F800000u) == 0x7F800000u;
}

// One CTA's work: the output tile of weight rows [o0, o0 + 128) and
// activation rows [m0, m0 + BN), over K slice `kslice` of `ksplit`.  With
// ksplit > 1 the tile's slices are the cluster's CTAs of ranks
// [kbase, kbase + ksplit), which reduce their partial sums among themselves;
// every CTA of the cluster must have the same ksplit (each reaches the
// cluster barriers exactly when ksplit > 1).
template <int FMT, int PIECES>
__device__ __forceinline__ void tc_tile(uint8_t *smem_raw, const float *__restrict__ X,
                                        const void *__restrict__ Wq, const void *__restrict__ S,
                                        const float *__restrict__ bias, float *__restrict__ Y,
                                        int M, int N, int K, int BN, int stages, int ksplit,
                                        int o0, int m0, int kslice, int kbase, DevCtl *ctl) {
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw);
    const int stage_bytes = tc_stage_bytes(BN);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + tc_region_bytes(BN, stages, ksplit));
    uint64_t *empty = full + stages;
    uint64_t *done = empty + stages;
    uint64_t *drain = done + 1;       // the MMA thread's own completion wait on a failed tile
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    uint32_t *cta_ok = tmem_slot + 1; // read by cluster peers before they store the tile
    const uint32_t tmem_cols = tmem_cols_for(BN);
    const unsigned long long *lim = &ctl->wait_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // split K: slice `kslice` takes K steps [kz0, kz0 + nk)
    const int nk = K / kTileK / ksplit;
    const int kz0 = kslice * nk;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], kConvThreads);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(drain, 1);
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

    if (warp < kConvWarps) {
        // The weights do not depend on the previous kernel in the stream:
        // start pulling this CTA's slice into L2 before waiting for it.
        const int o = o0 + (static_cast<int>(threadIdx.x) >> 1);
        if (o < N) {
            for (int ks = 0; ks < nk; ++ks) {
                const int k0 = (kz0 + ks) * kTileK;
                if (FMT == 4)
                    prefetch_l2(static_cast<const uint8_t *>(Wq) + static_cast<size_t>(o) * (K / 2) +
                                k0 / 2);
                else
                    prefetch_l2(static_cast<const int8_t *>(Wq) + static_cast<size_t>(o) * K + k0 +
                                (threadIdx.x & 1) * 32);
            }
        }
    }
    pdl_wait_prior_grid();
    // the next kernel may be scheduled now (it reads this one's output only
    // after its own wait for this grid's completion)
    pdl_launch_dependents();

    if (warp < kConvWarps) {
        const ConvThread ct = conv_thread(threadIdx.x);
        StageRegs<PIECES> r0, r1;
        // Converts the step held in R into stage ks % stages once the MMA has
        // released that stage.  (Test hook: with `inject`, thread 0 leaves out
        // its arrival for the first step, so the MMA thread's wait runs out.)
        auto consume = [&](const StageRegs<PIECES> &R, int ks) -> bool {
            const int s = ks % stages;
            if (ks >= stages &&
                !mbar_wait(&empty[s], static_cast<uint32_t>((ks / stages) - 1) & 1u, lim))
                return false;
            const uint32_t sA = base + s * stage_bytes;
            store_stage<FMT, PIECES>(R, ct, sA, sA + kAStageBytes, BN);
            fence_proxy_async_smem();
            if (!(ks == 0 && threadIdx.x == 0 && ctl->inject)) mbar_arrive(&full[s]);
            return true;
        };
        const int kb = kz0 * kTileK;
        load_stage<FMT, PIECES>(r0, ct, X, Wq, S, o0, m0, kb, M, N, K, BN);
        for (int ks = 0; ks < nk; ks += 2) {
            if (ks + 1 < nk)
                load_stage<FMT, PIECES>(r1, ct, X, Wq, S, o0, m0, kb + (ks + 1) * kTileK, M, N, K,
                                        BN);
            if (!(ok = consume(r0, ks))) break;
            if (ks + 1 >= nk) break;
            if (ks + 2 < nk)
                load_stage<FMT, PIECES>(r0, ct, X, Wq, S, o0, m0, kb + (ks + 2) * kTileK, M, N, K,
                                        BN);
            if (!(ok = consume(r1, ks + 1))) break;
        }
        // ---------------------------------------------------------- epilogue
        if (ok) ok = mbar_wait(done, 0, lim);
        // tcgen05.ld is warp-collective: the whole warp takes the epilogue or none of it
        ok = __all_sync(0xffffffffu, ok);
        bool ybad = false;                     // an output that is not finite
        if (ok) {
            tc_fence_after_sync();
            const int q = warp & 3;            // TMEM lane quadrant of this warp
            const int half = warp >> 2;        // which half of the columns
            const int row = q * 32 + lane;
            const int o = o0 + row;
            float sc = 1.f, b = 0.f;
            if (FMT == 8 && o < N) sc = __ldg(static_cast<const float *>(S) + o);
            if (bias && o < N) b = __ldg(bias + o);
            const int ncol = BN / 2;           // a multiple of 8
            const int c0 = half * ncol;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
            for (int c = c0; c < c0 + ncol; c += 16) {
                uint32_t v0[8], v1[8];
                const bool two = c + 8 < c0 + ncol;
                tmem_ld_x8(tbase + static_cast<uint32_t>(c), v0);
                if (two) tmem_ld_x8(tbase + static_cast<uint32_t>(c + 8), v1);
                tmem_ld_wait();
                if (ksplit > 1) {
                    // this CTA's partial sum, column-major [BN][128] in the
                    // retired stage ring; reduced across the cluster below
                    float *part = reinterpret_cast<float *>(smem);
#pragma unroll
                    for (int j = 0; j < 8; ++j) part[(c + j) * kTileO + row] = __uint_as_float(v0[j]);
                    if (two) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            part[(c + 8 + j) * kTileO + row] = __uint_as_float(v1[j]);
                    }
                } else if (o < N) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int m = m0 + c + j;
                        if (m < M) {
                            const float y = fmaf(__uint_as_float(v0[j]), sc, b);
                            ybad |= nonfinite(y);
                            Y[static_cast<size_t>(m) * N + o] = y;
                        }
                    }
                    if (two) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int m = m0 + c + 8 + j;
                            if (m < M) {
                                const float y = fmaf(__uint_as_float(v1[j]), sc, b);
                                ybad |= nonfinite(y);
                                Y[static_cast<size_t>(m) * N + o] = y;
                            }
                        }
                    }
                }
            }
        }
        if (__any_sync(0xffffffffu, ybad) && lane == 0) atomicOr(&ctl->status, 1u << kStatusRange);
    } else {
        // -------------------------------------------------------- MMA issuer
        // The whole warp walks the loop and waits; one elected lane issues.
        const uint32_t idesc = idesc_f16_f32acc(kTileO, BN);
        for (int ks = 0; ks < nk; ++ks) {
            const int s = ks % stages;
            const bool got = mbar_wait(&full[s], static_cast<uint32_t>(ks / stages) & 1u, lim);
            if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t sA = base + s * stage_bytes;
            const uint32_t sB = sA + kAStageBytes;
            const uint64_t adesc = sw128_kmajor_desc(sA);
            const uint64_t bdesc = sw128_kmajor_desc(sB);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kTileK / 16; ++kk) {
                    // +32 bytes per 16-element K step -> +2 in the 16-byte address field
                    tc_mma_f16kind(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                   (ks > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            __syncwarp();
        }
        if (ok) {
            if (elect_one()) tc_commit(done);
            __syncwarp();
        } else {
            // MMAs already issued may still read the stage ring and write
            // TMEM: wait (bounded) for them before the CTA releases either.
            if (elect_one()) tc_commit(drain);
            __syncwarp();
            mbar_wait(drain, 0, lim);
        }
    }
    __syncwarp();
    if (!ok) atomicOr(&ctl->status, 1u << kStatusTimeout);
    tc_fence_before_sync();
    const int all_ok = __syncthreads_and(ok ? 1 : 0);
    if (ksplit > 1) {
        // Every CTA of the cluster reaches both barriers on every path (a
        // timed-out wait only skips work), and a cluster's CTAs are resident
        // together, so neither barrier can hang.  A tile is stored only if
        // every CTA of its K slices finished.
        if (threadIdx.x == 0) *cta_ok = static_cast<uint32_t>(all_ok);
        cluster_sync();                       // all partials and flags written
        bool tile_ok = true;
        for (int r = 0; r < ksplit; ++r)
            tile_ok = tile_ok && ld_cluster_u32(cluster_map(smem_addr(cta_ok),
                                                            static_cast<uint32_t>(kbase + r))) != 0;
        if (warp < kConvWarps && tile_ok) {
            bool ybad = false;
            // Slice s sums columns [s * BN/ksplit, (s + 1) * BN/ksplit) over
            // the tile's partials in rank order (deterministic) and stores Y.
            const int cols = BN / ksplit;
            const int mbeg = kslice * cols;
            for (int idx = threadIdx.x; idx < cols * (kTileO / 4); idx += kConvThreads) {
                const int ml = mbeg + idx / (kTileO / 4), o4 = idx % (kTileO / 4);
                const int m = m0 + ml, o = o0 + 4 * o4;
                const uint32_t off = base + static_cast<uint32_t>((ml * kTileO + 4 * o4) * 4);
                float4 acc = ld_cluster_f4(cluster_map(off, static_cast<uint32_t>(kbase)));
                for (int r = 1; r < ksplit; ++r) {
                    const float4 v =
                        ld_cluster_f4(cluster_map(off, static_cast<uint32_t>(kbase + r)));
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
                if (m < M && o < N) {
                    float a[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (o + e < N) {
                            const float s = FMT == 8 ? __ldg(static_cast<const float *>(S) + o + e)
                                                     : 1.f;
                            a[e] = fmaf(a[e], s, bias ? __ldg(bias + o + e) : 0.f);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) ybad |= o + e < N && nonfinite(a[e]);
                    float *yp = Y + static_cast<size_t>(m) * N + o;
                    if ((N & 3) == 0 && o + 3 < N) {
                        *reinterpret_cast<float4 *>(yp) = make_float4(a[0], a[1], a[2], a[3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (o + e < N) yp[e] = a[e];
                    }
                }
            }
            if (__any_sync(0xffffffffu, ybad) && lane == 0)
                atomicOr(&ctl->status, 1u << kStatusRange);
        }
        cluster_sync();                       // peers are done reading this CTA's partial
    }
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, tmem_cols);
    }
}

template <int FMT, int PIECES>
__global__ void __launch_bounds__(kTcThreads, 2)
    tc_qgemm_kernel(const float *__restrict__ X, const void *__restrict__ Wq,
                    const void *__restrict__ S, const float *__restrict__ bias,
                    float *__restrict__ Y, int M, int N, int K, int BN, int stages, int ksplit,
                    DevCtl *ctl) {
    extern __shared__ uint8_t smem_raw[];
    tc_tile<FMT, PIECES>(smem_raw, X, Wq, S, bias, Y, M, N, K, BN, stages, ksplit,
                         static_cast<int>(blockIdx.x) * kTileO, static_cast<int>(blockIdx.y) * BN,
                         static_cast<int>(blockIdx.z), 0, ctl);
}

// Several independent projections that share M (<= BN, one activation tile)
// in one launch.  The launch's clusters have `csize` CTAs along z; problem i
// owns the clusters whose blockIdx.x lies in [cl0[i], cl0[i + 1]) and splits K
// by its own factor ks (a divisor of csize), so one cluster holds csize / ks of
// its 128-row weight tiles: CTA rank r works on tile r / ks of the cluster's
// run, K slice r % ks.  Every CTA of a cluster belongs to one problem.  Tiles
// past the problem's last one (a partly filled last cluster) compute zeros
// and store nothing.
struct TcProblem {
    const float *X;
    const void *Wq;
    const void *S;
    const float *bias;
    float *Y;
    int N, K, fmt, cl0, ks;
};

struct TcGroup {
    TcProblem p[kMaxGroup];
    int count;
};

template <int PIECES>
__global__ void __launch_bounds__(kTcThreads, 2)
    tc_group_kernel(const __grid_constant__ TcGroup g, int M, int BN, int stages, int csize,
                    DevCtl *ctl) {
    extern __shared__ uint8_t smem_raw[];
    const int bx = static_cast<int>(blockIdx.x);
    int i = 0;
    while (i + 1 < g.count && bx >= g.p[i + 1].cl0) ++i;
    const TcProblem &p = g.p[i];
    const int r = static_cast<int>(blockIdx.z);          // rank in the cluster
    const int tile = (bx - p.cl0) * (csize / p.ks) + r / p.ks;
    const int o0 = tile * kTileO;
    const int kslice = r % p.ks, kbase = r - kslice;
    if (p.fmt == kFmtQ4)
        tc_tile<kFmtQ4, PIECES>(smem_raw, p.X, p.Wq, p.S, p.bias, p.Y, M, p.N, p.K, BN, stages,
                                p.ks, o0, 0, kslice, kbase, ctl);
    else if (p.fmt == kFmtQ8)
        tc_tile<kFmtQ8, PIECES>(smem_raw, p.X, p.Wq, p.S, p.bias, p.Y, M, p.N, p.K, BN, stages,
                                p.ks, o0, 0, kslice, kbase, ctl);
    else
        tc_tile<kFmtE4M3, PIECES>(smem_raw, p.X, p.Wq, p.S, p.bias, p.Y, M, p.N, p.K, BN, stages,
                                  p.ks, o0, 0, kslice, kbase, ctl);
}

// Activation rows per tile: one tile when M <= 128; otherwise 128, halved
// (down to 64) while the grid would not give every SM one tile.  Each halving
// doubles how often the weight tile is dequantized, so it stops early.
int pick_bn(int M, int N) {
    if (M <= 128) return std::max(16, (M + 15) / 16 * 16);
    const int n_o = (N + kTileO - 1) / kTileO;
    int bn = 128;
    while (bn > 64 && static_cast<long>(n_o) * ((M + bn - 1) / bn) < 148) bn /= 2;
    return bn;
}

// K slices per output tile.  Small problems (one activation tile) have too
// few 128-row weight tiles to occupy the GPU -- q8 w2 and wo have 4 -- so K is
// split across a cluster of up to 8 CTAs, up to about two CTAs per SM.  The
// slices' partial sums are reduced through distributed shared memory.
int pick_ksplit(int M, int N, int K, int BN) {
    if (M > BN) return 1;
    const int nk = K / kTileK;
    const long tiles = static_cast<long>((N + kTileO - 1) / kTileO);
    int ks = 1;
    while (ks < 8 && nk % (2 * ks) == 0 && tiles * ks * 2 <= 2 * 148) ks *= 2;
    return ks;
}

template <int FMT, int PIECES>
cudaError_t launch_tc_pieces(const float *X, const void *Wq, const void *S, const float *bias,
                             float *Y, int M, int N, int K, int BN, DevCtl *ctl, cudaStream_t st) {
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(tc_qgemm_kernel<FMT, PIECES>, kMaxSmem, dev, attr_done)) != cudaSuccess)
        return e;
    const int ksplit = pick_ksplit(M, N, K, BN);
    const int nk = K / kTileK / ksplit;
    const int budget = kTwoCtaSmem;
    int stages = (budget - 1024 - 256) / tc_stage_bytes(BN);
    stages = std::max(1, std::min({stages, 4, nk}));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((N + kTileO - 1) / kTileO, (M + BN - 1) / BN, ksplit);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = tc_launch_smem(BN, stages, ksplit);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = static_cast<unsigned>(ksplit);
    cfg.attrs = attr;
    cfg.numAttrs = ksplit > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, tc_qgemm_kernel<FMT, PIECES>, X, Wq, S, bias, Y, M, N, K,
                              BN, stages, ksplit, ctl);
}

template <int FMT>
cudaError_t launch_tc_fmt(const float *X, const void *Wq, const void *S, const float *bias,
                          float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t st) {
    const int BN = pick_bn(M, N);
    if (BN <= 32) return launch_tc_pieces<FMT, 2>(X, Wq, S, bias, Y, M, N, K, BN, ctl, st);
    if (BN <= 64) return launch_tc_pieces<FMT, 4>(X, Wq, S, bias, Y, M, N, K, BN, ctl, st);
    return launch_tc_pieces<FMT, 8>(X, Wq, S, bias, Y, M, N, K, BN, ctl, st);
}

// K splits for a group.  A launch lasts as long as its longest chain of K
// steps, and the projections' K differ (the RT-J block has 8 K steps in qkvg,
// wo and w13 but 32 in w2), so each projection gets its own split: the
// smallest power of two (up to 8, dividing its step count) that brings it to
// at most T steps per CTA.  T starts at the longest projection's steps / 8 and
// doubles until the launch fits one wave of two CTAs per SM.  The cluster size
// is the largest split.  Fills g.p[i].ks and .cl0; returns the cluster size
// and the cluster count in *nclusters.
int plan_group(TcGroup &g, int *nclusters) {
    int max_nk = 1;
    for (int i = 0; i < g.count; ++i) max_nk = std::max(max_nk, g.p[i].K / kTileK);
    for (int T = std::max(1, (max_nk + 7) / 8);; T *= 2) {
        int csize = 1;
        for (int i = 0; i < g.count; ++i) {
            const int nk = g.p[i].K / kTileK;
            int ks = 1;
            while (ks < 8 && nk / ks > T && nk % (2 * ks) == 0) ks *= 2;
            g.p[i].ks = ks;
            csize = std::max(csize, ks);
        }
        int clusters = 0;
        for (int i = 0; i < g.count; ++i) {
            const int per = csize / g.p[i].ks;        // weight tiles per cluster
            const int tiles = (g.p[i].N + kTileO - 1) / kTileO;
            g.p[i].cl0 = clusters;
            clusters += (tiles + per - 1) / per;
        }
        if (static_cast<long>(clusters) * csize <= 2 * 148 || T >= max_nk) {
            *nclusters = clusters;
            return csize;
        }
    }
}

template <int PIECES>
cudaError_t launch_group_pieces(TcGroup g, int M, int BN, DevCtl *ctl, cudaStream_t st) {
    static std::atomic<bool> attr_done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = smem_attr_once(tc_group_kernel<PIECES>, kMaxSmem, dev, attr_done)) != cudaSuccess)
        return e;
    int nclusters = 0;
    const int csize = plan_group(g, &nclusters);
    int max_nk = 1;
    for (int i = 0; i < g.count; ++i) max_nk = std::max(max_nk, g.p[i].K / kTileK / g.p[i].ks);
    int stages = (kTwoCtaSmem - 1024 - 256) / tc_stage_bytes(BN);
    stages = std::max(1, std::min({stages, 4, max_nk}));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nclusters), 1, static_cast<unsigned>(csize));
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    // the partial-sum region is sized whenever some projection splits K
    cfg.dynamicSmemBytes = tc_launch_smem(BN, stages, csize);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = static_cast<unsigned>(csize);
    cfg.attrs = attr;
    cfg.numAttrs = csize > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, tc_group_kernel<PIECES>, g, M, BN, stages, csize, ctl);
}

cudaError_t launch_group(const TcGroup &g, int M, DevCtl *ctl, cudaStream_t st) {
    const int BN = pick_bn(M, 0);
    if (BN <= 32) return launch_group_pieces<2>(g, M, BN, ctl, st);
    if (BN <= 64) return launch_group_pieces<4>(g, M, BN, ctl, st);
    return launch_group_pieces<8>(g, M, BN, ctl, st);
}

}  // namespace

cudaError_t launch_tc_group(const GroupProblem *probs, int count, int M, DevCtl *ctl,
                            cudaStream_t s) {
    if (count < 1 || count > kMaxGroup || M < 1 || M > kTileO) return cudaErrorInvalidValue;
    TcGroup g = {};
    g.count = count;
    for (int i = 0; i < count; ++i) {
        const GroupProblem &q = probs[i];
        if (!fmt_valid(q.fmt) || q.N < 1 || q.K < kTileK || q.K % kTileK != 0)
            return cudaErrorInvalidValue;
        g.p[i] = {q.X, q.Wq, q.S, q.bias, q.Y, q.N, q.K, q.fmt, 0, 1};
    }
    return launch_group(g, M, ctl, s);
}

cudaError_t launch_tc(int fmt, const float *X, const void *Wq, const void *S, const float *bias,
                      float *Y, int M, int N, int K, DevCtl *ctl, cudaStream_t s) {
    if (fmt == kFmtQ4) return launch_tc_fmt<kFmtQ4>(X, Wq, S, bias, Y, M, N, K, ctl, s);
    if (fmt == kFmtQ8) return launch_tc_fmt<kFmtQ8>(X, Wq, S, bias, Y, M, N, K, ctl, s);
    return launch_tc_fmt<kFmtE4M3>(X, Wq, S, bias, Y, M, N, K, ctl, s);
}

}  // namespace rtq
