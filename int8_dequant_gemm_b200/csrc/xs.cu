// tcgen05 path for many activation rows and short K (K <= 512): activations
// stay resident in shared memory, TMA streams the packed weights past them.
//
// The tile product is the same transposed one as in tc.cu,
//   D[o, m] = sum_k W_hat[o, k] * X[m, k],
// with 128 weight rows as the MMA's M dimension and 128 activation rows as its
// N dimension, but the operands swap roles in memory: a CTA converts one
// 128-row block of X to 16-bit ONCE (all of K: 128 x K x 2 bytes of shared
// memory) and then walks a run of weight tiles against it.  Each activation
// byte crosses L2 once per CTA rather than once per 128-row weight tile; the
// weights (0.6 to 1.3 MB per projection, resident in L2) are re-read once per
// activation block instead.
//
// Work list: the (activation block, weight tile) pairs in activation-major
// order, split into one contiguous run per CTA (one CTA per SM), so a CTA
// changes activation block rarely.
//
// Roles (14 warps):
//   warp 13     TMA issuer (one thread): per weight tile the (scale, min)
//               block of its 128 rows (q4), and per 64-wide K step the
//               128-row slice of packed codes, into mbarrier-tracked rings
//               that run kRaw steps ahead.
//   warps 0-3   dequantizers: thread r owns row r of every weight tile; per K
//               step it reads its 32 (q4) or 64 (q8) bytes of codes from the
//               ring, dequantizes 64 weights and writes them into a 16 KB A
//               stage in the K-major 128-byte-swizzle layout.
//   warps 4-7   activation loaders: on every change of activation block they
//               convert its 128 rows x K fp32 into the resident X tile, one
//               64-column atom (and mbarrier) at a time.
//   warp 8      MMA issuer (one thread): per weight tile, K/64 stages x 4
//               tcgen05.mma (K = 16) into one of two TMEM accumulators.
//   warps 9-12  epilogue: TMEM -> registers (q8 row scale) -> fp32 Y with
//               128-byte coalesced rows, overlapping the next tile's MMAs.
//
// Every mbarrier wait is bounded; a wait that gives up latches
// RT_ERR_DEVICE_TIMEOUT in the device status word and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "dequant.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rtq {
namespace {

constexpr int kXsTileO = 128;                 // weight rows per tile (MMA M)
constexpr int kXsTileM = 128;                 // activation rows per block (MMA N)
constexpr int kAtomK = 64;                    // K per atom / stage (128-byte 16-bit rows)
constexpr int kXsMaxK = 512;
constexpr int kDeqWarps = 4, kXldWarps = 4, kEpiWarps = 4;
constexpr int kDeqThreads = kDeqWarps * 32;              // 128
constexpr int kXldThreads = kXldWarps * 32;              // 128
constexpr int kXldWarp0 = kDeqWarps;                     // 4
constexpr int kMmaWarp = kDeqWarps + kXldWarps;          // 8
constexpr int kEpiWarp0 = kMmaWarp + 1;                  // 9
constexpr int kTmaWarp = kEpiWarp0 + kEpiWarps;          // 13
constexpr int kEpiThreads = kEpiWarps * 32;              // 128
constexpr int kXsThreads = (kTmaWarp + 1) * 32;          // 448
constexpr int kAStage = kXsTileO * 128;                  // 16 KB
constexpr int kXAtom = kXsTileM * 128;                   // 16 KB
constexpr int kAStages = 3;
constexpr int kRaw = 4;                                  // packed-code ring depth (steps)
constexpr int kRawSlot = 8 * 1024;                       // 128 rows x 64 B (q8) or 32 B (q4)
constexpr int kScaleSlot = 8 * 1024;                     // 128 rows x 16 (scale, min) words
constexpr uint32_t kXsTmemCols = 256;                    // 2 accumulators x 128 columns
constexpr unsigned kStatusTimeout = 5u;

struct XsLayout {
    int x_off, a_off, raw_off, sc_off, bar_off, total;
};

__host__ __device__ inline XsLayout xs_layout(int K) {
    XsLayout L;
    L.x_off = 0;
    L.a_off = (K / kAtomK) * kXAtom;
    L.raw_off = L.a_off + kAStages * kAStage;
    L.sc_off = L.raw_off + kRaw * kRawSlot;
    L.bar_off = L.sc_off + 2 * kScaleSlot;
    // raw_full/empty[kRaw], sc_full/empty[2], a_full/empty[kAStages], x_full[8],
    // x_empty, acc_full/empty[2], + TMEM address slot
    L.total = L.bar_off + (2 * kRaw + 4 + 2 * kAStages + 8 + 1 + 4) * 8 + 16;
    return L;
}

__device__ __forceinline__ uint32_t swz128(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}

__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts_v2x(uint32_t saddr, uint2 v) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(saddr), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory; completes
// `bytes` of transaction on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
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

template <int FMT, Op16 OP>
__global__ void __launch_bounds__(kXsThreads, 1)
    xs_qgemm_kernel(const __grid_constant__ CUtensorMap w_map,
                    const __grid_constant__ CUtensorMap s_map, const float *__restrict__ X,
                    const float *__restrict__ S8, float *__restrict__ Y, int M, int N, int K,
                    int n_o_tiles, int n_items, unsigned *status) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const XsLayout L = xs_layout(K);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *raw_full = bars;
    uint64_t *raw_empty = raw_full + kRaw;
    uint64_t *sc_full = raw_empty + kRaw;
    uint64_t *sc_empty = sc_full + 2;
    uint64_t *a_full = sc_empty + 2;
    uint64_t *a_empty = a_full + kAStages;
    uint64_t *x_full = a_empty + kAStages;           // one per K atom
    uint64_t *x_empty = x_full + 8;
    uint64_t *acc_full = x_empty + 1;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / kAtomK;
    const int G = gridDim.x;
    const int first = static_cast<int>((static_cast<long long>(blockIdx.x) * n_items) / G);
    const int last = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * n_items) / G);
    const uint32_t raw_bytes = kXsTileO * (FMT == 4 ? 32 : 64);
    const uint32_t sc_bytes = kXsTileO * (K / 8);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRaw; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], kDeqThreads);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sc_full[b], 1);
            mbar_init(&sc_empty[b], kDeqThreads);
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiThreads);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], kDeqThreads);
            mbar_init(&a_empty[s], 1);
        }
        for (int a = 0; a < 8; ++a) mbar_init(&x_full[a], kXldThreads);
        mbar_init(x_empty, 1);
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
    bool ok = true;

    if (warp == kTmaWarp) {
        // ============================================================ TMA issuer
        // Packed weights do not depend on the previous kernel in the stream,
        // so this role starts before the dependency wait.
        if (lane == 0) {
            int j = 0;
            for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
                const int n_local = it.item - first;
                const int y0 = it.o_tile * kXsTileO;
                if (FMT == 4) {
                    const int b = n_local & 1;
                    if (n_local >= 2 &&
                        !mbar_wait(&sc_empty[b], static_cast<uint32_t>((n_local / 2) - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&sc_full[b], sc_bytes);
                    tma_load_2d(base + L.sc_off + b * kScaleSlot, &s_map, 0, y0, &sc_full[b]);
                }
                for (int ks = 0; ks < nk; ++ks, ++j) {
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
    } else if (warp < kDeqWarps) {
        // ============================================================ dequantizers
        const int r = threadIdx.x;                   // weight row within the tile
        const int rsw = r & 7;
        const uint32_t row_a = static_cast<uint32_t>(r * 128);
        int j = 0;
        for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            if (FMT == 4 && !mbar_wait(&sc_full[b], static_cast<uint32_t>(n_local / 2) & 1u)) {
                ok = false;
                break;
            }
            const uint32_t sc_row = base + L.sc_off + b * kScaleSlot + r * (K / 8);
            for (int ks = 0; ks < nk; ++ks, ++j) {
                const int slot = j % kRaw;
                if (!mbar_wait(&raw_full[slot], static_cast<uint32_t>(j / kRaw) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t src = base + L.raw_off + slot * kRawSlot;
                uint4 p0 = make_uint4(0, 0, 0, 0), p1 = p0, p2 = p0, p3 = p0;
                uint2 smw = make_uint2(0, 0);
                if (FMT == 4) {
                    // 32 bytes of this row; the half read first alternates every 4 rows
                    // so 8 consecutive threads cover all 32 banks
                    const uint32_t h0 = ((r >> 2) & 1) * 16;
                    const uint4 u = lds_v4(src + r * 32 + h0);
                    const uint4 w = lds_v4(src + r * 32 + (16 - h0));
                    p0 = h0 ? w : u;
                    p1 = h0 ? u : w;
                    smw = lds_v2(sc_row + ks * 8);
                } else {
                    // 64 bytes of this row, read in an order rotated by (r/2) % 4
                    const int rot = (r >> 1) & 3;
                    const uint4 u0 = lds_v4(src + r * 64 + ((0 + rot) & 3) * 16);
                    const uint4 u1 = lds_v4(src + r * 64 + ((1 + rot) & 3) * 16);
                    const uint4 u2 = lds_v4(src + r * 64 + ((2 + rot) & 3) * 16);
                    const uint4 u3 = lds_v4(src + r * 64 + ((3 + rot) & 3) * 16);
                    // chunk c was read at position (c - rot) & 3
                    p0 = rot == 0 ? u0 : rot == 1 ? u3 : rot == 2 ? u2 : u1;
                    p1 = rot == 0 ? u1 : rot == 1 ? u0 : rot == 2 ? u3 : u2;
                    p2 = rot == 0 ? u2 : rot == 1 ? u1 : rot == 2 ? u0 : u3;
                    p3 = rot == 0 ? u3 : rot == 1 ? u2 : rot == 2 ? u1 : u0;
                }
                const int s = j % kAStages;
                if (j >= kAStages &&
                    !mbar_wait(&a_empty[s], static_cast<uint32_t>((j / kAStages) - 1) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = base + L.a_off + s * kAStage + row_a;
                uint4 ch[8];
                if (FMT == 4) {
                    if (OP == Op16::f16) {
                        uint32_t s0, m0, s1, m1;
                        q4_scale_min_f16x2(smw.x, s0, m0);
                        q4_scale_min_f16x2(smw.y, s1, m1);
                        ch[0] = q4_word_f16(p0.x, s0, m0);
                        ch[1] = q4_word_f16(p0.y, s0, m0);
                        ch[2] = q4_word_f16(p0.z, s0, m0);
                        ch[3] = q4_word_f16(p0.w, s0, m0);
                        ch[4] = q4_word_f16(p1.x, s1, m1);
                        ch[5] = q4_word_f16(p1.y, s1, m1);
                        ch[6] = q4_word_f16(p1.z, s1, m1);
                        ch[7] = q4_word_f16(p1.w, s1, m1);
                    } else {
                        float sc0, mn0, sc1, mn1;
                        q4_scale_min(smw.x, sc0, mn0);
                        q4_scale_min(smw.y, sc1, mn1);
                        ch[0] = q4_word_bf16(p0.x, sc0, mn0);
                        ch[1] = q4_word_bf16(p0.y, sc0, mn0);
                        ch[2] = q4_word_bf16(p0.z, sc0, mn0);
                        ch[3] = q4_word_bf16(p0.w, sc0, mn0);
                        ch[4] = q4_word_bf16(p1.x, sc1, mn1);
                        ch[5] = q4_word_bf16(p1.y, sc1, mn1);
                        ch[6] = q4_word_bf16(p1.z, sc1, mn1);
                        ch[7] = q4_word_bf16(p1.w, sc1, mn1);
                    }
                } else {
                    if (OP == Op16::f16) {
                        ch[0] = q8_words_f16(p0.x, p0.y);
                        ch[1] = q8_words_f16(p0.z, p0.w);
                        ch[2] = q8_words_f16(p1.x, p1.y);
                        ch[3] = q8_words_f16(p1.z, p1.w);
                        ch[4] = q8_words_f16(p2.x, p2.y);
                        ch[5] = q8_words_f16(p2.z, p2.w);
                        ch[6] = q8_words_f16(p3.x, p3.y);
                        ch[7] = q8_words_f16(p3.z, p3.w);
                    } else {
                        ch[0] = q8_words_bf16(p0.x, p0.y);
                        ch[1] = q8_words_bf16(p0.z, p0.w);
                        ch[2] = q8_words_bf16(p1.x, p1.y);
                        ch[3] = q8_words_bf16(p1.z, p1.w);
                        ch[4] = q8_words_bf16(p2.x, p2.y);
                        ch[5] = q8_words_bf16(p2.z, p2.w);
                        ch[6] = q8_words_bf16(p3.x, p3.y);
                        ch[7] = q8_words_bf16(p3.z, p3.w);
                    }
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) sts_v4(sa + ((c ^ rsw) << 4), ch[c]);
                fence_proxy_async_smem();
                mbar_arrive(&a_full[s]);
                // The raw slot is handed back only now: its contents have been
                // consumed into the converted chunks above, and the proxy fence
                // orders these generic reads before the TMA (async proxy) that
                // refills the slot once the issuer sees the arrival.  Releasing
                // right after the loads let a refill overtake them.
                mbar_arrive(&raw_empty[slot]);
            }
            if (!ok) break;
            if (FMT == 4) mbar_arrive(&sc_empty[b]);
        }
    } else if (warp < kMmaWarp) {
        // ============================================================ activation loaders
        pdl_wait_prior_grid();
        const int t = threadIdx.x - kXldWarp0 * 32;      // 0..127
        const int p = t & 15, rb0 = t >> 4;              // piece, first row (8 rows per pass)
        const uint32_t xb_off = swz128(rb0, p >> 1) + (p & 1) * 8;
        int cur_m = -1, x_loads = 0;
        for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
            if (it.m_tile == cur_m) continue;
            cur_m = it.m_tile;
            if (x_loads > 0 && !mbar_wait(x_empty, static_cast<uint32_t>(x_loads - 1) & 1u)) {
                ok = false;
                break;
            }
            const int m0 = cur_m * kXsTileM;
            const float *xr = X + static_cast<size_t>(m0 + rb0) * K + p * 4;
            // one atom = 16 float4 per thread (rows rb0 + 8 i), handled in two halves of 8
            auto load8 = [&](float4 (&v)[8], int a, int half) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = rb0 + 8 * (half * 8 + i);
                    v[i] = (m0 + rr < M)
                               ? ldg_f4(xr + static_cast<size_t>(8 * (half * 8 + i)) * K + a * kAtomK)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            };
            auto store8 = [&](const float4 (&v)[8], int a, int half) {
                const uint32_t xa = base + L.x_off + a * kXAtom + xb_off;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    sts_v2x(xa + 1024u * (half * 8 + i), x4_op<OP>(v[i]));
            };
            float4 v0[8], v1[8];
            load8(v0, 0, 0);
            for (int a = 0; a < nk; ++a) {
                load8(v1, a, 1);
                store8(v0, a, 0);
                if (a + 1 < nk) load8(v0, a + 1, 0);
                store8(v1, a, 1);
                fence_proxy_async_smem();
                mbar_arrive(&x_full[a]);
            }
            ++x_loads;
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            const uint32_t idesc =
                idesc_f16kind_f32acc(kXsTileO, kXsTileM, static_cast<uint32_t>(OP));
            int cur_m = -1, x_loads = 0, j = 0;
            for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
                const int n_local = it.item - first;
                const int b = n_local & 1;
                const bool new_x = it.m_tile != cur_m;
                if (new_x) {
                    cur_m = it.m_tile;
                    ++x_loads;
                }
                // accumulator b must have been drained by the epilogue
                if (n_local >= 2 &&
                    !mbar_wait(&acc_empty[b], static_cast<uint32_t>((n_local / 2) - 1) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d = tmem + static_cast<uint32_t>(b * kXsTileM);
                for (int ks = 0; ks < nk; ++ks, ++j) {
                    if (new_x &&
                        !mbar_wait(&x_full[ks], static_cast<uint32_t>(x_loads - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    const int s = j % kAStages;
                    if (!mbar_wait(&a_full[s], static_cast<uint32_t>(j / kAStages) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t adesc = sw128_kmajor_desc(base + L.a_off + s * kAStage);
                    const uint64_t bdesc = sw128_kmajor_desc(base + L.x_off + ks * kXAtom);
#pragma unroll
                    for (int kk = 0; kk < kAtomK / 16; ++kk)
                        tc_mma_f16kind(d, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                       (ks > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&a_empty[s]);
                }
                if (!ok) break;
                tc_commit(&acc_full[b]);
                // last item of this activation block with another block to
                // follow: release the X tile once these MMAs have completed
                if (it.item + 1 < last && it.o_tile + 1 == n_o_tiles) tc_commit(x_empty);
            }
        }
        __syncwarp();
    } else {
        // ============================================================ epilogue
        const int q = warp & 3;                       // TMEM lane quadrant of this warp
        const int row = q * 32 + lane;
        const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
        for (ItemCursor it(first, last, n_o_tiles); it.valid() && ok; it.next()) {
            const int n_local = it.item - first;
            const int b = n_local & 1;
            ok = mbar_wait(&acc_full[b], static_cast<uint32_t>(n_local / 2) & 1u);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            const int m0 = it.m_tile * kXsTileM;
            const int o = it.o_tile * kXsTileO + row;
            float sc = 1.f;
            if (FMT == 8 && o < N) sc = __ldg(S8 + o);
            const int mlim = min(kXsTileM, M - m0);
            float *yo = Y + static_cast<size_t>(m0) * N + o;
            for (int c = 0; c < kXsTileM; c += 16) {
                uint32_t v[16];
                tmem_ld_x16(tq + static_cast<uint32_t>(b * kXsTileM + c), v);
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
        tmem_dealloc(tmem, kXsTmemCols);
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Row-major 2-D tensor [rows, cols] of `esize`-byte elements; box = {bcols, 128}.
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, int esize, const void *ptr,
               uint64_t cols, uint64_t rows, uint32_t bcols) {
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
    cuuint32_t box[2] = {bcols, static_cast<cuuint32_t>(kXsTileO)};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, Op16 OP>
cudaError_t launch_xs(const float *X, const void *Wq, const void *S, float *Y, int M, int N,
                      int K, unsigned *status, cudaStream_t st) {
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(xs_qgemm_kernel<FMT, OP>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    CUtensorMap w_map, s_map;
    bool enc_ok;
    if (FMT == 4) {
        enc_ok = encode_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K / 2, N, 32) &&
                 encode_2d(&s_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, S, K / 32, N, K / 32);
    } else {
        enc_ok = encode_2d(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, K, N, 64);
        s_map = w_map;   // unused by the q8 kernel
    }
    if (!enc_ok) return cudaErrorInvalidValue;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_o = (N + kXsTileO - 1) / kXsTileO;
    const int n_m = (M + kXsTileM - 1) / kXsTileM;
    const int items = n_o * n_m;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(std::min(items, sms), 1, 1);
    cfg.blockDim = dim3(kXsThreads, 1, 1);
    cfg.dynamicSmemBytes = xs_layout(K).total + 1024;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, xs_qgemm_kernel<FMT, OP>, w_map, s_map, X,
                              static_cast<const float *>(S), Y, M, N, K, n_o, items, status);
}

}  // namespace

// Shapes the activation-resident kernel takes: K a multiple of 128 up to 512
// (the (scale, min) rows are TMA boxes, whose global stride K/8 bytes must be
// a multiple of 16), at least two activation blocks, and enough work items
// to give most SMs one.
bool xs_supported(int M, int N, int K) {
    if (K % 128 != 0 || K > kXsMaxK) return false;
    const long items = static_cast<long>((N + kXsTileO - 1) / kXsTileO) *
                       ((M + kXsTileM - 1) / kXsTileM);
    return M >= 2 * kXsTileM && items >= 96;
}

cudaError_t launch_xs_q4(const float *X, const uint8_t *Wq, const uint16_t *SM, float *Y, int M,
                         int N, int K, bool bf16, unsigned *status, cudaStream_t s) {
    return bf16 ? launch_xs<4, Op16::bf16>(X, Wq, SM, Y, M, N, K, status, s)
                : launch_xs<4, Op16::f16>(X, Wq, SM, Y, M, N, K, status, s);
}

cudaError_t launch_xs_q8(const float *X, const int8_t *Wq, const float *S, float *Y, int M, int N,
                         int K, bool bf16, unsigned *status, cudaStream_t s) {
    return bf16 ? launch_xs<8, Op16::bf16>(X, Wq, S, Y, M, N, K, status, s)
                : launch_xs<8, Op16::f16>(X, Wq, S, Y, M, N, K, status, s);
}

}  // namespace rtq
