// Device pieces shared by the TMA-fed tcgen05 kernels (xs.cu, ws.cu):
// TMA loads and transaction barriers, shared-memory vector accesses, the
// 32x32b.x16 TMEM load, and the per-row dequantization step of the weight
// stream (one thread converts one 128-byte row of a 64-wide K slice).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "dequant.cuh"
#include "ptx.cuh"

namespace rtq {

constexpr int kTileRows = 128;      // MMA M (weight rows) and TMA box height
constexpr int kAtomK = 64;          // K per stage: one 128-byte row of 16-bit operands
constexpr int kOpStage = kTileRows * 128;   // 16 KB: one 128 x 64 16-bit operand tile

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

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory; completes
// its bytes of transaction on `bar`.  x (innermost) must be a multiple of 16
// bytes' worth of elements.
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

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// Raw bytes of one weight row for one K step, as staged by TMA: q4 -> 32 B
// of codes (row r at r*32) plus the two (scale, min) words of its groups;
// q8 -> 64 B of codes (row r at r*64).  The read order is rotated with the
// row so that 8 consecutive threads touch all 32 banks.
struct RowRaw {
    uint4 p0, p1, p2, p3;
    uint2 smw;
};

template <int FMT>
__device__ __forceinline__ RowRaw load_row_raw(uint32_t slot, int r, uint32_t sc_addr) {
    RowRaw R;
    if (FMT == 4) {
        const uint32_t h0 = ((r >> 2) & 1) * 16;
        const uint4 u = lds_v4(slot + r * 32 + h0);
        const uint4 w = lds_v4(slot + r * 32 + (16 - h0));
        R.p0 = h0 ? w : u;
        R.p1 = h0 ? u : w;
        R.p2 = R.p3 = make_uint4(0, 0, 0, 0);
        R.smw = lds_v2(sc_addr);
    } else {
        const int rot = (r >> 1) & 3;
        const uint4 u0 = lds_v4(slot + r * 64 + ((0 + rot) & 3) * 16);
        const uint4 u1 = lds_v4(slot + r * 64 + ((1 + rot) & 3) * 16);
        const uint4 u2 = lds_v4(slot + r * 64 + ((2 + rot) & 3) * 16);
        const uint4 u3 = lds_v4(slot + r * 64 + ((3 + rot) & 3) * 16);
        // chunk c was read at position (c - rot) & 3
        R.p0 = rot == 0 ? u0 : rot == 1 ? u3 : rot == 2 ? u2 : u1;
        R.p1 = rot == 0 ? u1 : rot == 1 ? u0 : rot == 2 ? u3 : u2;
        R.p2 = rot == 0 ? u2 : rot == 1 ? u1 : rot == 2 ? u0 : u3;
        R.p3 = rot == 0 ? u3 : rot == 1 ? u2 : rot == 2 ? u1 : u0;
        R.smw = make_uint2(0, 0);
    }
    return R;
}

// Dequantizes one row's 64 weights into 8 chunks of 8 16-bit operands (in the
// operand chunk order).
template <int FMT, Op16 OP>
__device__ __forceinline__ void row_chunks(const RowRaw &R, uint4 (&ch)[8]) {
    if (FMT == 4) {
        if (OP == Op16::f16) {
            uint32_t s0, m0, s1, m1;
            q4_scale_min_f16x2(R.smw.x, s0, m0);
            q4_scale_min_f16x2(R.smw.y, s1, m1);
            ch[0] = q4_word_f16(R.p0.x, s0, m0);
            ch[1] = q4_word_f16(R.p0.y, s0, m0);
            ch[2] = q4_word_f16(R.p0.z, s0, m0);
            ch[3] = q4_word_f16(R.p0.w, s0, m0);
            ch[4] = q4_word_f16(R.p1.x, s1, m1);
            ch[5] = q4_word_f16(R.p1.y, s1, m1);
            ch[6] = q4_word_f16(R.p1.z, s1, m1);
            ch[7] = q4_word_f16(R.p1.w, s1, m1);
        } else {
            float sc0, mn0, sc1, mn1;
            q4_scale_min(R.smw.x, sc0, mn0);
            q4_scale_min(R.smw.y, sc1, mn1);
            ch[0] = q4_word_bf16(R.p0.x, sc0, mn0);
            ch[1] = q4_word_bf16(R.p0.y, sc0, mn0);
            ch[2] = q4_word_bf16(R.p0.z, sc0, mn0);
            ch[3] = q4_word_bf16(R.p0.w, sc0, mn0);
            ch[4] = q4_word_bf16(R.p1.x, sc1, mn1);
            ch[5] = q4_word_bf16(R.p1.y, sc1, mn1);
            ch[6] = q4_word_bf16(R.p1.z, sc1, mn1);
            ch[7] = q4_word_bf16(R.p1.w, sc1, mn1);
        }
    } else {
        if (OP == Op16::f16) {
            ch[0] = q8_words_f16(R.p0.x, R.p0.y);
            ch[1] = q8_words_f16(R.p0.z, R.p0.w);
            ch[2] = q8_words_f16(R.p1.x, R.p1.y);
            ch[3] = q8_words_f16(R.p1.z, R.p1.w);
            ch[4] = q8_words_f16(R.p2.x, R.p2.y);
            ch[5] = q8_words_f16(R.p2.z, R.p2.w);
            ch[6] = q8_words_f16(R.p3.x, R.p3.y);
            ch[7] = q8_words_f16(R.p3.z, R.p3.w);
        } else {
            ch[0] = q8_words_bf16(R.p0.x, R.p0.y);
            ch[1] = q8_words_bf16(R.p0.z, R.p0.w);
            ch[2] = q8_words_bf16(R.p1.x, R.p1.y);
            ch[3] = q8_words_bf16(R.p1.z, R.p1.w);
            ch[4] = q8_words_bf16(R.p2.x, R.p2.y);
            ch[5] = q8_words_bf16(R.p2.z, R.p2.w);
            ch[6] = q8_words_bf16(R.p3.x, R.p3.y);
            ch[7] = q8_words_bf16(R.p3.z, R.p3.w);
        }
    }
}

// Dequantizes one row's 64 weights and writes them as 8 swizzled 16-byte
// chunks of row r of an A stage in shared memory (sa = stage base).
template <int FMT, Op16 OP>
__device__ __forceinline__ void store_row_op(const RowRaw &R, uint32_t sa, int r) {
    uint4 ch[8];
    row_chunks<FMT, OP>(R, ch);
    const uint32_t row = sa + static_cast<uint32_t>(r * 128);
    const int rsw = r & 7;
#pragma unroll
    for (int c = 0; c < 8; ++c) sts_v4(row + ((c ^ rsw) << 4), ch[c]);
}

// Dequantizes one row's 64 weights into 32 TMEM columns of this thread's lane
// (ta = the warp's lane base | first column): column 4c + i holds 32-bit word
// i of chunk c, i.e. K values 8c + 2i and 8c + 2i + 1 of the operand order.
// Must be reached by the whole warp (tcgen05.st is warp-collective).
template <int FMT, Op16 OP>
__device__ __forceinline__ void tmem_row_op(const RowRaw &R, uint32_t ta) {
    uint4 ch[8];
    row_chunks<FMT, OP>(R, ch);
    uint32_t w[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        w[4 * c + 0] = ch[c].x;
        w[4 * c + 1] = ch[c].y;
        w[4 * c + 2] = ch[c].z;
        w[4 * c + 3] = ch[c].w;
    }
    tmem_st_x32(ta, w);
}

// ---------------------------------------------------------------- host side
// Row-major 2-D tensor [rows, cols] of `esize`-byte elements as a TMA map
// with box {bcols, 128}; swizzle as given.  Returns false if the driver
// rejects it.
bool encode_tma_2d(CUtensorMap *map, CUtensorMapDataType dt, int esize, const void *ptr,
                   uint64_t cols, uint64_t rows, uint32_t bcols, CUtensorMapSwizzle swizzle);

}  // namespace rtq
