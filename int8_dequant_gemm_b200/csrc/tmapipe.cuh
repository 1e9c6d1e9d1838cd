// Device pieces shared by the TMA-fed tcgen05 kernels (xs.cu, ws.cu):
// TMA loads and transaction barriers, shared-memory vector accesses, TMEM
// loads and stores, and the half-row dequantization step of the weight
// stream (two threads per weight row and 64-wide K step).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "dequant.cuh"
#include "ptx.cuh"

namespace rtq {

constexpr int kTileRows = 128;      // MMA M (weight rows) and TMA box height
constexpr int kAtomK = 64;          // K per stage: one 128-byte row of 16-bit operands
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

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
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

// ---------------------------------------------- half-row dequantization
// The TMA-fed kernels split every K step between two threads per weight row:
// thread (r, h) converts K values [32h, 32h + 32) of the 64-wide step of row r
// into 16 TMEM columns.  Each step's A stage is then written by all dequant
// threads at once, which halves the latency from "stage free" to "stage
// full" -- the quantity that bounds a shallow ring of TMEM stages.

// One thread's raw bytes for one step: q4 -> 16 B of codes (one 32-group)
// plus that group's (scale, min) word; q8 -> 32 B of codes.
struct HalfRaw {
    uint4 p0, p1;
    uint32_t smw;
};

// A half-row read from a slot that holds two K steps per row, as one
// TMA box in a swizzled layout: q4 rows of 64 bytes (SWIZZLE_64B: 16-byte
// chunk c of row r sits at chunk c ^ ((r >> 1) & 3)), q8 rows of 128 bytes
// (SWIZZLE_128B: chunk c at c ^ (r & 7)).  u selects the step within the
// pair.  A TMA box costs about 3 cycles per row whatever its width, so two
// steps per box halve the weight stream's TMA time per step; the swizzle
// keeps 8 consecutive rows on 8 different bank groups.
template <int FMT>
__device__ __forceinline__ HalfRaw load_half_raw2(uint32_t slot, int r, int h, int u, uint32_t smw) {
    HalfRaw R;
    if (FMT == 4) {
        const int c = (2 * u + h) ^ ((r >> 1) & 3);
        R.p0 = lds_v4(slot + r * 64 + c * 16);
        R.p1 = make_uint4(0, 0, 0, 0);
        R.smw = smw;
    } else {
        const int c0 = 4 * u + 2 * h;
        R.p0 = lds_v4(slot + r * 128 + ((c0 ^ (r & 7)) * 16));
        R.p1 = lds_v4(slot + r * 128 + (((c0 + 1) ^ (r & 7)) * 16));
        R.smw = 0;
    }
    return R;
}

// 32 weights of a half step -> 16 32-bit fp16 operand words (4 chunks).
template <int FMT>
__device__ __forceinline__ void half_words(const HalfRaw &R, uint32_t (&w)[16]) {
    uint4 ch[4];
    if (FMT == 4) {
        uint32_t s2, m2;
        q4_scale_min_f16x2(R.smw, s2, m2);
        ch[0] = q4_word_f16(R.p0.x, s2, m2);
        ch[1] = q4_word_f16(R.p0.y, s2, m2);
        ch[2] = q4_word_f16(R.p0.z, s2, m2);
        ch[3] = q4_word_f16(R.p0.w, s2, m2);
    } else if (FMT == 8) {
        ch[0] = q8_words_f16(R.p0.x, R.p0.y);
        ch[1] = q8_words_f16(R.p0.z, R.p0.w);
        ch[2] = q8_words_f16(R.p1.x, R.p1.y);
        ch[3] = q8_words_f16(R.p1.z, R.p1.w);
    } else {   // e4m3: the q8 byte layout, another conversion
        ch[0] = e4m3_words_f16(R.p0.x, R.p0.y);
        ch[1] = e4m3_words_f16(R.p0.z, R.p0.w);
        ch[2] = e4m3_words_f16(R.p1.x, R.p1.y);
        ch[3] = e4m3_words_f16(R.p1.z, R.p1.w);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        w[4 * c + 0] = ch[c].x;
        w[4 * c + 1] = ch[c].y;
        w[4 * c + 2] = ch[c].z;
        w[4 * c + 3] = ch[c].w;
    }
}

// The (scale, min) words of row r for 8 K steps: a 64-byte row of a staged
// block (16 words, groups 0..15 of the block).  Thread (r, h) keeps word
// 2i + h, the group of step i's half h.  The four 16-byte reads are rotated
// with the row so that 8 consecutive rows hit 32 different banks.
__device__ __forceinline__ void load_scale_words(uint32_t row, int r, int h, uint32_t (&sw)[8]) {
    const int rot = (r >> 1) & 3;
    uint4 u[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) u[c] = lds_v4(row + ((c + rot) & 3) * 16);
    // u[c] holds chunk (c + rot) & 3; chunk k therefore sits at u[(k - rot) & 3]
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int i0 = (k - 0) & 3, i1 = (k - 1) & 3, i2 = (k - 2) & 3, i3 = (k - 3) & 3;
        const uint4 v = rot == 0 ? u[i0] : rot == 1 ? u[i1] : rot == 2 ? u[i2] : u[i3];
        // chunk k = words 4k .. 4k + 3 = steps 2k (words 4k, 4k + 1) and 2k + 1
        sw[2 * k] = h ? v.y : v.x;
        sw[2 * k + 1] = h ? v.w : v.z;
    }
}

// The (scale, min) words of row r for 8 K steps when thread (r, h) converts
// whole steps (step 2i + h of each pair i): it keeps the words of that step's
// two groups, 4i + 2h and 4i + 2h + 1, as sw[2i], sw[2i + 1].  Same rotated
// reads as load_scale_words.
__device__ __forceinline__ void load_scale_pairs(uint32_t row, int r, int h, uint32_t (&sw)[8]) {
    const int rot = (r >> 1) & 3;
    uint4 u[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) u[c] = lds_v4(row + ((c + rot) & 3) * 16);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int i0 = (k - 0) & 3, i1 = (k - 1) & 3, i2 = (k - 2) & 3, i3 = (k - 3) & 3;
        const uint4 v = rot == 0 ? u[i0] : rot == 1 ? u[i1] : rot == 2 ? u[i2] : u[i3];
        // chunk k = words 4k .. 4k + 3: step 2k (words 4k, 4k + 1), step 2k + 1
        sw[2 * k] = h ? v.z : v.x;
        sw[2 * k + 1] = h ? v.w : v.y;
    }
}

// ---------------------------------------------------------------- host side
// Row-major 2-D tensor [rows, cols] of `esize`-byte elements as a TMA map
// with box {bcols, brows}; swizzle as given.  Returns false if the driver
// rejects it.
bool encode_tma_2d(CUtensorMap *map, CUtensorMapDataType dt, int esize, const void *ptr,
                   uint64_t cols, uint64_t rows, uint32_t bcols, CUtensorMapSwizzle swizzle,
                   uint32_t brows = kTileRows);

}  // namespace rtq
