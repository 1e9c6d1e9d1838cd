// Parameters of the projection-list kernel (pl.cu): the projections, their
// weights' TMA tensor maps, the work items cut from them and each CTA's
// share, passed by value as one __grid_constant__ kernel parameter (under the
// 32 KB parameter limit).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace rtq {

constexpr int kPlMaxProj = 64;      // projections per launch
constexpr int kPlMaxItems = 1440;   // work items per launch
constexpr int kPlMaxCtas = 160;     // >= the SM count of one B200
constexpr int kPlMaxAcc = 8;        // accumulators in the TMEM ring

struct PlProj {
    const uint8_t *Xh;   // fp16 image of the projection's activations (pre-pass output)
    const void *Wq;      // q4: u8 [N, K/2]; q8: i8 [N, K]
    const void *S;       // q4: binary16 (scale, min) [N, K/32, 2]; q8: fp32 [N]
    const float *bias;   // fp32 [N] or null
    float *Y;            // fp32 [M, N]
    int N, K, fmt, xid;  // xid: index of the distinct activation image
    int pad;
};

// One work item: tiles [tile0, tile0 + ntiles) of a projection over all of
// K, 512-wide chunk by chunk.  A projection with K > 512 has one tile per
// item, its accumulator kept in TMEM across the chunks.
struct PlItem {
    uint32_t tile0;
    uint16_t proj;       // index into PlParams::proj
    uint8_t ntiles;
    uint8_t pad;
};

struct PlParams {
    // per projection: its codes as a [N, row bytes] u8 tensor (boxes of 128
    // rows x 128 bytes, 128-byte swizzle) and, for q4, its (scale, min) words
    // as a [N, K/32] u32 tensor (boxes of 128 rows x 16 words, 64-byte swizzle)
    CUtensorMap wmap[kPlMaxProj];
    CUtensorMap smap[kPlMaxProj];
    int M, bnp, nslots, nacc;
    int cta_items[kPlMaxCtas + 1];   // CTA b runs items [cta_items[b], cta_items[b + 1])
    PlProj proj[kPlMaxProj];
    PlItem items[kPlMaxItems];
};

struct PlPrepImage {
    const float *X;      // fp32 [M, K]
    uint8_t *Xh;         // fp16 image, pl_image_bytes(M, K) bytes
    int K, pad;
};

struct PlPrep {
    int M, bnp;
    PlPrepImage img[kPlMaxProj];
};

static_assert(sizeof(PlParams) + 8 <= 32764, "kernel parameter limit");
static_assert(sizeof(PlPrep) + 8 <= 32764, "kernel parameter limit");

}  // namespace rtq
