// Host-side quantizers that produce the packed tensors the GEMM kernels read.
//
// q4 g32: "RT-J -- int4 (Q4-style, mixed-precision) quantized checkpoints",
//   section "Quantization format" -- uint4 codes per group of 32 inputs, one
//   fp16 (scale, min) pair per group, W ~= code*scale + min, group range from
//   a min-MSE clip search over the shrink grid 1.0 -> 0.8.
// q8 per-row: "RT-J -- int8 (Q8_0-style) quantized checkpoints", section
//   "Quantization format" -- scale[o] = max|W[o,:]|/127, W ~= q*scale[o].
// e4m3: "RT-J -- FP8 E4M3 checkpoints", section "FP8 Format" -- weight
//   matrices hold float8_e4m3fn values, no scale.
//
// The grid, rounding and tie rules are spelled out in include/rtq.h.  All
// weight arithmetic is IEEE double with no contraction (this file is built
// with -ffp-contract=off); binary16 rounding uses the compiler's _Float16
// conversion, which rounds a double once, to nearest-even.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "../../include/rtq.h"

namespace {

inline uint16_t half_bits(double x) {
    _Float16 h = static_cast<_Float16>(x);
    uint16_t b;
    std::memcpy(&b, &h, sizeof b);
    return b;
}

inline double half_value(uint16_t b) {
    _Float16 h;
    std::memcpy(&h, &b, sizeof h);
    return static_cast<double>(h);
}

inline double grid_factor(int j, int n_grid) {
    return n_grid > 1 ? 1.0 - (0.2 * j) / (n_grid - 1) : 1.0;
}

void q4_rows(const float *W, int64_t r0, int64_t r1, int64_t K, int n_grid, uint8_t *Wq,
             uint16_t *sm) {
    const int64_t G = K / 32;
    for (int64_t o = r0; o < r1; ++o) {
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + o * K + g * 32;
            float lo_f = w[0], hi_f = w[0];
            for (int i = 1; i < 32; ++i) {
                lo_f = std::min(lo_f, w[i]);
                hi_f = std::max(hi_f, w[i]);
            }
            const double lo = lo_f, hi = hi_f;
            double best_err = INFINITY;
            uint16_t best_sc = 0, best_mn = 0;
            uint8_t best_q[32] = {0};
            for (int j = 0; j < n_grid; ++j) {
                const double s = grid_factor(j, n_grid);
                const double lo_j = s * lo, hi_j = s * hi;
                const uint16_t sc_b = half_bits((hi_j - lo_j) / 15.0);
                const uint16_t mn_b = half_bits(lo_j);
                const double sc = half_value(sc_b), mn = half_value(mn_b);
                uint8_t q[32];
                double err = 0.0;
                for (int i = 0; i < 32; ++i) {
                    const double wi = w[i];
                    int qi = 0;
                    if (sc != 0.0) {
                        const double t = std::nearbyint((wi - mn) / sc);
                        qi = t < 0.0 ? 0 : (t > 15.0 ? 15 : static_cast<int>(t));
                    }
                    q[i] = static_cast<uint8_t>(qi);
                    const double d = wi - (qi * sc + mn);
                    err += d * d;
                }
                if (err < best_err) {
                    best_err = err;
                    best_sc = sc_b;
                    best_mn = mn_b;
                    std::memcpy(best_q, q, sizeof q);
                }
            }
            uint8_t *dst = Wq + o * (K / 2) + g * 16;
            for (int b = 0; b < 16; ++b)
                dst[b] = static_cast<uint8_t>(best_q[2 * b] | (best_q[2 * b + 1] << 4));
            sm[(o * G + g) * 2 + 0] = best_sc;
            sm[(o * G + g) * 2 + 1] = best_mn;
        }
    }
}

void q8_rows(const float *W, int64_t r0, int64_t r1, int64_t K, int8_t *Wq, float *scale) {
    for (int64_t o = r0; o < r1; ++o) {
        const float *w = W + o * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) amax = std::max(amax, std::fabs(w[k]));
        const float sc = amax / 127.0f;
        scale[o] = sc;
        for (int64_t k = 0; k < K; ++k) {
            int q = 0;
            if (sc != 0.0f) {
                const double t = std::nearbyint(static_cast<double>(w[k]) / static_cast<double>(sc));
                q = t < -127.0 ? -127 : (t > 127.0 ? 127 : static_cast<int>(t));
            }
            Wq[o * K + k] = static_cast<int8_t>(q);
        }
    }
}

// Splits rows over hardware threads; each row is independent, so the result
// does not depend on the split.
template <class F>
void parallel_rows(int64_t N, int64_t work_per_row, F &&fn) {
    unsigned hw = std::max(1u, std::thread::hardware_concurrency());
    int64_t want = std::max<int64_t>(1, (N * work_per_row) / (1 << 16));
    int64_t T = std::min<int64_t>({static_cast<int64_t>(hw), want, std::max<int64_t>(N, 1)});
    if (T <= 1) {
        fn(0, N);
        return;
    }
    std::vector<std::thread> pool;
    const int64_t chunk = (N + T - 1) / T;
    for (int64_t t = 0; t < T; ++t) {
        const int64_t a = t * chunk, b = std::min(N, a + chunk);
        if (a < b) pool.emplace_back(fn, a, b);
    }
    for (auto &th : pool) th.join();
}

}  // namespace

extern "C" rt_status rt_quantize_q4_g32(const float *W, int64_t N, int64_t K, int n_grid,
                                        uint8_t *Wq, uint16_t *scale_min) {
    if (N < 0 || K < 0 || n_grid < 0) return RT_ERR_INVALID_ARG;
    if (K % 32 != 0) return RT_ERR_UNSUPPORTED_SHAPE;
    if (N == 0 || K == 0) return RT_OK;
    if (!W || !Wq || !scale_min) return RT_ERR_INVALID_ARG;
    if (n_grid == 0) n_grid = 21;
    for (int64_t i = 0; i < N * K; ++i)
        if (!std::isfinite(W[i]) || std::fabs(W[i]) > 65504.0f) return RT_ERR_VALUE_RANGE;
    parallel_rows(N, K * n_grid, [&](int64_t a, int64_t b) {
        q4_rows(W, a, b, K, n_grid, Wq, scale_min);
    });
    return RT_OK;
}

extern "C" rt_status rt_quantize_q8_row(const float *W, int64_t N, int64_t K, int8_t *Wq,
                                        float *scale) {
    if (N < 0 || K < 0) return RT_ERR_INVALID_ARG;
    if (N == 0) return RT_OK;
    if (!W || !Wq || !scale) return RT_ERR_INVALID_ARG;
    for (int64_t i = 0; i < N * K; ++i)
        if (!std::isfinite(W[i])) return RT_ERR_VALUE_RANGE;
    parallel_rows(N, K, [&](int64_t a, int64_t b) { q8_rows(W, a, b, K, Wq, scale); });
    return RT_OK;
}

namespace {

// One weight to its float8_e4m3fn code: round to nearest, ties to even, from
// the binade of |w|.  Below 2^-6 the step is 2^-9 (subnormal codes 0..7; a
// rounded 8 is the smallest normal code 0x08); from 2^-6 on, |w| = f * 2^E
// with f in [1, 2) takes code ((E + 7) << 3) + round(8 (f - 1)), where a
// rounded 8 carries into the exponent field.  Returns false for NaN and for
// |w| > 464, which would round past the largest finite value 448.
inline bool e4m3_code(float w, uint8_t *out) {
    const double a = std::fabs(static_cast<double>(w));
    if (std::isnan(w) || a > 464.0) return false;
    int code;
    if (a < 0.015625) {
        code = static_cast<int>(std::nearbyint(a * 512.0));
    } else {
        int E = 0;
        const double f = 2.0 * std::frexp(a, &E);   // a = f * 2^(E - 1), f in [1, 2)
        code = ((E - 1 + 7) << 3) + static_cast<int>(std::nearbyint((f - 1.0) * 8.0));
    }
    *out = static_cast<uint8_t>(code | (std::signbit(w) ? 0x80 : 0));
    return true;
}

}  // namespace

extern "C" rt_status rt_quantize_e4m3(const float *W, int64_t n, uint8_t *out) {
    if (n < 0) return RT_ERR_INVALID_ARG;
    if (n == 0) return RT_OK;
    if (!W || !out) return RT_ERR_INVALID_ARG;
    for (int64_t i = 0; i < n; ++i)
        if (!e4m3_code(W[i], &out[i])) return RT_ERR_VALUE_RANGE;
    return RT_OK;
}
