// Device-side dequantization of the two weight formats.  Every kernel of the
// library (SIMT GEMM, tensor-core GEMM, dequant exports) goes through these
// routines, so the exports test exactly what the GEMMs consume.
//
// q4 ("RT-J -- int4 ... quantized checkpoints", "Quantization format"):
//   a 32-bit word of the payload holds 8 consecutive codes of one row; byte b
//   holds code 2b in its low nibble and 2b+1 in its high nibble, so code i of
//   the word sits in bits [4i, 4i+4).  W = code*scale + min with the group's
//   binary16 (scale, min) widened to fp32; code*scale is exact in fp32 (4-bit
//   times 11-bit significands), so one fmaf yields the exact value rounded
//   once to fp32.
// q8 ("RT-J -- int8 ... quantized checkpoints", "Quantization format"):
//   W = q * scale[o]; q (|q| <= 127) is exact in fp32 and in fp16.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

namespace rtq {

// Integer 0..255 to fp32 without the I2F pipe: 2^23 + v has v in its low
// mantissa bits, and subtracting 2^23 is exact.
__device__ __forceinline__ float small_uint_to_f32(uint32_t v) {
    return __fsub_rn(__uint_as_float(0x4B000000u | v), 8388608.0f);
}

// (scale, min) pair packed as two binary16 values in one 32-bit word
// (scale in the low half, as stored: element 0 then element 1).
__device__ __forceinline__ void q4_scale_min(uint32_t sm, float &scale, float &mn) {
    scale = __half2float(__ushort_as_half(static_cast<unsigned short>(sm & 0xFFFFu)));
    mn = __half2float(__ushort_as_half(static_cast<unsigned short>(sm >> 16)));
}

// 8 codes of one payload word -> 8 fp32 weights.
__device__ __forceinline__ void q4_word_f32(uint32_t v, float scale, float mn, float (&w)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = fmaf(small_uint_to_f32((v >> (4 * i)) & 0xFu), scale, mn);
}

// Tensor-core operand chunks hold 8 consecutive K elements k .. k+7 as the
// four fp16 pairs (k + t, k + t + 4), t = 0..3, one 32-bit word per pair.
// Weights and activations use the same order, so the MMA's dot products are
// unchanged.  The order lets a q4 payload word (8 codes, code i in bits
// 4i .. 4i+3) split into its four pairs with one shift and four masks, each
// mask also setting the fp16 exponent pattern (see q4_word_f16); the two
// one-byte formats take one byte permute per pair.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 8 activations k .. k+7 (a = k .. k+3, b = k+4 .. k+7) -> one operand chunk,
// rounded to nearest-even.
__device__ __forceinline__ uint4 x8_f16(float4 a, float4 b) {
    return make_uint4(pack_f16x2(a.x, b.x), pack_f16x2(a.y, b.y), pack_f16x2(a.z, b.z),
                      pack_f16x2(a.w, b.w));
}

// Non-zero where a half of an fp16 pair word is infinite or NaN (exponent
// field all ones): an activation that fp16 cannot hold (|x| >= 65520 rounds
// to infinity) or that was not finite to begin with.
__device__ __forceinline__ uint32_t f16x2_nonfinite(uint2 w) {
    return __vcmpeq2(w.x & 0x7C007C00u, 0x7C007C00u) | __vcmpeq2(w.y & 0x7C007C00u, 0x7C007C00u);
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// q4, fp16 operands: 8 codes of one payload word -> one chunk.  Code i sits
// in bits 4i .. 4i+3, so codes t and t + 4 are the same nibble of the two
// 16-bit halves: in bits 0-3 (t = 0, and t = 2 after a shift by 8) under the
// exponent pattern 0x6400 a nibble reads as fp16 1024 + code, in bits 4-7
// (t = 1, 3) under 0x5400 as 64 + code (unit last place 1/16).  Both
// subtractions are exact; fma.rn.f16x2 then rounds code*scale + min once.
// s2 / m2 hold the group's scale / min in both halves.
__device__ __forceinline__ uint4 q4_word_f16(uint32_t v, uint32_t s2, uint32_t m2) {
    const __half2 k1024 = bits_h2(0x64006400u), k64 = bits_h2(0x54005400u);
    const __half2 s = bits_h2(s2), m = bits_h2(m2);
    const uint32_t v8 = v >> 8;
    return make_uint4(
        h2_bits(__hfma2(__hsub2(bits_h2((v & 0x000F000Fu) | 0x64006400u), k1024), s, m)),
        h2_bits(__hfma2(__hsub2(bits_h2((v & 0x00F000F0u) | 0x54005400u), k64), s, m)),
        h2_bits(__hfma2(__hsub2(bits_h2((v8 & 0x000F000Fu) | 0x64006400u), k1024), s, m)),
        h2_bits(__hfma2(__hsub2(bits_h2((v8 & 0x00F000F0u) | 0x54005400u), k64), s, m)));
}

// (scale, min) word -> (scale, scale) and (min, min).
__device__ __forceinline__ void q4_scale_min_f16x2(uint32_t sm, uint32_t &s2, uint32_t &m2) {
    s2 = __byte_perm(sm, 0u, 0x1010);
    m2 = __byte_perm(sm, 0u, 0x3232);
}

// int8 code (byte i of v, two's complement) -> fp32, exact.
__device__ __forceinline__ float q8_byte_f32(uint32_t v, int i) {
    // offset-binary byte (q + 128) in 0..255, then remove 2^23 + 128 exactly
    const uint32_t u = ((v ^ 0x80808080u) >> (8 * i)) & 0xFFu;
    return __fsub_rn(__uint_as_float(0x4B000000u | u), 8388736.0f);
}

// q8, fp16 operands: two payload words (codes 0..3, 4..7) -> one chunk.  The
// offset-binary byte q + 128 under an 0x64 high byte is fp16 1024 + q + 128;
// subtracting 1152 leaves q exactly.
// Byte t of a and byte t of b in the low bytes of the two 16-bit halves
// (the high bytes are bytes of a and b too: callers mask them).
__device__ __forceinline__ uint32_t pair_bytes(uint32_t a, uint32_t b, int t) {
    return __byte_perm(a, b, static_cast<uint32_t>(t | (t << 4) | ((4 + t) << 8) | ((4 + t) << 12)));
}

__device__ __forceinline__ uint4 q8_words_f16(uint32_t a, uint32_t b) {
    const __half2 k1152 = bits_h2(0x64806480u);
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t)   // mask the bytes, flip bit 7, set the 0x64 high bytes: one op
        w[t] = h2_bits(__hsub2(bits_h2((pair_bytes(a, b, t) & 0x00FF00FFu) ^ 0x64806480u), k1152));
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// FP8 E4M3 ("RT-J -- FP8 E4M3 checkpoints", "FP8 Format": weights stored
// directly as float8_e4m3fn, no scale).  A code b = S EEEE MMM reads as
// (1 + M/8) * 2^(E-7), or M * 2^-9 when E = 0.  Its low seven bits shifted left
// by 7 are an fp16 pattern worth exactly that value times 2^-8 (exponent bias
// 15 instead of 7; the E = 0 codes land on fp16 subnormals with the same
// factor), so one exact fp16 multiplication by 256 finishes the conversion.
// The two NaN codes S.1111.111 are not weights; they read as +-480.
__device__ __forceinline__ uint32_t e4m3_pair_f16(uint32_t x) {
    // x holds two codes in the low bytes of its 16-bit halves
    const uint32_t h = ((x & 0x007F007Fu) << 7) | ((x & 0x00800080u) << 8);
    return h2_bits(__hmul2(bits_h2(h), bits_h2(0x5C005C00u)));   // x 256, exact
}

// e4m3, fp16 operands: two payload words (codes 0..3, 4..7) -> one chunk.
__device__ __forceinline__ uint4 e4m3_words_f16(uint32_t a, uint32_t b) {
    return make_uint4(e4m3_pair_f16(pair_bytes(a, b, 0)), e4m3_pair_f16(pair_bytes(a, b, 1)),
                      e4m3_pair_f16(pair_bytes(a, b, 2)), e4m3_pair_f16(pair_bytes(a, b, 3)));
}

// e4m3 code (byte i of v) -> fp32, exact: the integer (8 + M) << (E - 1), or
// M for E = 0, times 2^-9.
__device__ __forceinline__ float e4m3_byte_f32(uint32_t v, int i) {
    const uint32_t b = (v >> (8 * i)) & 0xFFu;
    const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
    const uint32_t mag = e == 0 ? m : (8u + m) << (e - 1);
    const float f = static_cast<float>(mag) * 0.001953125f;   // 2^-9
    return (b & 0x80u) ? -f : f;
}

// Chunk in operand order -> natural order (for the dequantization exports).
__device__ __forceinline__ uint4 chunk_to_natural(uint4 c) {
    return make_uint4(__byte_perm(c.x, c.y, 0x5410), __byte_perm(c.z, c.w, 0x5410),
                      __byte_perm(c.x, c.y, 0x7632), __byte_perm(c.z, c.w, 0x7632));
}

}  // namespace rtq
