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
//   W = q * scale[o]; q (|q| <= 127) is exact in fp32 and in bf16.
#pragma once
#include <cuda_bf16.h>
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

// Tensor-core operand types: both MMA operands share one 16-bit type.
enum class Op16 { f16 = 0, bf16 = 1 };

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Two fp32 values -> two 16-bit operands (round to nearest-even), low first.
template <Op16 OP>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    return OP == Op16::f16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

// 8 codes of one payload word -> 8 16-bit weights (the fp32 value rounded to
// the operand type), packed low element first into one 16-byte smem chunk.
template <Op16 OP>
__device__ __forceinline__ uint4 q4_word_op(uint32_t v, float scale, float mn) {
    float w[8];
    q4_word_f32(v, scale, mn, w);
    return make_uint4(pack2<OP>(w[0], w[1]), pack2<OP>(w[2], w[3]), pack2<OP>(w[4], w[5]),
                      pack2<OP>(w[6], w[7]));
}

// int8 code (byte i of v, two's complement) -> fp32, exact.
__device__ __forceinline__ float q8_byte_f32(uint32_t v, int i) {
    // offset-binary byte (q + 128) in 0..255, then remove 2^23 + 128 exactly
    const uint32_t u = ((v ^ 0x80808080u) >> (8 * i)) & 0xFFu;
    return __fsub_rn(__uint_as_float(0x4B000000u | u), 8388736.0f);
}

// Two 32-bit words (8 int8 codes, lowest address first) -> 8 16-bit codes in
// one 16-byte chunk.  Exact in both types: |q| <= 128 needs at most 8
// significant bits.
template <Op16 OP>
__device__ __forceinline__ uint4 q8_words_op(uint32_t a, uint32_t b) {
    return make_uint4(pack2<OP>(q8_byte_f32(a, 0), q8_byte_f32(a, 1)),
                      pack2<OP>(q8_byte_f32(a, 2), q8_byte_f32(a, 3)),
                      pack2<OP>(q8_byte_f32(b, 0), q8_byte_f32(b, 1)),
                      pack2<OP>(q8_byte_f32(b, 2), q8_byte_f32(b, 3)));
}

}  // namespace rtq
