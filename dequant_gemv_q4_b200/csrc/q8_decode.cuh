// q8_decode.cuh -- Q8_0 block decoding shared by the GEMV and the debug
// dequant kernel.
//
// Format (GGML-style Q8_0, 34 bytes / 32 weights, little-endian): d (fp16)
// followed by 32 two's-complement int8 quants; weight i = d * q_i.
//
// Weight formation: u = q + 128 (the quant byte with its top bit flipped) is
// an unsigned byte; isolated at bit position p of a 32-bit word its bit
// pattern is the fp32 value u * 2^(p-149) (below 2^24 a bit pattern's value is
// pattern * 2^-149).  fma(u*2^(p-149), d*2^(85-p), -128*d*2^-64) is exactly
// q*d*2^-64: the result has at most 8+11 significant bits, so no rounding
// happens at all.
#pragma once

#include <cstdint>

namespace dq {

// Scale pairs for the byte positions 0/8 (bytes 0, 1 of a word) and 16/16
// (bytes 2 and 3, the latter shifted down by 8 bits), and the offset pair.
__device__ __forceinline__ void q8_scales(float d, float2 &s01, float2 &s23, float2 &off)
{
    s01 = make_float2(d * 0x1p85f, d * 0x1p77f);
    s23 = make_float2(d * 0x1p69f, d * 0x1p69f);
    const float o = -128.0f * d * 0x1p-64f;
    off = make_float2(o, o);
}

// Four weights of one quant word (bytes 0..3 = weights 4j .. 4j+3), times
// 2^-64: wv[0] = weights 4j, 4j+1; wv[1] = weights 4j+2, 4j+3.
__device__ __forceinline__ void q8_word_weights(uint32_t wq, float2 s01, float2 s23, float2 off, float2 wv[2])
{
    const uint32_t u = wq ^ 0x80808080u;
    const uint32_t v = u >> 8;
    wv[0] = __ffma2_rn(make_float2(__uint_as_float(u & 0xFFu), __uint_as_float(u & 0xFF00u)), s01, off);
    wv[1] = __ffma2_rn(make_float2(__uint_as_float(u & 0xFF0000u), __uint_as_float(v & 0xFF0000u)), s23, off);
}

}  // namespace dq
