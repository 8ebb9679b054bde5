// q4k_decode.cuh -- Q4_K super-block decoding shared by the GEMV and the
// debug-dequant kernels, so that the dequant entry point checks exactly the
// weight values the GEMV forms.
//
// Format (GGML-style Q4_K, 144 bytes / 256 weights, little-endian):
//   bytes 0..1 d (fp16), 2..3 dmin (fp16), 4..15 scale bytes, 16..143 quants.
//   weight i = d * scale_j * q_i - dmin * min_j, j = i / 32; quant byte
//   32c + r (r < 32) holds weight 64c + r in its low nibble and 64c + 32 + r
//   in its high nibble.
//
// Weight formation: a quant q isolated at bit position p of a 32-bit word is
// the fp32 bit pattern of q * 2^(p-149) (subnormal, or the smallest normal
// binade, where the value of a bit pattern below 2^24 is still pattern*2^-149).
// fma(q*2^(p-149), d*scale*2^(85-p), -dmin*min*2^-64) is then exactly
// (d*scale*q - dmin*min) * 2^-64 rounded once to fp32: every operand is exact
// (d: 11 significant bits, scale/min: 6, q: 4) and the fma rounds once.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#ifndef DQ_PAIR64
#define DQ_PAIR64 0
#endif

namespace dq {

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Eight quants of one 32-bit word of a 16-byte quant slice (see the file
// comment): bytes 0..3 of the word hold weights L+4t .. L+4t+3 in their low
// nibbles and H+4t .. H+4t+3 in their high nibbles (H = L + 32).
//   sL = {d*sc_lo*2^85, d*sc_lo*2^77}, sH = {d*sc_hi*2^81, d*sc_hi*2^73}
//   mL = -dmin*min_lo*2^-64 (both lanes), mH likewise.

// Decoded header of one super-block of one row.
struct Hdr {
    float2 dA;   // {d*2^85, d*2^77}
    float2 dB;   // {d*2^81, d*2^73}
    float ndm;   // -dmin*2^-64
    uint32_t sc03, mn03, sc47, mn47;   // four six-bit values per word, one per byte
};

__device__ __forceinline__ Hdr decode_hdr(uint4 h)
{
    Hdr r;
    const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x & 0xFFFFu)));
    const float dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x >> 16)));
    r.dA = f2(d * 0x1p85f, d * 0x1p77f);
    r.dB = f2(d * 0x1p81f, d * 0x1p73f);
    r.ndm = -dmin * 0x1p-64f;
    // GGML get_scale_min_k4 packing: scales/mins 0..3 are the low six bits of
    // bytes 0..3 / 4..7; 4..7 take their low four bits from bytes 8..11 (low
    // nibble for scales, high nibble for mins) and their top two bits from
    // bits 6..7 of bytes 0..3 (scales) / 4..7 (mins).
    r.sc03 = h.y & 0x3F3F3F3Fu;
    r.mn03 = h.z & 0x3F3F3F3Fu;
    r.sc47 = (h.w & 0x0F0F0F0Fu) | ((h.y >> 2) & 0x30303030u);
    r.mn47 = ((h.w >> 4) & 0x0F0F0F0Fu) | ((h.z >> 2) & 0x30303030u);
    return r;
}

// Per-chunk scale pairs for chunk c (sub-blocks 2c, 2c+1).
__device__ __forceinline__ void chunk_scales(const Hdr &h, int c, float2 &sL, float2 &mL, float2 &sH,
                                             float2 &mH)
{
    const uint32_t scw = (c < 2) ? h.sc03 : h.sc47;
    const uint32_t mnw = (c < 2) ? h.mn03 : h.mn47;
    const int sh = (c & 1) * 16;
    const float sclo = static_cast<float>((scw >> sh) & 0xFFu);
    const float schi = static_cast<float>((scw >> (sh + 8)) & 0xFFu);
    const float mnlo = static_cast<float>((mnw >> sh) & 0xFFu);
    const float mnhi = static_cast<float>((mnw >> (sh + 8)) & 0xFFu);
    sL = __fmul2_rn(h.dA, f2(sclo, sclo));
    sH = __fmul2_rn(h.dB, f2(schi, schi));
    mL = f2(h.ndm * mnlo, h.ndm * mnlo);
    mH = f2(h.ndm * mnhi, h.ndm * mnhi);
}


// The eight weights of one quant word, times 2^-64, as four pairs:
//   wv[0] = weights L+4t, L+4t+1   wv[1] = L+4t+2, L+4t+3   (low nibbles)
//   wv[2] = weights H+4t, H+4t+1   wv[3] = H+4t+2, H+4t+3   (high nibbles)
__device__ __forceinline__ void q4_word_weights(uint32_t w, float2 sL, float2 mL, float2 sH, float2 mH,
                                                float2 wv[4])
{
#if DQ_PAIR64
    // each pair isolated with one 64-bit AND of {w, w}, so that its two halves
    // land in one register pair
    const uint32_t u = w >> 16;
    const uint64_t ww = (static_cast<uint64_t>(w) << 32) | w;
    const uint64_t uu = (static_cast<uint64_t>(u) << 32) | u;
    const uint64_t a = ww & 0x00000F000000000Full, b = uu & 0x00000F000000000Full;
    const uint64_t c = ww & 0x0000F000000000F0ull, e = uu & 0x0000F000000000F0ull;
    wv[0] = __ffma2_rn(*reinterpret_cast<const float2 *>(&a), sL, mL);
    wv[1] = __ffma2_rn(*reinterpret_cast<const float2 *>(&b), sL, mL);
    wv[2] = __ffma2_rn(*reinterpret_cast<const float2 *>(&c), sH, mH);
    wv[3] = __ffma2_rn(*reinterpret_cast<const float2 *>(&e), sH, mH);
#else
    const uint32_t u = w >> 16;
    wv[0] = __ffma2_rn(f2(__uint_as_float(w & 0xFu), __uint_as_float(w & 0xF00u)), sL, mL);
    wv[1] = __ffma2_rn(f2(__uint_as_float(u & 0xFu), __uint_as_float(u & 0xF00u)), sL, mL);
    wv[2] = __ffma2_rn(f2(__uint_as_float(w & 0xF0u), __uint_as_float(w & 0xF000u)), sH, mH);
    wv[3] = __ffma2_rn(f2(__uint_as_float(u & 0xF0u), __uint_as_float(u & 0xF000u)), sH, mH);
#endif
}

}  // namespace dq
