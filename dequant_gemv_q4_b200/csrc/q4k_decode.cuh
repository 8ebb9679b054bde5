// q4k_decode.cuh -- Q4_K super-block decoding shared by the GEMV and the
// debug-dequant kernels, so that the dequant entry point checks exactly the
// weight values the GEMV forms.
//
// Format (GGML-style Q4_K, 144 bytes / 256 weights, little-endian):
//   bytes 0..1 d (fp16), 2..3 dmin (fp16), 4..15 scale bytes, 16..143 quants.
//   weight i = d * scale_j * q_i - dmin * min_j, j = i / 32; quant byte
//   32c + r (r < 32) holds weight 64c + r in its low nibble and 64c + 32 + r
//   in its high nibble, so one byte carries one weight of sub-block 2c ("lo")
//   and one of sub-block 2c+1 ("hi").
//
// Weight formation.  A quant q isolated at bit position p of a 32-bit word is
// the fp32 bit pattern of q * 2^(p-149): a subnormal, or a value in the
// smallest normal binade, where a bit pattern below 2^24 still means
// pattern * 2^-149.  fma(q*2^(p-149), d*scale*2^(85-p), -dmin*min*2^-64) is
// then exactly (d*scale*q - dmin*min) * 2^-64 rounded once to fp32: every
// operand is exact (d: 11 significant bits, scale and min: 6, q: 4) and the fma
// rounds once.  Weights are formed in pairs {lo, hi} of one byte with
// fma.rn.f32x2.
//
// Scales are turned into floats without an integer-to-float conversion: a
// byte v placed under the exponent byte 0x4B reads as 2^23 + v, and
// fma(2^23 + v, D, -2^23 * D) = v * D exactly (v * D has at most 6 + 11
// significant bits).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace dq {

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

constexpr uint32_t kMagic23 = 0x4B000000u;  // fp32 bits of 2^23

// Decoded header of one super-block of one row.  A word's quant pairs sit at
// bit positions (0, 4) and (8, 12) -- bytes 0 and 1 directly, bytes 2 and 3
// after a 16-bit shift -- so two scale-factor pairs cover all of them:
// D0 = {d*2^85, d*2^81}, D1 = {d*2^77, d*2^73}, with N0/N1 = -2^23 * D0/D1;
// DN = {-dmin*2^-64, -dmin*2^-64} and NN = -2^23 * DN for the mins.
struct Hdr {
    float2 D0, D1, N0, N1, DN, NN;
    uint32_t sc03, mn03, sc47, mn47;   // four six-bit values per word, one per byte
};

__device__ __forceinline__ Hdr decode_hdr(uint4 h)
{
    Hdr r;
    const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x & 0xFFFFu)));
    const float dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x >> 16)));
    r.D0 = f2(d * 0x1p85f, d * 0x1p81f);
    r.D1 = f2(d * 0x1p77f, d * 0x1p73f);
    r.N0 = f2(d * -0x1p108f, d * -0x1p104f);
    r.N1 = f2(d * -0x1p100f, d * -0x1p96f);
    const float ndm = dmin * -0x1p-64f;
    r.DN = f2(ndm, ndm);
    const float nnm = dmin * 0x1p-41f;   // -2^23 * ndm
    r.NN = f2(nnm, nnm);
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

// Scale pairs of chunk c (sub-blocks 2c = lo, 2c+1 = hi):
// S0 = {d*sc_lo*2^85, d*sc_hi*2^81}, S1 = S0 * 2^-8, M = {-dmin*min_lo, -dmin*min_hi}*2^-64.
struct ChunkScales {
    float2 S0, S1, M;
};

// Scale pairs of the sub-block pair held in bytes k, k+1 of the scale word scw
// and min word mnw.
__device__ __forceinline__ ChunkScales scales_from_words(const Hdr &h, uint32_t scw, uint32_t mnw, uint32_t k)
{
    // {2^23 + scale_lo, 2^23 + scale_hi} and the same for the mins
    const float2 fs = f2(__uint_as_float(__byte_perm(scw, kMagic23, 0x7540u + k)),
                         __uint_as_float(__byte_perm(scw, kMagic23, 0x7541u + k)));
    const float2 fm = f2(__uint_as_float(__byte_perm(mnw, kMagic23, 0x7540u + k)),
                         __uint_as_float(__byte_perm(mnw, kMagic23, 0x7541u + k)));
    ChunkScales s;
    s.S0 = __ffma2_rn(fs, h.D0, h.N0);
    s.S1 = __ffma2_rn(fs, h.D1, h.N1);
    s.M = __ffma2_rn(fm, h.DN, h.NN);
    return s;
}

__device__ __forceinline__ ChunkScales chunk_scales(const Hdr &h, int c)
{
    // sub-blocks 2c, 2c+1 sit in bytes 2(c%2), 2(c%2)+1 of the 0..3 or 4..7 words
    return scales_from_words(h, (c < 2) ? h.sc03 : h.sc47, (c < 2) ? h.mn03 : h.mn47, (c & 1) * 2);
}

// The eight weights of one quant word, times 2^-64: wv[k] = {lo, hi} weights of
// byte k of the word.
__device__ __forceinline__ void q4_word_weights(uint32_t w, const ChunkScales &s, float2 wv[4])
{
    const uint32_t u = w >> 16;
    wv[0] = __ffma2_rn(f2(__uint_as_float(w & 0xFu), __uint_as_float(w & 0xF0u)), s.S0, s.M);
    wv[1] = __ffma2_rn(f2(__uint_as_float(w & 0xF00u), __uint_as_float(w & 0xF000u)), s.S1, s.M);
    wv[2] = __ffma2_rn(f2(__uint_as_float(u & 0xFu), __uint_as_float(u & 0xF0u)), s.S0, s.M);
    wv[3] = __ffma2_rn(f2(__uint_as_float(u & 0xF00u), __uint_as_float(u & 0xF000u)), s.S1, s.M);
}

// One quant word (bytes 4t..4t+3 of a 16-byte slice): form its eight weights
// and accumulate weight*x.  xa = {x[L+4t], x[H+4t], x[L+4t+1], x[H+4t+1]},
// xb = the same for bytes 4t+2, 4t+3 (x is staged in (lo, hi) pairs).
__device__ __forceinline__ void q4_word(uint32_t w, const ChunkScales &cs, float4 xa, float4 xb, float2 &acc0,
                                        float2 &acc1)
{
    float2 wv[4];
    q4_word_weights(w, cs, wv);
    acc0 = __ffma2_rn(wv[0], f2(xa.x, xa.y), acc0);
    acc1 = __ffma2_rn(wv[1], f2(xa.z, xa.w), acc1);
    acc0 = __ffma2_rn(wv[2], f2(xb.x, xb.y), acc0);
    acc1 = __ffma2_rn(wv[3], f2(xb.z, xb.w), acc1);
}

// x of one super-block is staged (fp32) as 8 slices x 8 float4, float4 k of
// slice s = 2c+h holding {x[L+2k], x[H+2k], x[L+2k+1], x[H+2k+1]} (L = 64c+16h,
// H = L+32): the (lo, hi) weight pairs of quant bytes 2k and 2k+1.  16 bytes of
// padding per super-block.
constexpr int kXBlockPitch = 1040;

// Stages activations of super-blocks kb_begin .. kb_begin + nbs - 1 of B rows of
// x (row b at x + b*K) in that layout, super-block kbl of row b at
// xs + (b*nbs + kbl)*kXBlockPitch; each thread keeps kBatch loads in flight.
template <int kBatch>
__device__ __forceinline__ void stage_x_pairs(const float *x, int K, int B, int kb_begin, int nbs, uint8_t *xs)
{
    const int per_b = nbs * 64;  // float4 per batch row
    const int n_out = B * per_b;
    for (int base = threadIdx.x; base < n_out; base += kBatch * blockDim.x) {
        float2 lo[kBatch], hi[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int idx = base + u * blockDim.x;
            if (idx < n_out) {
                const int b = idx / per_b;
                const int rem = idx - b * per_b;
                const int kbl = rem >> 6;
                const int sl = (rem >> 3) & 7;    // slice
                const int k = rem & 7;            // float4 within the slice
                const float *xb = x + static_cast<long long>(b) * K + static_cast<long long>(kb_begin + kbl) * 256 +
                                  64 * (sl >> 1) + 16 * (sl & 1) + 2 * k;
                lo[u] = __ldg(reinterpret_cast<const float2 *>(xb));
                hi[u] = __ldg(reinterpret_cast<const float2 *>(xb + 32));
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int idx = base + u * blockDim.x;
            if (idx < n_out) {
                const int b = idx / per_b;
                const int rem = idx - b * per_b;
                *reinterpret_cast<float4 *>(xs + (b * nbs + (rem >> 6)) * kXBlockPitch + ((rem >> 3) & 7) * 128 +
                                            (rem & 7) * 16) = make_float4(lo[u].x, hi[u].x, lo[u].y, hi[u].y);
            }
        }
    }
}

}  // namespace dq
