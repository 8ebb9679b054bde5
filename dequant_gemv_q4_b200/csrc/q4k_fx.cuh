// q4k_fx.cuh -- the batch-1 Q4_K arithmetic shared by the GEMV kernels and the
// fused FFN block: activations staged as fixed-point limb planes, integer dot
// products on TMA-filled slots, the fp64 combine and the per-row error bound.
//
// Arithmetic.
//   x, per super-block sb of 256 activations: with e the exponent of the
//   largest |x_k| (2^e <= max < 2^(e+1)) and F = 29 - e (four limbs) or
//   F = 21 - e (three limbs, for blocks whose largest |x| is at most 6 times
//   their rms), xi_k = round(x_k 2^F), split into signed bytes (signed digits)
//   xi = l0 + 2^8 l1 + 2^16 l2 [+ 2^24 l3].  X_j is the exact sum of xi over
//   sub-block j and R bounds sum_k |x_k - xi_k 2^-F| from above.
//   Per row and sub-block j: A_l = sum_k q_k l_{l,k} (dp4a, exact), folded as
//   I_l += scale_j * A_l (exact; kept as 16 I_l < 2^29 because the high nibbles
//   enter dp4a as 16 q).  Per row and super-block, in fp64: I_s = sum_l 2^(8l)
//   I_l (exact), I_m = sum_j min_j X_j (exact) and y_sb = 2^-F (d I_s - dmin
//   I_m), evaluated with an error-free product so that the rounding is relative
//   to y_sb itself, even when the scale and min terms cancel.  Row sums stay in
//   fp64 and are rounded to fp32 once.
//   So a row's result is sum_k w_k xi_k 2^-F to fp64 accuracy.  Beside it the
//   row carries E (rounded up) = sum_sb (945 d + 63 dmin) R_sb, an upper bound
//   on the error the rounding of x caused (every weight of a super-block has
//   |w| <= 945 d + 63 dmin), and S (rounded down) = sum_sb |y_sb|, a lower bound
//   on sum_k |w_k x_k|; q4k_exact.cuh decides from them whether the row meets
//   |y - y_exact| <= 1e-4 sum |w x| + 1e-6 or must be recomputed exactly.
//   A super-block of x holding an infinity or a NaN makes the rows' results NaN.
//
// Work decomposition ("quarter-warp lanes").  A K-chunk is 4 super-blocks (one
// SoA group, 576 contiguous bytes of a row in both layouts).  Lane (g, i) =
// (lane / 8, lane % 8) handles super-block g of each chunk for rows i + 8r
// (r < R) of a row tile of 8R rows, so the eight lanes of a quarter-warp read
// the same activation bytes (a shared-memory broadcast) and distinct rows'
// quants.  A slot is one chunk of one tile, 8R rows x 576 bytes (at a 592-byte
// pitch, which places the eight rows a quarter-warp reads at one time in eight
// distinct bank groups); the four quarter sums of a row are added with two
// shuffles.
//   Warp pairs (R = 1).  When each warp would own only a few slots, the time a
// warp takes to work through them one after another, not the memory, bounds a
// small matrix.  Then two warps own each ring and its row tiles: warp h of the
// pair takes rows 8h .. 8h + 7 of every slot (lane (g, i): super-block g, row
// 8h + i), so a slot's arithmetic is done by twice the warps in half the time.
// The second warp of the pair to finish a slot refills it.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "q4k_stream.cuh"

namespace dq {

// Staged activations of one super-block: four limb planes of 256 bytes (plane
// l, byte k = limb l of xi_k) and 16 bytes of padding, which shifts the bank
// group from one super-block to the next; then, in a separate array of
// 80-byte records (FxAux), the sums X_j, 2^-F and the rounding residue R.
// The lanes of a quarter-warp read the same super-block, so these reads are
// broadcasts.
constexpr int kFxLimbPitch = 1040;
// Rows shorter than this many super-blocks always take four limbs.
constexpr int kFxMin3LimbBlocks = 16;

// Per staged super-block: X_j = sum of xi over sub-block j (exact); 2^-F (NaN
// when the block holds an infinity or a NaN); R >= sum_k |x_k - xi_k 2^-F|
// (fp32, rounded up): with |w_k| <= 945 d + 63 dmin for every weight of a
// super-block, R bounds the error the rounding of x causes in a row.
//
// Limbs.  In rows of at least 16 super-blocks, a block whose largest |x| is
// at most 6 times its rms is rounded to a 22-bit fixed point (three limbs, one
// dp4a fewer per four weights): a row's error bound then stays near 2e-5 of
// the sum of its blocks' |partial sums|, and with 16 or more blocks that sum
// is practically never small enough for the bound to fail the contract.
// Other blocks take the 30-bit fixed point (four limbs).
struct __align__(16) FxAux {
    double X[8];
    double s2f;
    float R;
    int nl;       // limbs of xi: 3 (22-bit fixed point) or 4 (30-bit)
};
static_assert(sizeof(FxAux) == 80, "one 80-byte record per super-block");
constexpr int kFxAuxPitch = sizeof(FxAux);

constexpr int kFxRows = 2;                     // rows per lane (R)
constexpr int kFxBPC = 4;                      // super-blocks per K-chunk
constexpr int kFxChunkBytes = kFxBPC * kQ4KBlockBytes;   // 576
constexpr int kFxTileRows = 8 * kFxRows;
constexpr int kFxRowPitch = kFxChunkBytes + 16;           // 592
constexpr int kFxSlotBytes = kFxTileRows * kFxRowPitch;
static_assert(kFxSlotBytes % 128 == 0, "slots must keep the ring 128-byte aligned");
constexpr int kFxMaxWarps = 12;
constexpr int kFxMaxPairWarps = 16;            // R = 1: eight pairs of warps
constexpr int kFxPairMaxSlots = 8;             // R = 1 for rings of at most this many slots
// Ring slots a warp fills before it stages its activations (the rest after).
constexpr int kFxPreIssue = 1;
// In-cluster split reduction: per ring a CTA finishes, stream and source rank,
// the 16 row partials (fp64) and their bounds (two floats).
constexpr int kFxClusterPartBytes = 2 * kFxTileRows * (8 + 8);
constexpr int kFxMaxCluster = 8;

// TMA descriptors of the weight matrices: SwiGLU's gate and up, or one per
// matrix of a grouped GEMV.
struct FxMaps {
    CUtensorMap m[kMaxGroup];
};

// Activations of the first kFxStagePre super-blocks a warp stages, loaded into
// registers before the weight copies are issued, so that these small loads are
// not queued behind the weight stream.
constexpr int kFxStagePre = 2;
struct FxXPre {
    float4 a[kFxStagePre], b[kFxStagePre];
};

// Eight activations of this lane: through the read-only path, or (COHERENT)
// through L2 only, for activations written earlier in the same kernel.
template <bool COHERENT>
__device__ __forceinline__ float4 fx_ld4(const float *p)
{
    if constexpr (COHERENT)
        return __ldcg(reinterpret_cast<const float4 *>(p));
    else
        return __ldg(reinterpret_cast<const float4 *>(p));
}

template <bool COHERENT = false>
__device__ __forceinline__ void fx_stage_load(const float *x, int kb_begin, int nbs, int warp, int nwarps, int lane,
                                              FxXPre &pre)
{
#pragma unroll
    for (int k = 0; k < kFxStagePre; ++k) {
        const int sb = warp + k * nwarps;
        if (sb < nbs) {
            const float *xg = x + static_cast<long long>(kb_begin + sb) * 256 + lane * 8;
            pre.a[k] = fx_ld4<COHERENT>(xg);
            pre.b[k] = fx_ld4<COHERENT>(xg + 4);
        }
    }
}

// Converts the activations of NB super-blocks sb[k] (this lane's eight of each:
// a[k], b[k]) into limb planes and FxAux records; one warp per super-block, NB
// of them at once so that their dependency chains interleave.  Block k is
// stored only when valid[k].
template <int NB>
__device__ __forceinline__ void fx_stage_blocks(const int (&sb)[NB], const float4 (&a)[NB], const float4 (&b)[NB],
                                                const bool (&valid)[NB], uint8_t *limbs, uint8_t *aux, int lane,
                                                bool allow3)
{
    float v[NB][8];
    uint32_t m[NB];
#pragma unroll
    for (int k = 0; k < NB; ++k) {
        v[k][0] = a[k].x; v[k][1] = a[k].y; v[k][2] = a[k].z; v[k][3] = a[k].w;
        v[k][4] = b[k].x; v[k][5] = b[k].y; v[k][6] = b[k].z; v[k][7] = b[k].w;
        m[k] = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m[k] = max(m[k], __float_as_uint(v[k][i]) & 0x7FFFFFFFu);
    }
#pragma unroll
    for (int k = 0; k < NB; ++k)
        m[k] = __reduce_max_sync(0xffffffffu, m[k]);   // |x| bit patterns order like the values
    int e[NB];
    bool finite[NB];
    float sq[NB];
#pragma unroll
    for (int k = 0; k < NB; ++k) {
        finite[k] = m[k] < 0x7F800000u;
        e[k] = 0;
        if (m[k] >= 0x00800000u)
            e[k] = static_cast<int>(m[k] >> 23) - 127;
        else if (m[k] != 0)
            e[k] = (31 - __clz(static_cast<int>(m[k]))) - 149;
        // the limb-count test on x 2^-e (largest |value| in [1, 2), squares
        // below 4, no overflow); blocks of extreme exponent take four limbs
        const float sc = (e[k] >= -100 && e[k] <= 100) ? __int_as_float((127 - e[k]) << 23) : 0.f;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            s0 = fmaf(v[k][i] * sc, v[k][i] * sc, s0);
            s1 = fmaf(v[k][i + 1] * sc, v[k][i + 1] * sc, s1);
        }
        sq[k] = s0 + s1;
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
#pragma unroll
        for (int k = 0; k < NB; ++k)
            sq[k] += __shfl_xor_sync(0xffffffffu, sq[k], o);

    uint32_t w[NB][4][2];
    double part[NB];
    float res[NB];   // sum of |x_k 2^F - xi_k| over this lane's elements
    bool three[NB];
    int F[NB];
#pragma unroll
    for (int k = 0; k < NB; ++k) {
        // three limbs when max |x| <= 6 rms, i.e. 256 max^2 <= 36 sum x^2 (taken
        // with a 2^-10 margin: the fp32 sum is not exact)
        const float mxs = (e[k] >= -100 && e[k] <= 100) ? __uint_as_float(m[k]) * __int_as_float((127 - e[k]) << 23)
                                                         : 0.f;
        three[k] = allow3 && finite[k] && e[k] >= -100 && e[k] <= 100 &&
                   256.f * mxs * mxs <= 36.f * sq[k] * (1.f - 0x1p-10f);
        // |x 2^F| < 2^(30 - 8 (4 - limbs)): the top signed digit stays within +-64
        F[k] = (three[k] ? 21 : 29) - e[k];   // in [-106, 178]
        const int F1 = F[k] / 2, F2 = F[k] - F1;   // each in [-53, 89]: normal powers of two
        const float p1 = __int_as_float((127 + F1) << 23);
        const float p2 = __int_as_float((127 + F2) << 23);
        float d[8];
        double pi[8];
#pragma unroll
        for (int l = 0; l < 4; ++l)
            w[k][l][0] = w[k][l][1] = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            // x * 2^F is exact wherever it is >= 1/2 in magnitude (two power-of-two
            // products with normal results), and then so is t - rint(t); below 1/2 it
            // rounds to 0, and the first product may have lost bits below 2^-150,
            // i.e. below 2^-61 after the second: 2^-60 covers that
            const float t = finite[k] ? (v[k][i] * p1) * p2 : 0.f;
            const float r = rintf(t);
            d[i] = fabsf(t - r) + ((r == 0.f && v[k][i] != 0.f) ? 0x1p-60f : 0.f);
            int ti = static_cast<int>(r);
            pi[i] = static_cast<double>(ti);
            // signed digits: the stored byte is ti's low byte, the carry rounds ti / 256
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                w[k][l][i >> 2] |= (static_cast<uint32_t>(ti) & 0xFFu) << (8 * (i & 3));
                ti = (ti + 128) >> 8;
            }
        }
        // sums as trees: part exact (integers below 2^33), res rounded (the bound
        // below allows for it)
        part[k] = ((pi[0] + pi[1]) + (pi[2] + pi[3])) + ((pi[4] + pi[5]) + (pi[6] + pi[7]));
        res[k] = ((d[0] + d[1]) + (d[2] + d[3])) + ((d[4] + d[5]) + (d[6] + d[7]));
        if (valid[k]) {
            uint8_t *lp = limbs + sb[k] * kFxLimbPitch + lane * 8;
#pragma unroll
            for (int l = 0; l < 4; ++l)
                *reinterpret_cast<uint2 *>(lp + 256 * l) = make_uint2(w[k][l][0], w[k][l][1]);
        }
    }
    // sub-block j = lanes 4j .. 4j+3; sums of at most 32 values below 2^30 are exact
    // (with three limbs the fourth plane is zero)
#pragma unroll
    for (int o = 1; o < 4; o <<= 1)
#pragma unroll
        for (int k = 0; k < NB; ++k)
            part[k] += __shfl_xor_sync(0xffffffffu, part[k], o);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
#pragma unroll
        for (int k = 0; k < NB; ++k)
            res[k] += __shfl_xor_sync(0xffffffffu, res[k], o);
#pragma unroll
    for (int k = 0; k < NB; ++k) {
        if (!valid[k])
            continue;
        FxAux *ap = reinterpret_cast<FxAux *>(aux + sb[k] * kFxAuxPitch);
        if ((lane & 3) == 0)
            ap->X[lane >> 2] = part[k];
        if (lane == 0) {
            const double s2f = __longlong_as_double(static_cast<long long>(1023 - F[k]) << 52);
            ap->s2f = finite[k] ? s2f : __longlong_as_double(0x7FF8000000000000LL);
            // the fp32 sum of 256 terms (a tree eight deep) is within 2^-20 of
            // the exact one: 2^-16 more keeps R an upper bound
            ap->R = finite[k] ? __double2float_ru(static_cast<double>(res[k]) * (1.0 + 0x1p-16) * s2f) : 0.f;
            ap->nl = three[k] ? 3 : 4;
        }
    }
}

// Stages super-blocks kb_begin .. kb_begin + nbs - 1: this warp's first
// kFxStagePre (= 2, together) from the registers fx_stage_load filled, the
// rest loaded here.
template <bool COHERENT = false>
__device__ __forceinline__ void fx_stage(const float *x, int kb_begin, int nbs, uint8_t *limbs, uint8_t *aux,
                                         int warp, int nwarps, int lane, const FxXPre &pre, bool allow3)
{
    static_assert(kFxStagePre == 2, "the preloaded blocks are staged as a pair");
    if (warp < nbs) {
        const int sb[2] = {warp, warp + nwarps};
        const bool valid[2] = {true, warp + nwarps < nbs};
        if (valid[1]) {
            fx_stage_blocks<2>(sb, pre.a, pre.b, valid, limbs, aux, lane, allow3);
        } else {
            const int sb1[1] = {warp};
            const float4 a1[1] = {pre.a[0]}, b1[1] = {pre.b[0]};
            const bool v1[1] = {true};
            fx_stage_blocks<1>(sb1, a1, b1, v1, limbs, aux, lane, allow3);
        }
    }
    for (int s = warp + kFxStagePre * nwarps; s < nbs; s += nwarps) {
        const float *xg = x + static_cast<long long>(kb_begin + s) * 256 + lane * 8;
        const int sb1[1] = {s};
        const float4 a1[1] = {fx_ld4<COHERENT>(xg)}, b1[1] = {fx_ld4<COHERENT>(xg + 4)};
        const bool v1[1] = {true};
        fx_stage_blocks<1>(sb1, a1, b1, v1, limbs, aux, lane, allow3);
    }
}

// dp4a with unsigned bytes in a (quants) and signed bytes in b (activation limbs).
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// One 16-byte quant slice of R rows against the limb planes: lo (low nibbles,
// sub-block 2c) and hi (high nibbles, sub-block 2c+1) sums per limb.  The high
// nibbles are used in place, as the bytes 16*q (one AND), so the hi sums are
// 16 times the sub-block sums.
template <int R, int NL>
__device__ __forceinline__ void fx_slice(const uint4 (&q)[R], const uint8_t *xlo, const uint8_t *xhi, int (&alo)[R][4],
                                         int (&ahi)[R][4])
{
    uint4 xa[NL], xb[NL];
#pragma unroll
    for (int l = 0; l < NL; ++l) {
        xa[l] = *reinterpret_cast<const uint4 *>(xlo + 256 * l);
        xb[l] = *reinterpret_cast<const uint4 *>(xhi + 256 * l);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint32_t w = (t == 0) ? q[r].x : (t == 1) ? q[r].y : (t == 2) ? q[r].z : q[r].w;
            const uint32_t lo = w & 0x0F0F0F0Fu;
            const uint32_t hi16 = w & 0xF0F0F0F0u;
#pragma unroll
            for (int l = 0; l < NL; ++l) {
                const uint32_t x0 = (t == 0) ? xa[l].x : (t == 1) ? xa[l].y : (t == 2) ? xa[l].z : xa[l].w;
                const uint32_t x1 = (t == 0) ? xb[l].x : (t == 1) ? xb[l].y : (t == 2) ? xb[l].z : xb[l].w;
                alo[r][l] = dp4a_us(lo, x0, alo[r][l]);
                ahi[r][l] = dp4a_us(hi16, x1, ahi[r][l]);
            }
        }
    }
}

// Integer sums of this lane's super-block of a slot for its R rows (row r at
// slot_row + 8 r pitches): isum[r][l] = 16 sum_j scale_j sum_{k in j} q_k limb_l(xi_k)
// for l < NL (exact; |isum| < 2^29); isum[r][NL..3] are left as they are.
template <int R, int NL>
__device__ __forceinline__ void fx_block_sums(const uint8_t *slot_row, BlockOffsets bo, const uint32_t (&sc03)[R],
                                              const uint32_t (&sc47)[R], const uint8_t *xb, int (&isum)[R][4])
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        int alo[R][4], ahi[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                alo[r][k] = 0;
                ahi[r][k] = 0;
            }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int s = 2 * c + h;  // 16-byte quant slice
            uint4 q[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                q[r] = *reinterpret_cast<const uint4 *>(slot_row + 8 * r * kFxRowPitch + bo.qs0 + s * bo.qs_step);
            fx_slice<R, NL>(q, xb + 64 * c + 16 * h, xb + 64 * c + 32 + 16 * h, alo, ahi);
        }
        // fold the scales of sub-blocks 2c (lo) and 2c+1 (hi); the sums are
        // kept 16 times larger (the hi sums already are): |16 I_l| < 2^29
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint32_t sw = (c < 2) ? sc03[r] : sc47[r];
            const int slo16 = static_cast<int>((sw >> (16 * (c & 1))) & 0xFFu) << 4;
            const int shi = static_cast<int>((sw >> (16 * (c & 1) + 8)) & 0xFFu);
#pragma unroll
            for (int k = 0; k < NL; ++k)
                isum[r][k] += slo16 * alo[r][k] + shi * ahi[r][k];
        }
    }
}

// One slot (a K-chunk of kFxBPC super-blocks of one row tile) for this lane:
// super-block g of the chunk, slot rows i + 8r (r < R).  slot is the slot's
// shared memory, limbs/aux point at the staged activations of the chunk's first
// super-block, nblk is the chunk's super-block count.  Adds each row's partial
// y_sb = 2^-F (d I_s - dmin I_m) (fp64), its error bound and |y_sb|.
// All 32 lanes must call it (the limb count is agreed across the warp).
template <int R, bool SOA>
__device__ __forceinline__ void fx_slot(const uint8_t *slot, const uint8_t *limbs, const uint8_t *aux, int nblk, int g,
                                        int i, double (&acc)[R], float (&ebound)[R], float (&sabs)[R])
{
    // this quarter-warp's block: 2^-F, rounding residue and limb count in one
    // 16-byte load; the chunk takes four limbs if any of its blocks needs them
    const FxAux *ap = reinterpret_cast<const FxAux *>(aux + min(g, nblk - 1) * kFxAuxPitch);
    const uint4 sn = *reinterpret_cast<const uint4 *>(&ap->s2f);
    const bool l4 = __any_sync(0xffffffffu, g < nblk && static_cast<int>(sn.w) == 4);
    if (g >= nblk)
        return;
    const uint8_t *slot_p = slot + i * kFxRowPitch;
    const BlockOffsets bo = block_offsets<SOA>(g, nblk);
    uint4 hd[R];
    uint32_t sc03[R], sc47[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        hd[r] = *reinterpret_cast<const uint4 *>(slot_p + 8 * r * kFxRowPitch + bo.hdr);
        // GGML get_scale_min_k4 packing: scales 0..3 are the low six bits of
        // bytes 0..3; scales 4..7 take their low four bits from the low nibbles
        // of bytes 8..11 and their top two bits from bits 6..7 of bytes 0..3
        sc03[r] = hd[r].y & 0x3F3F3F3Fu;
        sc47[r] = (hd[r].w & 0x0F0F0F0Fu) | ((hd[r].y >> 2) & 0x30303030u);
    }
    const uint8_t *xb = limbs + g * kFxLimbPitch;

    int isum[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int k = 0; k < 4; ++k)
            isum[r][k] = 0;
    if (l4)
        fx_block_sums<R, 4>(slot_p, bo, sc03, sc47, xb, isum);
    else
        fx_block_sums<R, 3>(slot_p, bo, sc03, sc47, xb, isum);

    // per row: y_sb = 2^-F (d I_s - dmin I_m) in fp64
    double X[8];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        const double2 t = *reinterpret_cast<const double2 *>(ap->X + j);
        X[j] = t.x;
        X[j + 1] = t.y;
    }
    const double s2f = __hiloint2double(static_cast<int>(sn.y), static_cast<int>(sn.x));
    const float rres = __uint_as_float(sn.z);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        // I_s = sum_l 2^(8l) I_l: exact in int64 (below 2^53), then one conversion
        const long long is64 =
            ((static_cast<long long>(isum[r][3]) << 24) + (static_cast<long long>(isum[r][2]) << 16)) +
            ((static_cast<long long>(isum[r][1]) << 8) + static_cast<long long>(isum[r][0]));
        const double is = static_cast<double>(is64);
        const uint32_t mn03 = hd[r].z & 0x3F3F3F3Fu;
        const uint32_t mn47 = ((hd[r].w >> 4) & 0x0F0F0F0Fu) | ((hd[r].z >> 2) & 0x30303030u);
        // I_m as a tree of exact products and sums (integers below 2^53)
        double pmn[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t mw = (j < 4) ? mn03 : mn47;
            // min_j as a double without a conversion: the bits of 2^52 + m, minus 2^52 (exact)
            const double mj = __hiloint2double(0x43300000, static_cast<int>((mw >> (8 * (j & 3))) & 0xFFu)) - 0x1p52;
            pmn[j] = mj * X[j];
        }
        const double im = ((pmn[0] + pmn[1]) + (pmn[2] + pmn[3])) + ((pmn[4] + pmn[5]) + (pmn[6] + pmn[7]));
        const float df = __half2float(__ushort_as_half(static_cast<unsigned short>(hd[r].x & 0xFFFFu)));
        const float dmf = __half2float(__ushort_as_half(static_cast<unsigned short>(hd[r].x >> 16)));
        // the 1/16 undoes the scaling of the integer sums (exact)
        const double d = static_cast<double>(df) * (s2f * 0.0625);
        const double dm = static_cast<double>(dmf) * s2f;
        const double pm = dm * im;            // rounded
        const double em = fma(dm, im, -pm);   // its exact rounding error
        const double ysb = fma(d, is, -pm) - em;
        acc[r] += ysb;
        // error bound (every |w| <= 945 d + 63 dmin) and sum_k |w x| >= |y_sb|
        ebound[r] = __fmaf_ru(__fmaf_ru(63.f, dmf, 945.f * df), rres, ebound[r]);
        sabs[r] = __fadd_rd(sabs[r], __double2float_rd(fabs(ysb)));
    }
}

// Adds the four quarter-warps' row sums (and their bounds, rounded outwards).
// R = 2: afterwards lanes of quarters 0, 1 hold row i and quarters 2, 3 row
// i + 8.  R = 1: every quarter holds the sums of its lanes' row.
template <int R>
__device__ __forceinline__ void fx_quarter_rows(double (&acc)[R], float (&ebound)[R], float (&sabs)[R], int lane,
                                                double &t, float &te, float &ts)
{
    if constexpr (R == 2) {
        const bool up = (lane & 16) != 0;
        t = (up ? acc[1] : acc[0]) + __shfl_xor_sync(0xffffffffu, up ? acc[0] : acc[1], 16);
        te = __fadd_ru(up ? ebound[1] : ebound[0], __shfl_xor_sync(0xffffffffu, up ? ebound[0] : ebound[1], 16));
        ts = __fadd_rd(up ? sabs[1] : sabs[0], __shfl_xor_sync(0xffffffffu, up ? sabs[0] : sabs[1], 16));
    } else {
        t = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 16);
        te = __fadd_ru(ebound[0], __shfl_xor_sync(0xffffffffu, ebound[0], 16));
        ts = __fadd_rd(sabs[0], __shfl_xor_sync(0xffffffffu, sabs[0], 16));
    }
    t += __shfl_xor_sync(0xffffffffu, t, 8);
    te = __fadd_ru(te, __shfl_xor_sync(0xffffffffu, te, 8));
    ts = __fadd_rd(ts, __shfl_xor_sync(0xffffffffu, ts, 8));
#pragma unroll
    for (int r = 0; r < R; ++r) {
        acc[r] = 0.0;
        ebound[r] = 0.f;
        sabs[r] = 0.f;
    }
}

}  // namespace dq
