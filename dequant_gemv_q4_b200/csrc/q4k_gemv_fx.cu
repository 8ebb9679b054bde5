// q4k_gemv_fx.cu -- batch-1 fused Q4_K dequantize + GEMV (plain, fused SwiGLU,
// optional argmax) with integer dot products on fixed-point activations, for
// sm_100a.
//
// The operation is the pages' fused dequant+GEMV over raw Q4_K bytes (trueno
// WgslForwardPass: upload_q4k_weight; qualiaDB cuda_lane: try_q4k_soa_gemv,
// try_q4k_soa_fused_swiglu).  The arithmetic below is this library's own.
//
// Why integers.  At batch 1 every weight is used once, so the cost per weight
// is what bounds the kernel.  Forming each fp32 weight (an AND to isolate the
// quant, an fma with scale and min) and then an fma with x costs three
// instructions per weight on two half-rate pipes.  Here four quants at a time
// are unpacked into bytes (one AND for the four low nibbles of a word, a shift
// and an AND for the four high nibbles) and multiplied against four bytes of x
// by one dp4a (four 8-bit products summed into an int32).
//
// Arithmetic.
//   x, per super-block sb of 256 activations: with e the exponent of the
//   largest |x_k| (2^e <= max < 2^(e+1)) and F = 29 - e, xi_k = round(x_k 2^F),
//   so |xi_k| < 2^30 and |x_k - xi_k 2^-F| <= 2^(e-30).  xi is split into four
//   signed bytes (signed digits) xi = l0 + 2^8 l1 + 2^16 l2 + 2^24 l3.  X_j is
//   the exact sum of xi over sub-block j.
//   Per row and sub-block j: A_l = sum_k q_k l_{l,k} (dp4a, exact), folded as
//   I_l += scale_j * A_l (exact, |I_l| < 2^25).  Per row and super-block, in
//   fp64: I_s = sum_l 2^(8l) I_l (exact, < 2^49), I_m = sum_j min_j X_j (exact,
//   < 2^44) and y_sb = 2^-F (d I_s - dmin I_m), evaluated with an error-free
//   product so that the rounding is relative to y_sb itself, even when the
//   scale and min terms cancel.  Row sums stay in fp64 and are rounded to fp32
//   once.
//   So the result is sum_k w_k xi_k 2^-F to fp64 accuracy; the only
//   approximation is the rounding of x:
//     |y - sum_k w_k x_k| <= sum_sb 2^(e_sb - 30) sum_{k in sb} |w_k|,
//   i.e. 2^-30 of the largest activation of each super-block.
//   A super-block of x holding an infinity or a NaN makes the rows' results NaN.
//
// Work decomposition: the full-block lanes of the fp32 kernel (lane l of a row
// group owns super-block l of each K-chunk, two rows per lane) and its
// per-warp bulk-copy rings; only the staging of x and the per-weight
// arithmetic differ.

#include <cuda_fp16.h>
#include <cstdint>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "q4k_stream.cuh"

namespace dq {

// Staged activations of one super-block: four limb planes of 256 bytes (plane
// l, byte k = limb l of xi_k), 16 bytes of padding so that the lanes of one
// shared-memory phase (eight consecutive super-blocks) hit distinct bank
// groups; then, in a separate array, X_0..X_7 and 2^-F as fp64 (80-byte pitch,
// again a distinct bank group per super-block).
constexpr int kFxLimbPitch = 1040;
constexpr int kFxAuxPitch = 80;

int q4k_fx_stage_bytes_per_block() { return kFxLimbPitch + kFxAuxPitch; }

// Converts the activations of super-blocks kb_begin .. kb_begin + nbs - 1 into
// limb planes and sums; one warp per super-block.
__device__ __forceinline__ void fx_stage(const float *x, int kb_begin, int nbs, uint8_t *limbs, uint8_t *aux,
                                         int warp, int nwarps, int lane)
{
    for (int sb = warp; sb < nbs; sb += nwarps) {
        const float *xg = x + static_cast<long long>(kb_begin + sb) * 256 + lane * 8;
        const float4 a = __ldg(reinterpret_cast<const float4 *>(xg));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(xg + 4));
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
        m = __reduce_max_sync(0xffffffffu, m);   // |x| bit patterns order like the values
        const bool finite = m < 0x7F800000u;
        int e = 0;
        if (m >= 0x00800000u)
            e = static_cast<int>(m >> 23) - 127;
        else if (m != 0)
            e = (31 - __clz(static_cast<int>(m))) - 149;
        const int F = 29 - e;                  // in [-98, 178]
        const int F1 = F / 2, F2 = F - F1;     // each in [-49, 89]: normal powers of two
        const float p1 = __int_as_float((127 + F1) << 23);
        const float p2 = __int_as_float((127 + F2) << 23);

        uint32_t w[4][2] = {};
        double part = 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            // x * 2^F is exact wherever it is >= 1/2 in magnitude (two power-of-two
            // products with normal results); smaller values round to 0 either way
            int t = finite ? __float2int_rn((v[i] * p1) * p2) : 0;
            part += static_cast<double>(t);
            // signed digits: the stored byte is t's low byte, the carry rounds t / 256
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                w[l][i >> 2] |= (static_cast<uint32_t>(t) & 0xFFu) << (8 * (i & 3));
                t = (t + 128) >> 8;
            }
        }
        uint8_t *lp = limbs + sb * kFxLimbPitch + lane * 8;
#pragma unroll
        for (int l = 0; l < 4; ++l)
            *reinterpret_cast<uint2 *>(lp + 256 * l) = make_uint2(w[l][0], w[l][1]);
        // sub-block j = lanes 4j .. 4j+3; sums of at most 32 values below 2^30 are exact
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        double *ap = reinterpret_cast<double *>(aux + sb * kFxAuxPitch);
        if ((lane & 3) == 0)
            ap[lane >> 2] = part;
        if (lane == 0)
            ap[8] = finite ? __longlong_as_double(static_cast<long long>(1023 - F) << 52)
                           : __longlong_as_double(0x7FF8000000000000LL);
    }
}

// One 16-byte quant slice of R rows against the limb planes: lo (low nibbles,
// sub-block 2c) and hi (high nibbles, sub-block 2c+1) sums per limb.
template <int R>
__device__ __forceinline__ void fx_slice(const uint4 (&q)[R], const uint8_t *xlo, const uint8_t *xhi, int (&alo)[R][4],
                                         int (&ahi)[R][4])
{
    uint4 xa[4], xb[4];
#pragma unroll
    for (int l = 0; l < 4; ++l) {
        xa[l] = *reinterpret_cast<const uint4 *>(xlo + 256 * l);
        xb[l] = *reinterpret_cast<const uint4 *>(xhi + 256 * l);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint32_t w = (t == 0) ? q[r].x : (t == 1) ? q[r].y : (t == 2) ? q[r].z : q[r].w;
            const int lo = static_cast<int>(w & 0x0F0F0F0Fu);
            const int hi = static_cast<int>((w >> 4) & 0x0F0F0F0Fu);
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                const uint32_t x0 = (t == 0) ? xa[l].x : (t == 1) ? xa[l].y : (t == 2) ? xa[l].z : xa[l].w;
                const uint32_t x1 = (t == 0) ? xb[l].x : (t == 1) ? xb[l].y : (t == 2) ? xb[l].z : xb[l].w;
                alo[r][l] = __dp4a(lo, static_cast<int>(x0), alo[r][l]);
                ahi[r][l] = __dp4a(hi, static_cast<int>(x1), ahi[r][l]);
            }
        }
    }
}

template <int LPR, int NS, bool SOA>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) q4k_gemv_fx_kernel(const Q4KParams p)
{
    constexpr int R = 2;
    using G = Geo<LPR, R>;

    extern __shared__ __align__(128) uint8_t smem[];
    const int nwarps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rg = lane / LPR;
    const int l = lane % LPR;

    const int split = blockIdx.x / p.ctas_per_split;
    const int cj = blockIdx.x % p.ctas_per_split;
    const int nchunk_total = (p.nb + LPR - 1) / LPR;
    const int c_begin = split * p.chunks_per_split;
    const int c_end = min(c_begin + p.chunks_per_split, nchunk_total);
    const int nch = c_end - c_begin;
    const int kb_begin = c_begin * LPR;
    const int nbs = min(nch * LPR, p.nb - kb_begin);  // super-blocks of this split

    // shared memory: [limb planes][sums and scales][barriers][ring][argmax scratch]
    const int x_bytes = (nbs * (kFxLimbPitch + kFxAuxPitch) + 127) & ~127;
    uint8_t *limbs = smem;
    uint8_t *aux = smem + nbs * kFxLimbPitch;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + x_bytes);
    const int bar_bytes = (nwarps * p.depth * 8 + 127) & ~127;
    uint8_t *ring = smem + x_bytes + bar_bytes;
    uint8_t *my_ring = ring + static_cast<size_t>(warp) * p.depth * G::SLOT_BYTES;
    const uint32_t my_ring_s = smem_u32(my_ring);
    const uint32_t my_bars_s = smem_u32(bars + warp * p.depth);
    ArgmaxCand *red = reinterpret_cast<ArgmaxCand *>(ring + static_cast<size_t>(nwarps) * p.depth * G::SLOT_BYTES);

    // this warp's tiles: t0, t0 + tstride, ... (warp-major order)
    const long long tstride = static_cast<long long>(p.ctas_per_split) * nwarps;
    const long long t0 = static_cast<long long>(warp) * p.ctas_per_split + cj;
    const long long ntiles_w = (t0 < p.tiles) ? (p.tiles - t0 + tstride - 1) / tstride : 0;
    const long long total = ntiles_w * NS * nch;
    const long long row_step = tstride * G::TR;

    // After the row-group reduction of the two row sums, lane 0 of the group
    // holds row 0 and lane LPR/2 row 1 (LPR >= 2).
    const bool writer = (l & (LPR / 2 - 1)) == 0;
    const int wrow = (l >= LPR / 2) ? 1 : 0;

    Cursor pc{t0 * G::TR, 0, 0};
    long long issued = 0;
    if (lane == 0) {
        for (int s = 0; s < p.depth; ++s)
            mbar_init(my_bars_s + s * 8, 1);
        mbar_fence_init();
    }
    for (int s = 0; s < p.depth && issued < total; ++s, ++issued) {
        if (lane == 0)
            issue_slot<G>(p, pc, s, c_begin, my_ring_s, my_bars_s);
        pc.advance(nch, NS, row_step);
    }

    fx_stage(p.x, kb_begin, nbs, limbs, aux, warp, nwarps, lane);
    __syncthreads();

    float best_v = -INFINITY;
    long long best_i = 0x7fffffffffffffffLL;
    bool failed = false;
    long long consumed = 0;
    double acc[R] = {0.0, 0.0};
    double gsum = 0.0;  // stream-0 sum kept for the SwiGLU epilogue

    Cursor cc{t0 * G::TR, 0, 0};
    int slot = 0;
    uint32_t parity = 0;
    for (; consumed < total; ++consumed) {
        const bool ok = mbar_wait_bounded(my_bars_s + slot * 8, parity, p.err);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        const int kb0 = (c_begin + cc.kcl) * LPR;
        const int nblk = min(LPR, p.nb - kb0);
        if (l < nblk) {
            const uint8_t *slot_p = my_ring + slot * G::SLOT_BYTES + rg * G::RG_PITCH;
            int hdr_off, qs_off0, qs_step;
            if constexpr (SOA) {
                hdr_off = 16 * l;
                qs_off0 = 16 * nblk + 16 * l;
                qs_step = 16 * nblk;
            } else {
                hdr_off = kQ4KBlockBytes * l;
                qs_off0 = hdr_off + 16;
                qs_step = 16;
            }
            uint4 hd[R];
            uint32_t sc03[R], sc47[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                hd[r] = *reinterpret_cast<const uint4 *>(slot_p + r * G::ROW_BYTES + hdr_off);
                // GGML get_scale_min_k4 packing: scales 0..3 are the low six bits of
                // bytes 0..3; scales 4..7 take their low four bits from the low nibbles
                // of bytes 8..11 and their top two bits from bits 6..7 of bytes 0..3
                sc03[r] = hd[r].y & 0x3F3F3F3Fu;
                sc47[r] = (hd[r].w & 0x0F0F0F0Fu) | ((hd[r].y >> 2) & 0x30303030u);
            }
            const uint8_t *xb = limbs + (kb0 - kb_begin + l) * kFxLimbPitch;

            int isum[R][4];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    isum[r][k] = 0;
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
                        q[r] = *reinterpret_cast<const uint4 *>(slot_p + r * G::ROW_BYTES + qs_off0 + s * qs_step);
                    fx_slice<R>(q, xb + 64 * c + 16 * h, xb + 64 * c + 32 + 16 * h, alo, ahi);
                }
                // fold the scales of sub-blocks 2c (lo) and 2c+1 (hi)
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint32_t sw = (c < 2) ? sc03[r] : sc47[r];
                    const int slo = static_cast<int>((sw >> (16 * (c & 1))) & 0xFFu);
                    const int shi = static_cast<int>((sw >> (16 * (c & 1) + 8)) & 0xFFu);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        isum[r][k] += slo * alo[r][k] + shi * ahi[r][k];
                }
            }

            // per row: y_sb = 2^-F (d I_s - dmin I_m) in fp64
            const double *ap = reinterpret_cast<const double *>(aux + (kb0 - kb_begin + l) * kFxAuxPitch);
            double X[8];
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const double2 t = *reinterpret_cast<const double2 *>(ap + j);
                X[j] = t.x;
                X[j + 1] = t.y;
            }
            const double s2f = ap[8];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                double is = static_cast<double>(isum[r][3]);
                is = fma(is, 256.0, static_cast<double>(isum[r][2]));
                is = fma(is, 256.0, static_cast<double>(isum[r][1]));
                is = fma(is, 256.0, static_cast<double>(isum[r][0]));
                const uint32_t mn03 = hd[r].z & 0x3F3F3F3Fu;
                const uint32_t mn47 = ((hd[r].w >> 4) & 0x0F0F0F0Fu) | ((hd[r].z >> 2) & 0x30303030u);
                double im = 0.0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t mw = (j < 4) ? mn03 : mn47;
                    im = fma(static_cast<double>((mw >> (8 * (j & 3))) & 0xFFu), X[j], im);
                }
                const double d = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(hd[r].x & 0xFFFFu)))) * s2f;
                const double dm = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(hd[r].x >> 16)))) * s2f;
                const double pm = dm * im;            // rounded
                const double em = fma(dm, im, -pm);   // its exact rounding error
                acc[r] += fma(d, is, -pm) - em;
            }
        }

        __syncwarp();
        if (issued < total) {
            if (lane == 0) {
                fence_proxy_async_smem();
                issue_slot<G>(p, pc, slot, c_begin, my_ring_s, my_bars_s);
            }
            pc.advance(nch, NS, row_step);
            ++issued;
        }

        const int cur_st = cc.st;
        const long long row0 = cc.row0;
        const bool last_chunk = (cc.kcl == nch - 1);
        cc.advance(nch, NS, row_step);
        if (++slot == p.depth) {
            slot = 0;
            parity ^= 1u;
        }
        if (!last_chunk)
            continue;

        // end of this stream's K range for the tile: reduce across the row group
        double v[R] = {acc[0], acc[1]};
        acc[0] = 0.0;
        acc[1] = 0.0;
        GroupReduce<LPR / 2, R, double>::run(v, l);
        if constexpr (NS == 2) {
            if (cur_st == 0) {
                gsum = v[0];
                continue;
            }
        }
        const long long n = row0 + rg * R + wrow;
        if (!writer || n >= p.N)
            continue;
        if (p.splits > 1) {
            if constexpr (NS == 2) {
                p.part[(static_cast<long long>(split) * 2 + 0) * p.N + n] = static_cast<float>(gsum);
                p.part[(static_cast<long long>(split) * 2 + 1) * p.N + n] = static_cast<float>(v[0]);
            } else {
                p.part[static_cast<long long>(split) * p.N + n] = static_cast<float>(v[0]);
            }
        } else {
            float out;
            if constexpr (NS == 2) {
                const float g = static_cast<float>(gsum);
                out = g / (1.0f + expf(-g)) * static_cast<float>(v[0]);
            } else {
                out = static_cast<float>(v[0]);
            }
            p.y[n] = out;
            if (p.argmax && cand_better(out, n, best_v, best_i)) {
                best_v = out;
                best_i = n;
            }
        }
    }

    if (failed) {
        // the copies already issued into this warp's ring must land before the CTA exits
        for (long long i = consumed; i < issued; ++i) {
            mbar_wait_bounded(my_bars_s + slot * 8, parity, nullptr);
            if (++slot == p.depth) {
                slot = 0;
                parity ^= 1u;
            }
        }
    }

    if (p.argmax && p.splits == 1) {
        // CTA-wide (max, lowest index) candidate
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
            const long long oi = __shfl_xor_sync(0xffffffffu, best_i, o);
            if (cand_better(ov, oi, best_v, best_i)) {
                best_v = ov;
                best_i = oi;
            }
        }
        if (lane == 0) {
            red[warp].v = best_v;
            red[warp].idx = best_i;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            ArgmaxCand c = red[0];
            for (int w = 1; w < nwarps; ++w)
                if (cand_better(red[w].v, red[w].idx, c.v, c.idx))
                    c = red[w];
            p.cand[blockIdx.x] = c;
        }
    }
}

template <int LPR, int NS>
static cudaError_t launch_fx(const Q4KParams &p, const Q4KPlan &pl, cudaStream_t s)
{
    auto k = p.soa ? q4k_gemv_fx_kernel<LPR, NS, true> : q4k_gemv_fx_kernel<LPR, NS, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess)
        return e;
    k<<<pl.grid, pl.warps * 32, pl.smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t q4k_gemv_fx_launch(const Q4KParams &p, const Q4KPlan &pl, int NS, cudaStream_t s)
{
    if (pl.lpr == 16)
        return NS == 1 ? launch_fx<16, 1>(p, pl, s) : launch_fx<16, 2>(p, pl, s);
    return NS == 1 ? launch_fx<4, 1>(p, pl, s) : launch_fx<4, 2>(p, pl, s);
}

}  // namespace dq
