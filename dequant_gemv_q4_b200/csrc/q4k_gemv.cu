// q4k_gemv.cu -- fused Q4_K dequantize + GEMV (plain, fused SwiGLU, B <= 8,
// optional argmax) for sm_100a.
//
// The operation is the pages' fused dequant+GEMV over raw Q4_K bytes (trueno
// WgslForwardPass: upload_q4k_weight; qualiaDB cuda_lane: try_q4k_soa_gemv,
// try_q4k_soa_fused_swiglu).  The kernel design below is this library's own.
//
// Work decomposition
//   A warp owns a set of row tiles.  A row tile is TR = (32/LPR)*R rows; lane
//   (rg, l) = (lane / LPR, lane % LPR) handles rows rg*R .. rg*R+R-1 of the
//   tile and, in every K-chunk of LPR super-blocks, super-block l of each of
//   those rows.  One "slot" is one K-chunk of one tile of one weight stream
//   (TR rows x LPR super-blocks, 9 KB for R = 2).  Each warp streams its own
//   ring of `depth` slots: lane 0 issues 1-D bulk copies (cp.async.bulk from
//   this GPU's global memory into the warp's shared-memory slot, completing on
//   an mbarrier), the whole warp computes on the oldest slot and lane 0 reuses
//   it for the slot `depth` steps ahead.  CTAs are persistent: a grid of about
//   one CTA per SM walks all tiles.  K may be split across CTAs (split-K) when
//   the activations of all of K do not fit in shared memory or when there are
//   too few row tiles to occupy the GPU; split partial sums go to the caller's
//   workspace and a second kernel reduces them in a fixed order.
//
// Arithmetic (per weight, no factoring of scales or mins)
//   A quant q at bit position p of a 32-bit word, isolated with one AND, is
//   the fp32 bit pattern q*2^p, i.e. the subnormal (or smallest-normal) value
//   q*2^(p-149).  One fma with d*scale*2^(85-p) and -dmin*min*2^-64 then gives
//   (d*scale*q - dmin*min) * 2^-64 rounded once: exactly the fp32 weight that
//   q4k_dequant returns, times 2^-64 (all operands are exact: d has 11
//   significant bits, scale and min 6, q 4).  A second fma accumulates
//   weight*x.  Sums are taken in units of 2^-64 and scaled back at the end, so
//   any finite fp32 x is accepted.  Both fmas run as fma.rn.f32x2 on pairs.
//   Subnormal operands are kept (the library is built without flush-to-zero).

#include <cuda_fp16.h>
#include <cstdint>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "q4k_decode.cuh"
#include "q4k_stream.cuh"

namespace dq {

template <int LPR, int B, int NS, bool SOA>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) q4k_gemv_kernel(const Q4KParams p)
{
    pdl_wait();
    pdl_launch_dependents();
    constexpr int R = 2;
    using G = Geo<LPR, R>;
    constexpr int MV = R * B;                         // values per lane per stream
    constexpr int MP = Pow2Ceil<MV>::value;           // padded to a power of two
    constexpr int VPL = (MP > LPR) ? MP / LPR : 1;    // values per lane after reduce

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

    // shared memory: [x staging][barriers][ring][argmax scratch]
    const int x_bytes = (B * nbs * kXBlockPitch + 127) & ~127;
    uint8_t *xs = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + x_bytes);
    const int bar_bytes = (nwarps * p.depth * 8 + 127) & ~127;
    uint8_t *ring = smem + x_bytes + bar_bytes;
    uint8_t *my_ring = ring + static_cast<size_t>(warp) * p.depth * G::SLOT_BYTES;
    const uint32_t my_ring_s = smem_u32(my_ring);
    const uint32_t my_bars_s = smem_u32(bars + warp * p.depth);
    ArgmaxCand *red = reinterpret_cast<ArgmaxCand *>(ring + static_cast<size_t>(nwarps) * p.depth * G::SLOT_BYTES);

    // this warp's tiles: t0, t0 + tstride, ...
    const long long tstride = static_cast<long long>(p.ctas_per_split) * nwarps;
    // warp-major tile order: the last, partial round of tiles spreads over all SMs
    const long long t0 = static_cast<long long>(warp) * p.ctas_per_split + cj;
    const long long ntiles_w = (t0 < p.tiles) ? (p.tiles - t0 + tstride - 1) / tstride : 0;
    const long long total = ntiles_w * NS * nch;
    const long long row_step = tstride * G::TR;

    // After the row-group reduction this lane holds value indices
    // off .. off + VPL - 1 (value index = r * B + b); only `writer` lanes store.
    int off = 0;
    bool writer = true;
    {
        int m = MP;
#pragma unroll
        for (int o = LPR / 2; o >= 1; o >>= 1) {
            if (m > 1) {
                if (l & o)
                    off += m / 2;
                m /= 2;
            } else if (l & o) {
                writer = false;
            }
        }
    }

    // producer cursor (used by lane 0, advanced in every lane)
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

    // stage this split's activations in (lo, hi) pairs (fp32, padded per super-block);
    // each thread keeps 8 loads in flight before storing (one at a time for
    // large B, whose kernels have no registers to spare)
    stage_x_pairs<(B <= 2) ? 8 : 1>(p.x, p.K, B, kb_begin, nbs, xs);
    __syncthreads();

    float best_v = -INFINITY;
    long long best_i = 0x7fffffffffffffffLL;
    bool failed = false;
    long long consumed = 0;

    float2 acc0[R][B], acc1[R][B];
    float gsum[NS == 2 ? VPL : 1];  // stream-0 sums kept for the SwiGLU epilogue
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) {
            acc0[r][b] = f2(0.f, 0.f);
            acc1[r][b] = f2(0.f, 0.f);
        }

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
            // byte offsets of this lane's header and quant slices within a row of the slot
            const BlockOffsets bo = block_offsets<SOA>(l, nblk);
            const int hdr_off = bo.hdr, qs_off0 = bo.qs0, qs_step = bo.qs_step;
            Hdr hd[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                hd[r] = decode_hdr(*reinterpret_cast<const uint4 *>(slot_p + r * G::ROW_BYTES + hdr_off));
            const uint8_t *xblk = xs + (kb0 - kb_begin + l) * kXBlockPitch;

#pragma unroll
            for (int c = 0; c < 4; ++c) {
                ChunkScales cs[R];
#pragma unroll
                for (int r = 0; r < R; ++r)
                    cs[r] = chunk_scales(hd[r], c);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int s = 2 * c + h;  // 16-byte quant slice
                    uint4 q[R];
#pragma unroll
                    for (int r = 0; r < R; ++r)
                        q[r] = *reinterpret_cast<const uint4 *>(slot_p + r * G::ROW_BYTES + qs_off0 + s * qs_step);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
#pragma unroll
                        for (int b = 0; b < B; ++b) {
                            const uint8_t *xq = xblk + b * nbs * kXBlockPitch + s * 128 + 32 * t;
                            const float4 xa = *reinterpret_cast<const float4 *>(xq);
                            const float4 xb = *reinterpret_cast<const float4 *>(xq + 16);
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                const uint32_t wv = (t == 0) ? q[r].x : (t == 1) ? q[r].y : (t == 2) ? q[r].z : q[r].w;
                                q4_word(wv, cs[r], xa, xb, acc0[r][b], acc1[r][b]);
                            }
                        }
                    }
                }
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
        float v[MP];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int b = 0; b < B; ++b) {
                const float2 a = __fadd2_rn(acc0[r][b], acc1[r][b]);
                v[r * B + b] = a.x + a.y;
                acc0[r][b] = f2(0.f, 0.f);
                acc1[r][b] = f2(0.f, 0.f);
            }
#pragma unroll
        for (int j = MV; j < MP; ++j)
            v[j] = 0.f;
        if constexpr (LPR > 1)
            GroupReduce<LPR / 2, MP>::run(v, l);

        if constexpr (NS == 2) {
            if (cur_st == 0) {
#pragma unroll
                for (int j = 0; j < VPL; ++j)
                    gsum[j] = v[j];
                continue;
            }
        }
        if (!writer)
            continue;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int idx = off + j;
            if (idx >= MV)
                continue;
            const int r = idx / B;
            const int b = idx % B;
            const long long n = row0 + rg * R + r;
            if (n >= p.N)
                continue;
            if (p.splits > 1) {
                if constexpr (NS == 2) {
                    p.part[((static_cast<long long>(split) * 2 + 0) * B + b) * p.N + n] = gsum[j] * 0x1p64f;
                    p.part[((static_cast<long long>(split) * 2 + 1) * B + b) * p.N + n] = v[j] * 0x1p64f;
                } else {
                    p.part[(static_cast<long long>(split) * B + b) * p.N + n] = v[j] * 0x1p64f;
                }
            } else {
                float out;
                if constexpr (NS == 2) {
                    const float g = gsum[j] * 0x1p64f;
                    const float u = v[j] * 0x1p64f;
                    out = g / (1.0f + expf(-g)) * u;
                } else {
                    out = v[j] * 0x1p64f;
                }
                *gemv_out_addr(p.y, p.g, p.qg_hd, p.N, b, n) = out;
                if (p.argmax && cand_better(out, n, best_v, best_i)) {
                    best_v = out;
                    best_i = n;
                }
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

// ---------------------------------------------------------------------------
// Batch-1 kernel with half-block lanes (GeoHalf): each lane owns two of the
// four 64-weight chunks of one super-block for two rows, so a slot is 4.5 KB
// and sixteen warps (four per scheduler) fit beside their two-deep rings.
// x keeps the (lo, hi) pair staging, with the two 512-byte halves of every
// super-block kXHalfGap bytes apart and kXHalfPitch bytes per super-block, so
// the eight lanes of one shared-memory phase read eight distinct bank groups.
// ---------------------------------------------------------------------------
constexpr int kB1Warps = 16;
constexpr int kXHalfPitch = 1056;
constexpr int kXHalfGap = 528;

template <int LPR, int NS, bool SOA>
__global__ void __launch_bounds__(kB1Warps * 32, 1) q4k_gemv_b1_kernel(const Q4KParams p)
{
    pdl_wait();
    pdl_launch_dependents();
    using G = GeoHalf<LPR>;
    constexpr int R = G::R;

    extern __shared__ __align__(128) uint8_t smem[];
    const int nwarps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rg = lane / LPR;
    const int l = lane % LPR;
    const int bl = l >> 1;   // super-block of the chunk
    const int hh = l & 1;    // half: chunks 2*hh and 2*hh + 1

    const int split = blockIdx.x / p.ctas_per_split;
    const int cj = blockIdx.x % p.ctas_per_split;
    const int nchunk_total = (p.nb + G::BPC - 1) / G::BPC;
    const int c_begin = split * p.chunks_per_split;
    const int c_end = min(c_begin + p.chunks_per_split, nchunk_total);
    const int nch = c_end - c_begin;
    const int kb_begin = c_begin * G::BPC;
    const int nbs = min(nch * G::BPC, p.nb - kb_begin);

    // shared memory: [x staging][barriers][ring][argmax scratch]
    const int x_bytes = (nbs * kXHalfPitch + 127) & ~127;
    uint8_t *xs = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + x_bytes);
    const int bar_bytes = (nwarps * p.depth * 8 + 127) & ~127;
    uint8_t *ring = smem + x_bytes + bar_bytes;
    uint8_t *my_ring = ring + static_cast<size_t>(warp) * p.depth * G::SLOT_BYTES;
    const uint32_t my_ring_s = smem_u32(my_ring);
    const uint32_t my_bars_s = smem_u32(bars + warp * p.depth);
    ArgmaxCand *red = reinterpret_cast<ArgmaxCand *>(ring + static_cast<size_t>(nwarps) * p.depth * G::SLOT_BYTES);

    const long long tstride = static_cast<long long>(p.ctas_per_split) * nwarps;
    // warp-major tile order: the last, partial round of tiles spreads over all SMs
    const long long t0 = static_cast<long long>(warp) * p.ctas_per_split + cj;
    const long long ntiles_w = (t0 < p.tiles) ? (p.tiles - t0 + tstride - 1) / tstride : 0;
    const long long total = ntiles_w * NS * nch;
    const long long row_step = tstride * G::TR;

    // After the row-group reduction lane 0 of the group holds row 0's sum and
    // lane LPR/2 row 1's; the other lanes hold copies.
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

    // stage x in (lo, hi) pairs, 8 loads in flight per thread
    {
        constexpr int kStageBatch = 8;
        const int n_out = nbs * 64;
        for (int base = threadIdx.x; base < n_out; base += kStageBatch * blockDim.x) {
            float2 lo[kStageBatch], hi[kStageBatch];
#pragma unroll
            for (int u = 0; u < kStageBatch; ++u) {
                const int idx = base + u * blockDim.x;
                if (idx < n_out) {
                    const int kbl = idx >> 6, sl = (idx >> 3) & 7, k = idx & 7;
                    const float *xb = p.x + static_cast<long long>(kb_begin + kbl) * 256 + 64 * (sl >> 1) +
                                      16 * (sl & 1) + 2 * k;
                    lo[u] = __ldg(reinterpret_cast<const float2 *>(xb));
                    hi[u] = __ldg(reinterpret_cast<const float2 *>(xb + 32));
                }
            }
#pragma unroll
            for (int u = 0; u < kStageBatch; ++u) {
                const int idx = base + u * blockDim.x;
                if (idx < n_out) {
                    const int kbl = idx >> 6, sl = (idx >> 3) & 7, k = idx & 7;
                    *reinterpret_cast<float4 *>(xs + kbl * kXHalfPitch + (sl >> 2) * kXHalfGap + (sl & 3) * 128 +
                                                k * 16) = make_float4(lo[u].x, hi[u].x, lo[u].y, hi[u].y);
                }
            }
        }
    }
    __syncthreads();

    float best_v = -INFINITY;
    long long best_i = 0x7fffffffffffffffLL;
    bool failed = false;
    long long consumed = 0;
    float gsum = 0.f;  // stream-0 sum kept for the SwiGLU epilogue

    float2 acc0[R], acc1[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        acc0[r] = f2(0.f, 0.f);
        acc1[r] = f2(0.f, 0.f);
    }

    Cursor cc{t0 * G::TR, 0, 0};
    int slot = 0;
    uint32_t parity = 0;
    for (; consumed < total; ++consumed) {
        const bool ok = mbar_wait_bounded(my_bars_s + slot * 8, parity, p.err);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        const int kb0 = (c_begin + cc.kcl) * G::BPC;
        const int nblk = min(G::BPC, p.nb - kb0);
        if (bl < nblk) {
            const uint8_t *slot_p = my_ring + slot * G::SLOT_BYTES + rg * G::RG_PITCH;
            // this lane's header and its first quant slice (slice 4*hh of the super-block)
            const BlockOffsets bo = block_offsets<SOA>(bl, nblk);
            const int hdr_off = bo.hdr, qs_step = bo.qs_step;
            const int qs_off0 = bo.qs0 + 4 * hh * bo.qs_step;
            Hdr hd[R];
            uint32_t scw[R], mnw[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                hd[r] = decode_hdr(*reinterpret_cast<const uint4 *>(slot_p + r * G::ROW_BYTES + hdr_off));
                scw[r] = hh ? hd[r].sc47 : hd[r].sc03;
                mnw[r] = hh ? hd[r].mn47 : hd[r].mn03;
            }
            const uint8_t *xl = xs + (kb0 - kb_begin + bl) * kXHalfPitch + hh * kXHalfGap;

#pragma unroll
            for (int cp = 0; cp < 2; ++cp) {  // chunk 2*hh + cp
                ChunkScales cs[R];
#pragma unroll
                for (int r = 0; r < R; ++r)
                    cs[r] = scales_from_words(hd[r], scw[r], mnw[r], cp * 2);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int sl = 2 * cp + h;  // slice within the half
                    uint4 q[R];
#pragma unroll
                    for (int r = 0; r < R; ++r)
                        q[r] = *reinterpret_cast<const uint4 *>(slot_p + r * G::ROW_BYTES + qs_off0 + sl * qs_step);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint8_t *xq = xl + sl * 128 + 32 * t;
                        const float4 xa = *reinterpret_cast<const float4 *>(xq);
                        const float4 xb = *reinterpret_cast<const float4 *>(xq + 16);
#pragma unroll
                        for (int r = 0; r < R; ++r) {
                            const uint32_t wv = (t == 0) ? q[r].x : (t == 1) ? q[r].y : (t == 2) ? q[r].z : q[r].w;
                            q4_word(wv, cs[r], xa, xb, acc0[r], acc1[r]);
                        }
                    }
                }
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

        float v[2];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float2 a = __fadd2_rn(acc0[r], acc1[r]);
            v[r] = a.x + a.y;
            acc0[r] = f2(0.f, 0.f);
            acc1[r] = f2(0.f, 0.f);
        }
        GroupReduce<LPR / 2, 2>::run(v, l);
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
                p.part[(static_cast<long long>(split) * 2 + 0) * p.N + n] = gsum * 0x1p64f;
                p.part[(static_cast<long long>(split) * 2 + 1) * p.N + n] = v[0] * 0x1p64f;
            } else {
                p.part[static_cast<long long>(split) * p.N + n] = v[0] * 0x1p64f;
            }
        } else {
            float out;
            if constexpr (NS == 2) {
                const float g = gsum * 0x1p64f;
                out = g / (1.0f + expf(-g)) * (v[0] * 0x1p64f);
            } else {
                out = v[0] * 0x1p64f;
            }
            *gemv_out_addr(p.y, p.g, p.qg_hd, p.N, 0, n) = out;
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

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

int q4k_slot_bytes(int lpr) { return lpr == 16 ? Geo<16, 2>::SLOT_BYTES : Geo<4, 2>::SLOT_BYTES; }

// Launch plan for a shape; the same function sizes the workspace, so the two
// always agree.
// Warps per CTA for `tiles` row tiles on `sm_count` SMs (one CTA per SM):
// enough to give every SM work and at least one per scheduler; with `round4`
// a multiple of four, so the four schedulers of an SM carry equal numbers of
// warps (the full-block kernel skips the rounding when its shared memory
// would then force a K split).
int q4k_pick_warps(long long tiles, int sm_count, int max_warps, bool round4)
{
    long long w = (tiles + sm_count - 1) / sm_count;
    if (round4)
        w = (w + 3) / 4 * 4;
    if (w < 4)
        w = 4;
    if (w > max_warps)
        w = max_warps;
    return static_cast<int>(w);
}

static Q4KPlan q4k_plan_half(long long N, int nb, int NS, int sm_count, int smem_optin)
{
    Q4KPlan pl{};
    const int misc = 256 /*argmax scratch*/ + 512 /*barriers*/;
    // 16-block chunks when they tile the row, else 4-block chunks (both start
    // at SoA group boundaries)
    const int lpr = (nb % 16 == 0) ? 32 : 8;
    const int bpc = lpr / 2;
    const int sb = (lpr == 32) ? GeoHalf<32>::SLOT_BYTES : GeoHalf<8>::SLOT_BYTES;
    const int TR = (32 / lpr) * 2;
    const long long tiles = (N + TR - 1) / TR;
    const int nchunk = (nb + bpc - 1) / bpc;
    const int w0 = q4k_pick_warps(tiles, sm_count, kB1Warps, true);
    for (int warps = w0; warps >= 4 && !pl.ok; warps = (warps > 4 && warps / 2 < 4) ? 4 : warps / 2) {
        int splits = 1, cps = nchunk;
        for (;;) {
            cps = (nchunk + splits - 1) / splits;
            if (cps * bpc * kXHalfPitch + warps * 2 * sb + misc <= smem_optin || cps == 1)
                break;
            ++splits;
        }
        const long long warps_total = static_cast<long long>(sm_count) * warps;
        while (tiles * NS * splits * 2 < warps_total && splits < nchunk) {
            ++splits;
            cps = (nchunk + splits - 1) / splits;
        }
        splits = (nchunk + cps - 1) / cps;
        const int x_bytes = (cps * bpc * kXHalfPitch + 127) & ~127;
        int depth = (smem_optin - x_bytes - misc) / (warps * sb);
        if (depth > 4)
            depth = 4;
        if (depth < 2)
            continue;
        long long ctas = (tiles + warps - 1) / warps;
        const long long max_ctas = sm_count / splits > 0 ? sm_count / splits : 1;
        if (ctas > max_ctas)
            ctas = max_ctas;
        pl.half = true;
        pl.lpr = lpr;
        pl.R = 2;
        pl.warps = warps;
        pl.tiles = tiles;
        pl.splits = splits;
        pl.chunks_per_split = cps;
        pl.depth = depth;
        pl.ctas_per_split = static_cast<int>(ctas);
        pl.grid = pl.ctas_per_split * splits;
        pl.smem = x_bytes + ((warps * depth * 8 + 127) & ~127) + warps * depth * sb + 256;
        pl.ok = pl.smem <= smem_optin;
    }
    return pl;
}

// Full-block plan of the fp32 kernel: `stage_bytes` is the shared memory the
// staged activations take per super-block.
static Q4KPlan plan_full_block(long long N, int nb, int NS, int sm_count, int smem_optin, int stage_bytes)
{
    Q4KPlan pl{};
    const int misc = 256 /*argmax scratch, 16 B per warp*/ + 256 /*barriers*/;
    // 16-block chunks when they tile the row, else 4-block chunks (both start
    // at SoA group boundaries)
    const int lpr_opts[2] = {(nb % 16 == 0) ? 16 : 4, 4};
    const int n_opts = (nb % 16 != 0) ? 1 : 2;
    for (int oi = 0; oi < n_opts && !pl.ok; ++oi) {
        const int lpr = lpr_opts[oi];
        const int R = 2;
        const int sb = q4k_slot_bytes(lpr);
        const int TR = (32 / lpr) * R;
        const long long tiles = (N + TR - 1) / TR;
        const int nchunk = (nb + lpr - 1) / lpr;
        const int w0 = q4k_pick_warps(tiles, sm_count, kMaxWarps, false);
        for (int warps = w0; warps >= 4 && !pl.ok; warps = (warps > 4 && warps / 2 < 4) ? 4 : warps / 2) {
            const int min_ring = warps * 2 * sb;
            // smallest split count whose activations fit beside a two-deep ring
            int splits = 1;
            int cps = nchunk;
            for (;;) {
                cps = (nchunk + splits - 1) / splits;
                const int xb = cps * lpr * stage_bytes;
                if (xb + min_ring + misc <= smem_optin || cps == 1)
                    break;
                ++splits;
            }
            // split K further while fewer than half of the warps would have a tile
            const long long warps_total = static_cast<long long>(sm_count) * warps;
            while (tiles * NS * splits * 2 < warps_total && splits < nchunk) {
                ++splits;
                cps = (nchunk + splits - 1) / splits;
            }
            splits = (nchunk + cps - 1) / cps;
            const int x_bytes = (cps * lpr * stage_bytes + 127) & ~127;
            int depth = (smem_optin - x_bytes - misc) / (warps * sb);
            if (depth > 4)
                depth = 4;
            if (depth < 2)
                continue;
            long long ctas = (tiles + warps - 1) / warps;
            const long long max_ctas = sm_count / splits > 0 ? sm_count / splits : 1;
            if (ctas > max_ctas)
                ctas = max_ctas;
            pl.lpr = lpr;
            pl.R = R;
            pl.warps = warps;
            pl.tiles = tiles;
            pl.splits = splits;
            pl.chunks_per_split = cps;
            pl.depth = depth;
            pl.ctas_per_split = static_cast<int>(ctas);
            pl.grid = pl.ctas_per_split * splits;
            pl.smem = x_bytes + ((warps * depth * 8 + 127) & ~127) + warps * depth * sb + 256;
            pl.ok = pl.smem <= smem_optin;
        }
    }
    return pl;
}

Q4KPlan q4k_plan(long long N, int K, int B, int NS, int soa, int sm_count, int smem_optin)
{
    const int nb = K / kQ4KBlockElems;
    // quarter-warp lanes with TMA slots: integer dot products on fixed-point
    // activations at batch 1, exact fp32 weights at batch 2..8
    const Q4KPlan pf = q4k_plan_fx(N, nb, B, NS, sm_count, smem_optin);
    if (pf.ok)
        return pf;
    if (B == 1) {
        // Half-block lanes halve each warp's serial chain of slots (better when
        // every warp gets only a few slots); full-block lanes spend fewer
        // instructions per weight (better for long matrices).
        const int full_lpr = (nb % 16 == 0) ? 16 : 4;
        const long long full_tiles = (N + (32 / full_lpr) * 2 - 1) / ((32 / full_lpr) * 2);
        const long long slots = full_tiles * NS * ((nb + full_lpr - 1) / full_lpr);
        if (slots < 8LL * sm_count * kMaxWarps) {
            const Q4KPlan ph = q4k_plan_half(N, nb, NS, sm_count, smem_optin);
            if (ph.ok)
                return ph;
        }
    }
    return plan_full_block(N, nb, NS, sm_count, smem_optin, B * kXBlockPitch);
}

template <int LPR, int B, int NS>
static cudaError_t launch_one(const Q4KParams &p, const Q4KPlan &pl, cudaStream_t s)
{
    auto k = p.soa ? q4k_gemv_kernel<LPR, B, NS, true> : q4k_gemv_kernel<LPR, B, NS, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(k, dim3(pl.grid), dim3(pl.warps * 32), pl.smem, s, p);
}

template <int LPR, int NS>
static cudaError_t launch_b(const Q4KParams &p, const Q4KPlan &pl, int B, cudaStream_t s)
{
    switch (B) {
    case 1: return launch_one<LPR, 1, NS>(p, pl, s);
    case 2: return launch_one<LPR, 2, NS>(p, pl, s);
    case 3: return launch_one<LPR, 3, NS>(p, pl, s);
    case 4: return launch_one<LPR, 4, NS>(p, pl, s);
    case 5: return launch_one<LPR, 5, NS>(p, pl, s);
    case 6: return launch_one<LPR, 6, NS>(p, pl, s);
    case 7: return launch_one<LPR, 7, NS>(p, pl, s);
    case 8: return launch_one<LPR, 8, NS>(p, pl, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int LPR, int NS>
static cudaError_t launch_half(const Q4KParams &p, const Q4KPlan &pl, cudaStream_t s)
{
    auto k = p.soa ? q4k_gemv_b1_kernel<LPR, NS, true> : q4k_gemv_b1_kernel<LPR, NS, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(k, dim3(pl.grid), dim3(pl.warps * 32), pl.smem, s, p);
}

cudaError_t q4k_gemv_launch(const Q4KParams &p, const Q4KPlan &pl, int B, int NS, cudaStream_t s)
{
    if (pl.fx)
        return q4k_gemv_fx_launch(p, pl, B, NS, s);
    if (pl.half) {
        if (pl.lpr == 32)
            return NS == 1 ? launch_half<32, 1>(p, pl, s) : launch_half<32, 2>(p, pl, s);
        return NS == 1 ? launch_half<8, 1>(p, pl, s) : launch_half<8, 2>(p, pl, s);
    }
    if (pl.lpr == 16)
        return NS == 1 ? launch_b<16, 1>(p, pl, B, s) : launch_b<16, 2>(p, pl, B, s);
    return NS == 1 ? launch_b<4, 1>(p, pl, B, s) : launch_b<4, 2>(p, pl, B, s);
}

}  // namespace dq
