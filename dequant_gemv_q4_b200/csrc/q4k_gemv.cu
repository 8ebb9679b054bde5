// q4k_gemv.cu -- fused Q4_K dequantize + GEMV for sm_100a: plain, fused
// SwiGLU, Q/gate split, grouped matrices and argmax at batch 1
// (q4k_gemv_fx_kernel: integer dot products on fixed-point activations), and
// batches of 2..8 (q4k_gemv_fxb_kernel: exact fp32 weights).
//
// The operation is the pages' fused dequant+GEMV over raw Q4_K bytes (trueno
// WgslForwardPass: upload_q4k_weight; qualiaDB cuda_lane: try_q4k_soa_gemv,
// try_q4k_soa_fused_swiglu).  The arithmetic below is this library's own.
//
// Why integers.  At batch 1 every weight is used once, so the cost per weight
// is what bounds the kernel.  Forming each fp32 weight (an AND to isolate the
// quant, an fma with scale and min) and then an fma with x costs three
// instructions per weight on two half-rate pipes.  Here four quants at a time
// are unpacked into bytes (one AND for the four low nibbles of a word, one AND
// for the four high nibbles, left in place as 16 q) and multiplied against four
// bytes of x by one dp4a (four 8-bit products summed into an int32).
//
// The arithmetic and the lane layout are described in q4k_fx.cuh.
//
// Slot copies.  Slot rows sit at a 592-byte pitch (576 + 16), which places the
// eight rows a quarter-warp reads at one time in eight distinct bank groups.
// One TMA tile copy moves a slot: the matrix is described to the TMA unit as
// [N rows][row bytes / 4] 32-bit words and a box of 16 rows x 148 words is
// copied, i.e. each row's chunk plus the next 16 bytes of that row (zeros past
// its end), so the box itself lays the rows out at the padded pitch.  Without
// the driver's tensor-map encoder each row is its own 1-D bulk copy instead.

#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "q4k_decode.cuh"
#include "q4k_stream.cuh"
#include "q4k_exact.cuh"
#include "q4k_fx.cuh"

namespace dq {

int q4k_fx_tile_rows() { return kFxTileRows; }

// The matrix a slot reads and its rows: SwiGLU stream st of the same rows, or,
// for a grouped GEMV, the matrix holding padded row row0 and the row there.
struct FxRows {
    int sel;
    long long row0;
    long long nrows;
};
__device__ __forceinline__ FxRows fx_rows(const Q4KParams &p, int st, long long row0)
{
    if (p.grp.n == 0)
        return {st, row0, p.N};
    int m = 0;
#pragma unroll
    for (int k = 1; k < kMaxGroup; ++k)
        if (k < p.grp.n && row0 >= p.grp.base[k])
            m = k;
    const long long base = m == 0 ? p.grp.base[0] : m == 1 ? p.grp.base[1] : m == 2 ? p.grp.base[2] : p.grp.base[3];
    const long long rows = m == 0 ? p.grp.N[0] : m == 1 ? p.grp.N[1] : m == 2 ? p.grp.N[2] : p.grp.N[3];
    return {m, row0 - base, rows};
}
__device__ __forceinline__ const uint8_t *fx_weights(const Q4KParams &p, int sel)
{
    if (p.grp.n == 0)
        return sel == 0 ? p.w[0] : p.w[1];
    return sel == 0 ? p.gw[0] : sel == 1 ? p.gw[1] : sel == 2 ? p.gw[2] : p.gw[3];
}
__device__ __forceinline__ float *fx_group_out(const Q4KParams &p, int sel)
{
    return sel == 0 ? p.grp.y[0] : sel == 1 ? p.grp.y[1] : sel == 2 ? p.grp.y[2] : p.grp.y[3];
}

// Issues the copies of one slot: super-blocks kb0 .. kb0 + 3 of stream st (or,
// in a grouped GEMV, of the matrix holding padded row row0) for the row tile at
// row0, into shared memory at dst, completing on the mbarrier at bar.  TMA:
// lane 0 arms the barrier and issues one tile copy (elements past the matrix
// are filled with zeros and still counted).  Otherwise lane 0 arms the barrier
// with the slot's byte count and lane r copies row r.  `lost` (a test hook)
// arms the barrier and issues nothing, so that the wait for this slot runs out.
template <bool TMA>
__device__ __forceinline__ void fx_issue_copy(const Q4KParams &p, const FxMaps &maps, int st, long long row0, int kb0,
                                              uint32_t dst, uint32_t bar, int lane, bool lost = false)
{
    const FxRows fr = fx_rows(p, st, row0);
    if constexpr (TMA) {
        if (lane == 0) {
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kFxSlotBytes));
            if (lost)
                return;
            const CUtensorMap *m = fr.sel == 0 ? &maps.m[0] : fr.sel == 1 ? &maps.m[1] : fr.sel == 2 ? &maps.m[2]
                                                                                                      : &maps.m[3];
            // x = kb0 * 36 words: a multiple of 4 words, i.e. of 16 bytes.  The
            // weights are read once: first out of L2
            asm volatile(
                "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
                "[%1, {%2, %3}], [%4], %5;" ::"r"(dst),
                "l"(m), "r"(kb0 * (kQ4KBlockBytes / 4)), "r"(static_cast<int>(fr.row0)), "r"(bar),
                "l"(l2_evict_first_policy())
                : "memory");
        }
    } else {
        const long long row_bytes_g = static_cast<long long>(p.nb) * kQ4KBlockBytes;
        const int rows = static_cast<int>(max(0LL, min(static_cast<long long>(kFxTileRows), fr.nrows - fr.row0)));
        const int nblk = min(kFxBPC, p.nb - kb0);
        const uint32_t bytes = static_cast<uint32_t>(nblk * kQ4KBlockBytes);
        if (lane == 0)
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * bytes);
        __syncwarp();
        if (lane < rows && !lost) {
            const uint8_t *src = fx_weights(p, fr.sel) + (fr.row0 + lane) * row_bytes_g +
                                 static_cast<long long>(kb0) * kQ4KBlockBytes;
            bulk_g2s_hint(dst + lane * kFxRowPitch, src, bytes, bar, l2_evict_first_policy());
        }
    }
}

// The slot at cursor cur (K-chunk c_begin + cur.kcl of stream cur.st of the
// tile at cur.row0) into ring slot `slot` of a warp's ring.
template <bool TMA>
__device__ __forceinline__ void fx_issue_slot(const Q4KParams &p, const FxMaps &maps, const Cursor &cur, int slot,
                                              int c_begin, uint32_t ring_s, uint32_t bars_s, int lane,
                                              bool lost = false)
{
    fx_issue_copy<TMA>(p, maps, cur.st, cur.row0, (c_begin + cur.kcl) * kFxBPC, ring_s + slot * kFxSlotBytes,
                       bars_s + slot * 8, lane, lost);
}

// R = 2: every warp owns a ring and its tiles.  R = 1: warps 2t and 2t + 1 own
// ring t and its tiles together, warp 2t + h reading rows 8h .. 8h + 7 of each
// slot; a counter per slot tells the second of the two to finish it, which
// refills it.
template <int NS, bool SOA, bool TMA, int R>
__global__ void __launch_bounds__((R == 2 ? kFxMaxWarps : kFxMaxPairWarps) * 32, 1)
    q4k_gemv_fx_kernel(const __grid_constant__ Q4KParams p, const __grid_constant__ FxMaps maps)
{
    static_assert(R == 1 || R == 2, "one or two rows per lane");
    constexpr int kTeam = 3 - R;   // warps per ring

    extern __shared__ __align__(128) uint8_t smem[];
    const int nwarps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nteams = nwarps / kTeam;
    const int team = warp / kTeam;
    const int half = warp % kTeam;       // R = 1: rows 8 half .. 8 half + 7 of each slot
    const int g = lane >> 3;             // super-block of each chunk
    const int i = lane & 7;
    const int srow = i + 8 * half;       // this lane's (first) row of each slot: rows srow + 8r, r < R

    // the splits of one CTA column are consecutive blocks (one cluster when the
    // splits are reduced in-kernel)
    const int split = blockIdx.x % p.splits;
    const int cj = blockIdx.x / p.splits;
    const int nchunk_total = (p.nb + kFxBPC - 1) / kFxBPC;
    const int c_begin = split * p.chunks_per_split;
    const int c_end = min(c_begin + p.chunks_per_split, nchunk_total);
    const int nch = c_end - c_begin;
    const int kb_begin = c_begin * kFxBPC;
    const int nbs = min(nch * kFxBPC, p.nb - kb_begin);  // super-blocks of this split

    // shared memory: [limb planes][sums and scales][barriers][ring][argmax scratch]
    // [cluster scratch], laid out for a full split in every CTA, so that each
    // part sits at the same offset in all CTAs of a cluster (a shorter last
    // split stages fewer super-blocks)
    const int x_bytes = (p.chunks_per_split * kFxBPC * (kFxLimbPitch + kFxAuxPitch) + 127) & ~127;
    uint8_t *limbs = smem;
    uint8_t *aux = smem + nbs * kFxLimbPitch;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + x_bytes);
    const int bar_bytes = (nwarps * p.depth * 8 + 127) & ~127;
    // TMA writes shared memory at 128-byte aligned addresses: align the ring
    const uint32_t ring_pad = (128u - ((smem_u32(smem) + x_bytes + bar_bytes) & 127u)) & 127u;
    uint8_t *ring = smem + x_bytes + bar_bytes + ring_pad;
    uint8_t *my_ring = ring + static_cast<size_t>(team) * p.depth * kFxSlotBytes;
    const uint32_t my_ring_s = smem_u32(my_ring);
    const uint32_t my_bars_s = smem_u32(bars + team * p.depth);
    // R = 1: per slot, how many times a warp of the pair has finished it (after the barriers)
    const uint32_t my_cnt_s = smem_u32(bars + nteams * p.depth) + team * p.depth * 4;
    ArgmaxCand *red = reinterpret_cast<ArgmaxCand *>(ring + static_cast<size_t>(nteams) * p.depth * kFxSlotBytes);
    // cluster reduction scratch of the rings this CTA finishes (ring t is
    // finished by rank t % splits, as its local ring t / splits): per local ring,
    // stream, source rank and tile row the fp64 partial sum, then its (error
    // bound, sum of |y_sb|)
    const int cl_rings = (nteams + p.splits - 1) / p.splits;
    double *cpart = reinterpret_cast<double *>(reinterpret_cast<uint8_t *>(red) + 256);
    float2 *cbnd = reinterpret_cast<float2 *>(cpart + cl_rings * 2 * p.splits * kFxTileRows);
    if (p.cluster)   // first phase of the cluster barrier: this CTA has started
        asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

    // this ring's tiles: t0, t0 + tstride, ... (ring-major order)
    const long long tstride = static_cast<long long>(p.ctas_per_split) * nteams;
    const long long t0 = static_cast<long long>(team) * p.ctas_per_split + cj;
    const long long ntiles_w = (t0 < p.tiles) ? (p.tiles - t0 + tstride - 1) / tstride : 0;
    const long long total = ntiles_w * NS * nch;
    const long long row_step = tstride * kFxTileRows;

    // after the quarter reduction (R = 2) lanes of quarters 0, 1 hold row i and
    // quarters 2, 3 row i + 8, and quarters 0 and 2 store; (R = 1) every
    // quarter holds row srow, and quarter 0 stores
    const bool writer = (R == 2) ? (lane & 8) == 0 : lane < 8;
    const int wrow = (R == 2) ? i + ((lane & 16) ? 8 : 0) : srow;

    Cursor pc{t0 * kFxTileRows, 0, 0};
    long long issued = 0;
    if (lane == 0 && half == 0) {
        for (int s = 0; s < p.depth; ++s) {
            mbar_init(my_bars_s + s * 8, 1);
            if (R == 1)
                st_shared_u32(my_cnt_s + s * 4, 0u);
        }
        mbar_fence_init();
        if (TMA && warp < (p.grp.n > 0 ? p.grp.n : NS))
            asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.m[warp]) : "memory");
    }
    __syncwarp();
    // the weights too may come from the previous kernel (a repack, an upload)
    pdl_wait();
    pdl_launch_dependents();
    FxXPre pre;
    fx_stage_load(p.x, kb_begin, nbs, warp, nwarps, lane, pre);
    // only the first slots before staging: the activation loads are not to
    // wait behind every SM's full ring of weight requests
    // (R = 1: the first warp of the pair issues, both follow the cursor)
    for (int s = 0; s < min(p.depth, kFxPreIssue) && issued < total; ++s, ++issued) {
        const bool lost = p.lost_copy && s == 0 && warp == 0 && blockIdx.x == 0;
        if (half == 0)
            fx_issue_slot<TMA>(p, maps, pc, s, c_begin, my_ring_s, my_bars_s, lane, lost);
        pc.advance(nch, NS, row_step);
    }

    fx_stage(p.x, kb_begin, nbs, limbs, aux, warp, nwarps, lane, pre, p.nb >= kFxMin3LimbBlocks);
    for (int s = static_cast<int>(issued); s < p.depth && issued < total; ++s, ++issued) {
        const bool lost = p.lost_copy && s == 0 && warp == 0 && blockIdx.x == 0;
        if (half == 0)
            fx_issue_slot<TMA>(p, maps, pc, s, c_begin, my_ring_s, my_bars_s, lane, lost);
        pc.advance(nch, NS, row_step);
    }
    __syncthreads();

    float best_v = -INFINITY;
    long long best_i = 0x7fffffffffffffffLL;
    bool failed = false;
    long long consumed = 0;
    double acc[R];
    float ebound[R], sabs[R];   // per row: error bound (rounded up), sum of |y_sb| (rounded down)
#pragma unroll
    for (int r = 0; r < R; ++r) {
        acc[r] = 0.0;
        ebound[r] = 0.f;
        sabs[r] = 0.f;
    }
    double gsum = 0.0;  // stream-0 sum kept for the SwiGLU epilogue
    float gE = 0.f, gS = 0.f;
    double csum = 0.0;  // cluster mode: the last stream's sum of the ring's one tile
    float cE = 0.f, cS = 0.f;

    Cursor cc{t0 * kFxTileRows, 0, 0};
    int slot = 0;
    uint32_t parity = 0;
    for (; consumed < total; ++consumed) {
        const bool ok = mbar_wait_bounded(my_bars_s + slot * 8, parity, p.err, p.wait_ns);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        const int kb0 = (c_begin + cc.kcl) * kFxBPC;
        const int nblk = min(kFxBPC, p.nb - kb0);
        fx_slot<R, SOA>(my_ring + slot * kFxSlotBytes, limbs + (kb0 - kb_begin) * kFxLimbPitch,
                        aux + (kb0 - kb_begin) * kFxAuxPitch, nblk, g, srow, acc, ebound, sabs);

        // every lane's reads of this slot are done (their values are used):
        // the slot may be refilled (R = 1: once both warps of the pair are done)
        __syncwarp();
        if (issued < total) {
            bool refill = true;
            if constexpr (R == 1) {
                uint32_t done = 0;
                if (lane == 0)
                    done = atom_add_acq_rel_shared_u32(my_cnt_s + slot * 4, 1u);
                refill = (__shfl_sync(0xffffffffu, done, 0) & 1u) != 0;
            }
            if (refill)
                fx_issue_slot<TMA>(p, maps, pc, slot, c_begin, my_ring_s, my_bars_s, lane);
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

        // end of this stream's K range for the tile: add the four quarters' sums
        double t;
        float te, ts;
        fx_quarter_rows<R>(acc, ebound, sabs, lane, t, te, ts);
        if constexpr (NS == 2) {
            if (cur_st == 0) {
                gsum = t;
                gE = te;
                gS = ts;
                continue;
            }
        }
        const long long n = row0 + wrow;
        if (p.cluster) {
            // the ring's only tile: its partials go to the cluster reduction
            csum = t;
            cE = te;
            cS = ts;
            continue;
        }
        if (p.splits > 1) {
            // partial sums and their bounds for the reduction kernel: planes of
            // [splits][NS][N] floats (sums, bounds rounded up, |y| sums rounded down)
            if (writer && n < p.N) {
                const long long P = static_cast<long long>(p.splits) * NS * p.N;
                const long long i0 = static_cast<long long>(split) * NS * p.N + n;
                if constexpr (NS == 2) {
                    p.part[i0] = static_cast<float>(gsum);
                    p.part[P + i0] = gE;
                    p.part[2 * P + i0] = gS;
                }
                const long long i1 = i0 + (NS - 1) * p.N;
                p.part[i1] = static_cast<float>(t);
                p.part[P + i1] = te;
                p.part[2 * P + i1] = ts;
            }
            continue;
        }
        // the whole K range is here: check each row's bound (a rare row is recomputed
        // exactly by the warp) and store
        const FxRows fr = fx_rows(p, 0, row0);
        const bool valid = writer && fr.row0 + wrow < fr.nrows;
        const long long row_bytes = static_cast<long long>(p.nb) * kQ4KBlockBytes;
        if constexpr (NS == 2)
            gsum = fx_fix_rows(gsum, gE, gS, valid, p.w[0] + (fr.row0 + wrow) * row_bytes, p.nb, p.soa, p.x);
        t = fx_fix_rows(t, te, ts, valid, fx_weights(p, NS == 2 ? 1 : fr.sel) + (fr.row0 + wrow) * row_bytes, p.nb,
                        p.soa, p.x);
        if (!valid)
            continue;
        if (p.grp.n > 0) {
            fx_group_out(p, fr.sel)[fr.row0 + wrow] = static_cast<float>(t);
            continue;
        }
        float out;
        if constexpr (NS == 2) {
            const float gv = static_cast<float>(gsum);
            out = gv / (1.0f + expf(-gv)) * static_cast<float>(t);
        } else {
            out = static_cast<float>(t);
            if (p.res)
                out += p.res[n];
        }
        *gemv_out_addr(p.y, p.g, p.qg_hd, p.N, 0, n) = out;
        if (p.argmax && cand_better(out, n, best_v, best_i)) {
            best_v = out;
            best_i = n;
        }
    }

    if (failed) {
        // the copies already issued into this warp's ring must land before the CTA exits
        for (long long k = consumed; k < issued; ++k) {
            mbar_wait_bounded(my_bars_s + slot * 8, parity, nullptr, p.wait_ns);
            if (++slot == p.depth) {
                slot = 0;
                parity ^= 1u;
            }
        }
    }

    if (p.cluster) {
        // Splits of a CTA column are one cluster and their rings hold the same
        // tiles: ring t's tile is finished (by the ring's first warp) in the CTA
        // of rank t % splits.  Every CTA stores its partials into that CTA's
        // shared memory, one cluster barrier makes them visible there, and the
        // finishing warp adds them in rank order 0, 1, ...
        namespace cg = cooperative_groups;
        cg::cluster_group cl = cg::this_cluster();
        // every CTA of the cluster has started (the first phase), so its shared
        // memory may be written
        asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
        const int fin = team % p.splits;
        const int lt = team / p.splits;
        if (writer && t0 < p.tiles && !failed) {
            double *rp = cl.map_shared_rank(cpart, fin);
            float2 *rb = cl.map_shared_rank(cbnd, fin);
            const int e0 = ((lt * 2 + 0) * p.splits + split) * kFxTileRows + wrow;
            rp[e0] = (NS == 2) ? gsum : csum;
            rb[e0] = (NS == 2) ? make_float2(gE, gS) : make_float2(cE, cS);
            if (NS == 2) {
                const int e1 = ((lt * 2 + 1) * p.splits + split) * kFxTileRows + wrow;
                rp[e1] = csum;
                rb[e1] = make_float2(cE, cS);
            }
        }
        cl.sync();
        if (fin == split && half == 0 && t0 < p.tiles) {
            // lane r < 16 finishes row r of the tile: partial sums in fp64, bounds
            // rounded outwards, in rank order
            double g = 0.0, u = 0.0;
            float ge = 0.f, gs = 0.f, ue = 0.f, us = 0.f;
            const int lr = lane & (kFxTileRows - 1);
            for (int r = 0; r < p.splits; ++r) {
                const int e0 = ((lt * 2 + 0) * p.splits + r) * kFxTileRows + lr;
                const float2 b0 = cbnd[e0];
                g += cpart[e0];
                ge = __fadd_ru(ge, b0.x);
                gs = __fadd_rd(gs, b0.y);
                if (NS == 2) {
                    const int e1 = ((lt * 2 + 1) * p.splits + r) * kFxTileRows + lr;
                    const float2 b1 = cbnd[e1];
                    u += cpart[e1];
                    ue = __fadd_ru(ue, b1.x);
                    us = __fadd_rd(us, b1.y);
                }
            }
            const long long n = t0 * kFxTileRows + lane;
            const FxRows fr = fx_rows(p, 0, t0 * kFxTileRows);
            const bool valid = lane < kFxTileRows && fr.row0 + lane < fr.nrows;
            const long long row_bytes = static_cast<long long>(p.nb) * kQ4KBlockBytes;
            const long long wr = (fr.row0 + lr) * row_bytes;
            g = fx_fix_rows(g, ge, gs, valid, fx_weights(p, fr.sel) + wr, p.nb, p.soa, p.x);
            if constexpr (NS == 2)
                u = fx_fix_rows(u, ue, us, valid, p.w[1] + wr, p.nb, p.soa, p.x);
            if (valid && p.grp.n > 0) {
                fx_group_out(p, fr.sel)[fr.row0 + lane] = static_cast<float>(g);
            } else if (valid) {
                float out;
                if constexpr (NS == 2) {
                    const float gv = static_cast<float>(g);
                    out = gv / (1.0f + expf(-gv)) * static_cast<float>(u);
                } else {
                    out = static_cast<float>(g);
                    if (p.res)
                        out += p.res[n];
                }
                *gemv_out_addr(p.y, p.g, p.qg_hd, p.N, 0, n) = out;
                if (p.argmax && cand_better(out, n, best_v, best_i)) {
                    best_v = out;
                    best_i = n;
                }
            }
        }
    }

    if (p.argmax && (p.splits == 1 || p.cluster)) {
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
// Batches of 2..8 activation rows: the same quarter-warp lanes, TMA slots and
// rings, with exact fp32 weights (q4k_decode.cuh: formed once per weight, used
// B times) and fp32 accumulation.  x is staged in fp32 (lo, hi) pairs; each
// quarter-warp reads its super-block's pairs as a broadcast.
// ---------------------------------------------------------------------------

// Sums the values of the four quarter-warps (lanes i, i+8, i+16, i+24) with a
// transposing butterfly over lane bits 4 and 3: on entry every lane holds M
// values (M a multiple of 4); on exit it holds the totals of indices
// off .. off + M/4 - 1, off = (bit 4 ? M/2 : 0) + (bit 3 ? M/4 : 0).
template <int M>
__device__ __forceinline__ void quarter_sum(float (&v)[M], int lane)
{
    static_assert(M % 4 == 0, "four quarter-warps share the values");
    const bool up16 = (lane & 16) != 0;
#pragma unroll
    for (int k = 0; k < M / 2; ++k) {
        const float send = up16 ? v[k] : v[k + M / 2];
        const float keep = up16 ? v[k + M / 2] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    const bool up8 = (lane & 8) != 0;
#pragma unroll
    for (int k = 0; k < M / 4; ++k) {
        const float send = up8 ? v[k] : v[k + M / 4];
        const float keep = up8 ? v[k + M / 4] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
}

constexpr int kFxbMaxWarps(int B) { return B <= 2 ? 12 : 8; }

// Chunks of K per split at batches 2-8.  A lane's four fp32 accumulators per
// (row, batch row) each take 64 products per chunk, so a split adds at most
// 1024 products into one; with the few additions after that (the quarter-warp
// sum, the splits), the recursive-summation bound stays below
// 1100 * 2^-24 ~ 6.6e-5 of sum |w x|, inside the 1e-4 contract for any K.
constexpr int kFxbMaxChunks = 16;

template <int B, int NS, bool SOA, bool TMA>
__global__ void __launch_bounds__(kFxbMaxWarps(B) * 32, 1)
    q4k_gemv_fxb_kernel(const __grid_constant__ Q4KParams p, const __grid_constant__ FxMaps maps)
{
    constexpr int R = kFxRows;
    constexpr int MV = R * B;                 // values per lane per stream (index r*B + b)
    constexpr int MP = (MV + 3) / 4 * 4;      // padded for the quarter-warp butterfly
    constexpr int VPL = MP / 4;               // values per lane after it
    static_assert(R == 2 && B >= 2 && B <= 8, "two rows per lane, batches of 2 to 8");

    extern __shared__ __align__(128) uint8_t smem[];
    const int nwarps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 3;   // super-block of each chunk
    const int i = lane & 7;    // rows i and i + 8 of each tile
    const int voff = ((lane & 16) ? MP / 2 : 0) + ((lane & 8) ? MP / 4 : 0);

    const int split = blockIdx.x / p.ctas_per_split;
    const int cj = blockIdx.x % p.ctas_per_split;
    const int nchunk_total = (p.nb + kFxBPC - 1) / kFxBPC;
    const int c_begin = split * p.chunks_per_split;
    const int c_end = min(c_begin + p.chunks_per_split, nchunk_total);
    const int nch = c_end - c_begin;
    const int kb_begin = c_begin * kFxBPC;
    const int nbs = min(nch * kFxBPC, p.nb - kb_begin);

    // shared memory: [x pairs][barriers][ring]
    const int x_bytes = (B * nbs * kXBlockPitch + 127) & ~127;
    uint8_t *xs = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + x_bytes);
    const int bar_bytes = (nwarps * p.depth * 8 + 127) & ~127;
    const uint32_t ring_pad = (128u - ((smem_u32(smem) + x_bytes + bar_bytes) & 127u)) & 127u;
    uint8_t *ring = smem + x_bytes + bar_bytes + ring_pad;
    uint8_t *my_ring = ring + static_cast<size_t>(warp) * p.depth * kFxSlotBytes;
    const uint32_t my_ring_s = smem_u32(my_ring);
    const uint32_t my_bars_s = smem_u32(bars + warp * p.depth);

    const long long tstride = static_cast<long long>(p.ctas_per_split) * nwarps;
    const long long t0 = static_cast<long long>(warp) * p.ctas_per_split + cj;
    const long long ntiles_w = (t0 < p.tiles) ? (p.tiles - t0 + tstride - 1) / tstride : 0;
    const long long total = ntiles_w * NS * nch;
    const long long row_step = tstride * kFxTileRows;

    Cursor pc{t0 * kFxTileRows, 0, 0};
    long long issued = 0;
    if (lane == 0) {
        for (int s = 0; s < p.depth; ++s)
            mbar_init(my_bars_s + s * 8, 1);
        mbar_fence_init();
    }
    __syncwarp();
    pdl_wait();
    pdl_launch_dependents();
    for (int s = 0; s < p.depth && issued < total; ++s, ++issued) {
        fx_issue_slot<TMA>(p, maps, pc, s, c_begin, my_ring_s, my_bars_s, lane);
        pc.advance(nch, NS, row_step);
    }

    stage_x_pairs<(B <= 2) ? 4 : 1>(p.x, p.K, B, kb_begin, nbs, xs);
    __syncthreads();

    bool failed = false;
    long long consumed = 0;
    float2 acc0[R][B], acc1[R][B];
    float gsum[NS == 2 ? VPL : 1];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) {
            acc0[r][b] = f2(0.f, 0.f);
            acc1[r][b] = f2(0.f, 0.f);
        }

    Cursor cc{t0 * kFxTileRows, 0, 0};
    int slot = 0;
    uint32_t parity = 0;
    for (; consumed < total; ++consumed) {
        const bool ok = mbar_wait_bounded(my_bars_s + slot * 8, parity, p.err, p.wait_ns);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        const int kb0 = (c_begin + cc.kcl) * kFxBPC;
        const int nblk = min(kFxBPC, p.nb - kb0);
        if (g < nblk) {
            const uint8_t *slot_p = my_ring + slot * kFxSlotBytes + i * kFxRowPitch;
            const BlockOffsets bo = block_offsets<SOA>(g, nblk);
            Hdr hd[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                hd[r] = decode_hdr(*reinterpret_cast<const uint4 *>(slot_p + 8 * r * kFxRowPitch + bo.hdr));
            const uint8_t *xblk = xs + (kb0 - kb_begin + g) * kXBlockPitch;
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
                        q[r] = *reinterpret_cast<const uint4 *>(slot_p + 8 * r * kFxRowPitch + bo.qs0 +
                                                                s * bo.qs_step);
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

        // every lane's reads of this slot are done (their values are used):
        // the slot may be refilled
        __syncwarp();
        if (issued < total) {
            fx_issue_slot<TMA>(p, maps, pc, slot, c_begin, my_ring_s, my_bars_s, lane);
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

        // end of this stream's K range for the tile: add the four quarters' sums
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
        for (int k = MV; k < MP; ++k)
            v[k] = 0.f;
        quarter_sum<MP>(v, lane);
        if constexpr (NS == 2) {
            if (cur_st == 0) {
#pragma unroll
                for (int k = 0; k < VPL; ++k)
                    gsum[k] = v[k];
                continue;
            }
        }
#pragma unroll
        for (int k = 0; k < VPL; ++k) {
            const int idx = voff + k;
            if (idx >= MV)
                continue;
            const int r = idx / B;
            const int b = idx % B;
            const long long n = row0 + i + 8 * r;
            if (n >= p.N)
                continue;
            if (p.splits > 1) {
                if constexpr (NS == 2) {
                    p.part[((static_cast<long long>(split) * 2 + 0) * B + b) * p.N + n] = gsum[k] * 0x1p64f;
                    p.part[((static_cast<long long>(split) * 2 + 1) * B + b) * p.N + n] = v[k] * 0x1p64f;
                } else {
                    p.part[(static_cast<long long>(split) * B + b) * p.N + n] = v[k] * 0x1p64f;
                }
            } else {
                float out;
                if constexpr (NS == 2) {
                    const float gv = gsum[k] * 0x1p64f;
                    out = gv / (1.0f + expf(-gv)) * (v[k] * 0x1p64f);
                } else {
                    out = v[k] * 0x1p64f;
                    if (p.res)
                        out += p.res[static_cast<long long>(b) * p.N + n];
                }
                *gemv_out_addr(p.y, p.g, p.qg_hd, p.N, b, n) = out;
            }
        }
    }

    if (failed) {
        // the copies already issued into this warp's ring must land before the CTA exits
        for (long long k = consumed; k < issued; ++k) {
            mbar_wait_bounded(my_bars_s + slot * 8, parity, nullptr, p.wait_ns);
            if (++slot == p.depth) {
                slot = 0;
                parity ^= 1u;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Warps per CTA for `tiles` row tiles on `sm_count` SMs (one CTA per SM):
// enough to give every SM work and at least one per scheduler.
static int pick_warps(long long tiles, int sm_count, int max_warps)
{
    long long w = (tiles + sm_count - 1) / sm_count;
    if (w < 4)
        w = 4;
    if (w > max_warps)
        w = max_warps;
    return static_cast<int>(w);
}

// The driver's tensor-map encoder, looked up once (null when unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

// How many clusters of `size` CTAs of the batch-1 kernel (warps x 32 threads,
// smem bytes of shared memory each, R rows per lane) the device runs at once; 0
// when the runtime cannot tell.  Cached per shape.
static int cluster_capacity(int size, int warps, int smem, int R)
{
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, int>, int> cache;
    const auto key = std::make_tuple(size, warps, smem, R);
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(key);
    if (it != cache.end())
        return it->second;
    auto k = R == 1 ? q4k_gemv_fx_kernel<1, false, true, 1> : q4k_gemv_fx_kernel<1, false, true, 2>;
    int n = 0;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(size);
        cfg.blockDim = dim3(warps * 32);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = size;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess)
            n = 0;
    }
    cudaGetLastError();
    cache[key] = n;
    return n;
}

// Launch plan.  Slot copies by TMA when the driver's encoder is available.  K
// is split until there are about eight tile tasks per SM (or each split is one
// chunk), warps per CTA follow from the tasks per SM (batch 1) or from covering
// the tiles with whole groups of four warps (batches 2-8), and K is split further
// if the activations would not fit beside a two-deep ring per warp; the ring
// is as deep as shared memory allows, up to 4 slots.  When the batch-1 splits
// are added inside clusters, all clusters must be resident at once: the plan
// then takes the fewest warps per CTA (the most CTAs, hence SMs) whose clusters
// fit in one wave, and gives up the clusters if none does.  At batch 1, rings
// that would hold at most kFxPairMaxSlots slots are owned by pairs of warps
// (R = 1), when the CTA has room for twice the warps.
static Q4KPlan plan_quarter_warp(long long N, int nb, int B, int NS, int sm_count, int smem_optin)
{
    // DQGEMV_NO_TMA=1 selects the per-row bulk copies (same shared-memory
    // layout, bit-identical results), for comparing the two copy paths
    const char *no_tma = getenv("DQGEMV_NO_TMA");
    const bool tma = N < 0x7FFFFFFFLL && tensor_map_encoder() != nullptr && !(no_tma && no_tma[0] == '1');
    const int misc = 256 /*argmax scratch, 16 B per warp*/ + 512 /*barriers*/ + 128 /*ring alignment*/;
    // staged activations per super-block: limb planes and sums (batch 1), or B
    // rows of fp32 pairs
    const int stage = (B == 1) ? kFxLimbPitch + kFxAuxPitch : B * kXBlockPitch;
    const int max_warps = (B == 1) ? kFxMaxWarps : kFxbMaxWarps(B);
    const long long tiles = (N + kFxTileRows - 1) / kFxTileRows;
    const int nchunk = (nb + kFxBPC - 1) / kFxBPC;
    int splits_par = 1;
    while (tiles * splits_par < 8LL * sm_count && splits_par < nchunk)
        ++splits_par;
    auto plan_for = [&](int warps, bool allow_cluster) {
        Q4KPlan pl{};
        int splits = splits_par;
        // batches 2-8 sum fp32 products: at most kFxbMaxChunks chunks per split
        // keeps each accumulator to 64 * kFxbMaxChunks products
        if (B > 1 && (nchunk + splits - 1) / splits > kFxbMaxChunks)
            splits = (nchunk + kFxbMaxChunks - 1) / kFxbMaxChunks;
        int cps = (nchunk + splits - 1) / splits;
        while (cps * kFxBPC * stage + warps * 2 * kFxSlotBytes + misc > smem_optin && cps > 1) {
            ++splits;
            cps = (nchunk + splits - 1) / splits;
        }
        splits = (nchunk + cps - 1) / cps;
        const int x_bytes = (cps * kFxBPC * stage + 127) & ~127;
        int depth = (smem_optin - x_bytes - misc) / (warps * kFxSlotBytes);
        if (depth > 4)
            depth = 4;
        if (depth < 2)
            return pl;
        long long ctas = (tiles + warps - 1) / warps;
        const long long max_ctas = sm_count / splits > 0 ? sm_count / splits : 1;
        if (ctas > max_ctas)
            ctas = max_ctas;
        // `warps` rings; each owned by two warps when it holds few slots
        const long long ring_slots = (tiles + ctas * warps - 1) / (ctas * warps) * NS * cps;
        const int team = (B == 1 && 2 * warps <= kFxMaxPairWarps && ring_slots <= kFxPairMaxSlots) ? 2 : 1;
        pl.tma = tma;
        pl.R = team == 2 ? 1 : kFxRows;
        pl.warps = warps * team;
        pl.tiles = tiles;
        pl.splits = splits;
        pl.chunks_per_split = cps;
        pl.depth = depth;
        pl.ctas_per_split = static_cast<int>(ctas);
        pl.grid = pl.ctas_per_split * splits;
        // barriers (and R = 1 refill counters) are sized for 8 bytes per warp and slot
        pl.smem = x_bytes + ((pl.warps * depth * 8 + 127) & ~127) + 128 + warps * depth * kFxSlotBytes + 256;
        // batch-1 splits of at most one tile per warp are added inside a cluster
        // (each CTA finishes the tiles of every splits-th ring and holds the
        // partials of all splits for them)
        const int cl_bytes = (warps + splits - 1) / splits * splits * kFxClusterPartBytes;
        pl.cluster = allow_cluster && B == 1 && splits > 1 && splits <= kFxMaxCluster &&
                     tiles <= static_cast<long long>(pl.ctas_per_split) * warps && pl.smem + cl_bytes <= smem_optin;
        if (pl.cluster)
            pl.smem += cl_bytes;
        pl.ok = pl.smem <= smem_optin;
        return pl;
    };
    // Warps per CTA to start from.  Batch 1: from the tile tasks per SM.  Batches 2-8 (one tile per
    // warp and the same work per tile): the fewest warps, in multiples of four (one per scheduler),
    // whose CTAs cover every tile on the SMs left to each split once the splits are whole numbers of
    // chunks; a count that is not a multiple of four leaves one scheduler with an extra tile.
    int w_start = pick_warps(tiles * splits_par, sm_count, max_warps);
    if (B > 1) {
        const int cps0 = (nchunk + splits_par - 1) / splits_par;
        const int splits_eff = (nchunk + cps0 - 1) / cps0;
        const long long per_split = sm_count / splits_eff > 0 ? sm_count / splits_eff : 1;
        w_start = max_warps;
        for (int w = 4; w <= max_warps; w += 4)
            if ((tiles + w - 1) / w <= per_split) {
                w_start = w;
                break;
            }
    }
    auto first_fit = [&](bool allow_cluster) {
        Q4KPlan pl{};
        for (int warps = w_start; warps >= 4 && !pl.ok; --warps)
            pl = plan_for(warps, allow_cluster);
        return pl;
    };
    Q4KPlan pl = first_fit(true);
    if (pl.ok && pl.cluster) {
        const int cap = cluster_capacity(pl.splits, pl.warps, pl.smem, pl.R);
        if (cap > 0) {
            for (int warps = 4; warps <= max_warps; ++warps) {
                const Q4KPlan c = plan_for(warps, true);
                if (c.ok && c.cluster && c.ctas_per_split <= cluster_capacity(c.splits, c.warps, c.smem, c.R))
                    return c;
            }
            if (pl.ctas_per_split > cap)
                pl = first_fit(false);
        }
    }
    return pl;
}

// Describes one weight matrix to the TMA unit as [N][row bytes / 4] 32-bit words
// with a box of one slot: 16 rows x (576 + 16) bytes.
static cudaError_t encode_weight_map(CUtensorMap *m, const uint8_t *w, long long N, int nb)
{
    const cuuint64_t row = static_cast<cuuint64_t>(nb) * kQ4KBlockBytes;
    const cuuint64_t dims[2] = {row / 4, static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {row};
    const cuuint32_t box[2] = {kFxRowPitch / 4, kFxTileRows};
    const cuuint32_t es[2] = {1, 1};
    const CUresult r = tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t *>(w), dims,
                                            strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int NS, bool TMA>
static cudaError_t launch_fx(const Q4KParams &p, const FxMaps &maps, const Q4KPlan &pl, cudaStream_t s)
{
    auto k = pl.R == 1 ? (p.soa ? q4k_gemv_fx_kernel<NS, true, TMA, 1> : q4k_gemv_fx_kernel<NS, false, TMA, 1>)
                       : (p.soa ? q4k_gemv_fx_kernel<NS, true, TMA, 2> : q4k_gemv_fx_kernel<NS, false, TMA, 2>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess)
        return e;
    if (!pl.cluster)
        return launch_pdl(k, dim3(pl.grid), dim3(pl.warps * 32), pl.smem, s, p, maps);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(pl.warps * 32);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = pl.splits;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k, p, maps);
}

template <int B, int NS, bool TMA>
static cudaError_t launch_fxb(const Q4KParams &p, const FxMaps &maps, const Q4KPlan &pl, cudaStream_t s)
{
    auto k = p.soa ? q4k_gemv_fxb_kernel<B, NS, true, TMA> : q4k_gemv_fxb_kernel<B, NS, false, TMA>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(k, dim3(pl.grid), dim3(pl.warps * 32), pl.smem, s, p, maps);
}

template <int NS, bool TMA>
static cudaError_t launch_fx_b(const Q4KParams &p, const FxMaps &maps, const Q4KPlan &pl, int B, cudaStream_t s)
{
    switch (B) {
    case 1: return launch_fx<NS, TMA>(p, maps, pl, s);
    case 2: return launch_fxb<2, NS, TMA>(p, maps, pl, s);
    case 3: return launch_fxb<3, NS, TMA>(p, maps, pl, s);
    case 4: return launch_fxb<4, NS, TMA>(p, maps, pl, s);
    case 5: return launch_fxb<5, NS, TMA>(p, maps, pl, s);
    case 6: return launch_fxb<6, NS, TMA>(p, maps, pl, s);
    case 7: return launch_fxb<7, NS, TMA>(p, maps, pl, s);
    case 8: return launch_fxb<8, NS, TMA>(p, maps, pl, s);
    default: return cudaErrorInvalidValue;
    }
}

Q4KPlan q4k_plan(long long N, int K, int B, int NS, int soa, int sm_count, int smem_optin)
{
    (void)soa;   // both layouts move 4-block chunks as one contiguous span per row
    return plan_quarter_warp(N, K / kQ4KBlockElems, B, NS, sm_count, smem_optin);
}

cudaError_t q4k_gemv_launch(const Q4KParams &p, const Q4KPlan &pl, int B, int NS, cudaStream_t s)
{
    FxMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (pl.tma) {
        if (p.grp.n > 0) {
            for (int m = 0; m < p.grp.n; ++m) {
                const cudaError_t e = encode_weight_map(&maps.m[m], p.gw[m], p.grp.N[m], p.nb);
                if (e != cudaSuccess)
                    return e;
            }
        } else {
            for (int st = 0; st < NS; ++st) {
                const cudaError_t e = encode_weight_map(&maps.m[st], p.w[st], p.N, p.nb);
                if (e != cudaSuccess)
                    return e;
            }
        }
        return NS == 1 ? launch_fx_b<1, true>(p, maps, pl, B, s) : launch_fx_b<2, true>(p, maps, pl, B, s);
    }
    return NS == 1 ? launch_fx_b<1, false>(p, maps, pl, B, s) : launch_fx_b<2, false>(p, maps, pl, B, s);
}

}  // namespace dq
