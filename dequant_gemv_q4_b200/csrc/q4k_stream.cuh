// q4k_stream.cuh -- the streaming machinery shared by the Q4_K GEMV kernels:
// slot geometry, per-warp slot cursors, bulk-copy issue of one slot, and the
// row-group butterfly reduction.
//
// A warp owns a set of row tiles.  A row tile is TR = (32/LPR)*R rows; lane
// (rg, l) = (lane / LPR, lane % LPR) handles rows rg*R .. rg*R+R-1 of the tile.
// One "slot" is one K-chunk of one tile of one weight stream.  Each warp
// streams its own ring of `depth` slots: lane 0 issues 1-D bulk copies
// (cp.async.bulk from this GPU's global memory into the warp's shared-memory
// slot, completing on an mbarrier), the whole warp computes on the oldest slot
// and lane 0 reuses it for the slot `depth` steps ahead.
#pragma once

#include <cstdint>

#include "dq_common.cuh"
#include "dq_internal.h"

namespace dq {

constexpr int kMaxWarps = 8;

// Slot geometry.  LPR lanes per row group, RG = 32/LPR row groups per warp, R
// rows per lane, BPC super-blocks per K-chunk.  A slot is TR = RG*R rows x BPC
// super-blocks; rows of a row group are contiguous, row groups RG_PITCH apart.
//   Geo     ("full-block" lanes): lane l owns super-block l of each chunk (BPC = LPR).
//   GeoHalf ("half-block" lanes): lane l owns chunks 2(l%2), 2(l%2)+1 of super-block
//           l/2 of each chunk (BPC = LPR/2), so a slot is half as large.
template <int LPR, int RR>
struct Geo {
    static constexpr int R = RR;
    static constexpr int RG = 32 / LPR;
    static constexpr int TR = RG * R;
    static constexpr int BPC = LPR;
    static constexpr int ROW_BYTES = BPC * kQ4KBlockBytes;
    static constexpr int PAD = (LPR < 8) ? 64 : 0;            // bank-shift between row groups
    static constexpr int RG_PITCH = R * ROW_BYTES + PAD;
    static constexpr int SLOT_BYTES = RG * RG_PITCH;
    static_assert(SLOT_BYTES % 128 == 0, "slot must keep 128-byte alignment");
};

template <int LPR>
struct GeoHalf {
    static constexpr int RG = 32 / LPR;
    static constexpr int R = 2;
    static constexpr int TR = RG * R;
    static constexpr int BPC = LPR / 2;
    static constexpr int ROW_BYTES = BPC * kQ4KBlockBytes;
    static constexpr int PAD = 0;
    static constexpr int RG_PITCH = R * ROW_BYTES;
    static constexpr int SLOT_BYTES = RG * RG_PITCH;
    static_assert(LPR == 32 || LPR == 8, "half-block lanes are laid out for 32 or 8 lanes per row group");
    static_assert(SLOT_BYTES % 128 == 0, "slot must keep 128-byte alignment");
};

// Transposing butterfly over the LPR lanes of a row group: on entry each lane
// holds M partial values; on exit lane l holds the sums of a contiguous run of
// value indices (the kernel recomputes which).  M is a power of two.
template <int O, int M, class T = float>
struct GroupReduce {
    static __device__ __forceinline__ void run(T *v, int lane)
    {
        if constexpr (M > 1) {
            const bool up = (lane & O) != 0;
#pragma unroll
            for (int i = 0; i < M / 2; ++i) {
                const T send = up ? v[i] : v[i + M / 2];
                const T keep = up ? v[i + M / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
            }
            if constexpr (O > 1)
                GroupReduce<O / 2, M / 2, T>::run(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
            if constexpr (O > 1)
                GroupReduce<O / 2, 1, T>::run(v, lane);
        }
    }
};

template <int N>
struct Pow2Ceil {
    static constexpr int value = (N <= 1) ? 1 : 2 * Pow2Ceil<(N + 1) / 2>::value;
};
template <>
struct Pow2Ceil<1> {
    static constexpr int value = 1;
};

// Byte offsets, within one row of a K-chunk of nblk super-blocks that starts
// at an SoA group boundary, of super-block t's 16-byte header and of its first
// quant slice, and the distance between its slices.
struct BlockOffsets {
    int hdr;
    int qs0;
    int qs_step;
};
template <bool SOA>
__device__ __forceinline__ BlockOffsets block_offsets(int t, int nblk)
{
    if constexpr (SOA) {
        const int grp = t / kQ4KSoaGroup;
        const int tt = t % kQ4KSoaGroup;
        const int gsz = min(kQ4KSoaGroup, nblk - grp * kQ4KSoaGroup);
        const int base = grp * kQ4KSoaGroup * kQ4KBlockBytes;
        return {base + 16 * tt, base + 16 * gsz + 16 * tt, 16 * gsz};
    } else {
        return {kQ4KBlockBytes * t, kQ4KBlockBytes * t + 16, 16};
    }
}

// Position of a warp in its slot sequence: the tile's first row row0, weight
// stream st, K-chunk kcl (relative to the split's first chunk).  row0 moves by
// the warp's tile stride once every stream and chunk of a tile are done.
struct Cursor {
    long long row0;
    int st;
    int kcl;
    __device__ __forceinline__ bool advance(int nch, int ns, long long row_step)
    {
        if (++kcl == nch) {
            kcl = 0;
            if (++st == ns) {
                st = 0;
                row0 += row_step;
                return true;
            }
        }
        return false;
    }
};

// Issues the bulk copies of one slot (K-chunk c_begin + cur.kcl of stream
// cur.st of the tile at cur.row0) into ring slot `slot`.
template <class G>
__device__ __forceinline__ void issue_slot(const Q4KParams &p, const Cursor &cur, int slot, int c_begin,
                                           uint32_t ring_s, uint32_t bars_s)
{
    const long long row_bytes_g = static_cast<long long>(p.nb) * kQ4KBlockBytes;
    const int rows = static_cast<int>(min(static_cast<long long>(G::TR), p.N - cur.row0));
    const int kb0 = (c_begin + cur.kcl) * G::BPC;
    const int nblk = min(G::BPC, p.nb - kb0);
    const uint8_t *src = (cur.st == 0 ? p.w[0] : p.w[1]) + cur.row0 * row_bytes_g + kb0 * kQ4KBlockBytes;
    const uint32_t dst = ring_s + slot * G::SLOT_BYTES;
    const uint32_t bar = bars_s + slot * 8;
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows * nblk * kQ4KBlockBytes));
    if (nblk == p.nb && p.nb == G::BPC) {
        if (G::PAD == 0) {
            // whole rows of a contiguous tile, laid out without padding: one copy
            bulk_g2s(dst, src, static_cast<uint32_t>(rows * G::ROW_BYTES), bar);
        } else {
            for (int g = 0; g * G::R < rows; ++g) {
                const int gr = min(G::R, rows - g * G::R);
                bulk_g2s(dst + g * G::RG_PITCH, src + static_cast<long long>(g) * G::R * row_bytes_g,
                         static_cast<uint32_t>(gr * G::ROW_BYTES), bar);
            }
        }
    } else {
        for (int r = 0; r < rows; ++r)
            bulk_g2s(dst + (r / G::R) * G::RG_PITCH + (r % G::R) * G::ROW_BYTES, src + r * row_bytes_g,
                     static_cast<uint32_t>(nblk * kQ4KBlockBytes), bar);
    }
}

}  // namespace dq
