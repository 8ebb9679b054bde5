// q4k_stream.cuh -- helpers of the Q4_K GEMV's slot streaming: where a
// super-block's header and quant slices sit inside a K-chunk of a row (both
// layouts), and the per-warp slot cursor.
//
// A warp owns a set of row tiles.  One "slot" is one K-chunk of one tile of one
// weight stream.  Each warp streams its own ring of `depth` slots: copies from
// this GPU's global memory land in the warp's shared-memory slot and complete
// on an mbarrier, the whole warp computes on the oldest slot, and the slot is
// refilled with the one `depth` steps ahead.
#pragma once

#include <cstdint>

#include "dq_common.cuh"
#include "dq_internal.h"

namespace dq {

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

}  // namespace dq
