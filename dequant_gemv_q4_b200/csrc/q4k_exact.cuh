// q4k_exact.cuh -- the batch-1 GEMV's rigorous fallback: one row of a Q4_K
// GEMV recomputed with the exact weights in fp64.
//
// The batch-1 kernels round activations to a fixed point shared by each
// super-block (q4k_gemv.cu) and carry, per output row, an upper bound on the
// error that rounding caused and a lower bound on sum_k |w_k x_k|.  When the
// bound cannot show the GEMV contract |y - y_exact| <= 1e-4 sum |w x| + 1e-6
// (only on activations whose range inside a super-block is extreme AND whose
// large values meet near-zero weights), the row is recomputed here: every
// weight d*scale*q - dmin*min is exact in fp64 (all terms are multiples of
// 2^-24 below 2^26, i.e. at most 50 significant bits), each product with x is
// rounded once, and the sum is taken in fp64.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "dq_common.cuh"
#include "q4k_stream.cuh"

namespace dq {

// Offsets of super-block kb's header and quant slices within a row of nb
// super-blocks, in the AoS or the SoA layout.
__device__ __forceinline__ BlockOffsets row_block_offsets(int kb, int nb, bool soa)
{
    if (soa) {
        const int first = kb / kQ4KSoaGroup * kQ4KSoaGroup;
        const int gs = min(kQ4KSoaGroup, nb - first);
        const int t = kb - first;
        const int base = first * kQ4KBlockBytes;
        return {base + 16 * t, base + 16 * gs + 16 * t, 16 * gs};
    }
    return {kb * kQ4KBlockBytes, kb * kQ4KBlockBytes + 16, 16};
}

// sum_k W[k] x[k] over one row (wrow: its nb super-blocks) with exact weights,
// in fp64.  Called by all 32 lanes of a warp: the row's 16-byte quant slices
// (32 weights each) are spread over the lanes; every lane returns the same sum,
// added in a fixed order.
static __device__ __noinline__ double q4k_exact_row(const uint8_t *wrow, int nb, int soa, const float *x)
{
    const int lane = threadIdx.x & 31;
    double acc = 0.0;
    for (int u = lane; u < nb * 8; u += 32) {
        const int kb = u >> 3, s = u & 7;
        const BlockOffsets bo = row_block_offsets(kb, nb, soa != 0);
        const uint4 h = __ldg(reinterpret_cast<const uint4 *>(wrow + bo.hdr));
        const double d = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(h.x & 0xFFFFu))));
        const double dm = static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(h.x >> 16))));
        // get_scale_min_k4 fields, four per word (one per byte)
        const uint32_t scw[2] = {h.y & 0x3F3F3F3Fu, (h.w & 0x0F0F0F0Fu) | ((h.y >> 2) & 0x30303030u)};
        const uint32_t mnw[2] = {h.z & 0x3F3F3F3Fu, ((h.w >> 4) & 0x0F0F0F0Fu) | ((h.z >> 2) & 0x30303030u)};
        // slice s holds bytes 16(s%2) .. 16(s%2)+15 of chunk c = s/2: low nibbles are
        // weights 64c + r of sub-block 2c, high nibbles 64c + 32 + r of sub-block 2c+1
        const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(wrow + bo.qs0 + s * bo.qs_step));
        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
        const int c = s >> 1;
        const int jl = 2 * c, jh = 2 * c + 1;
        const double al = d * static_cast<double>((scw[jl >> 2] >> (8 * (jl & 3))) & 0xFFu);
        const double bl = dm * static_cast<double>((mnw[jl >> 2] >> (8 * (jl & 3))) & 0xFFu);
        const double ah = d * static_cast<double>((scw[jh >> 2] >> (8 * (jh & 3))) & 0xFFu);
        const double bh = dm * static_cast<double>((mnw[jh >> 2] >> (8 * (jh & 3))) & 0xFFu);
        const float *xl = x + static_cast<long long>(kb) * kQ4KBlockElems + 64 * c + 16 * (s & 1);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            // x through L2 (it may have been written earlier in the same kernel)
            const float4 xa = __ldcg(reinterpret_cast<const float4 *>(xl + 4 * v));
            const float4 xb = __ldcg(reinterpret_cast<const float4 *>(xl + 32 + 4 * v));
            const float xlo[4] = {xa.x, xa.y, xa.z, xa.w};
            const float xhi[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint32_t byte = (qw[v] >> (8 * t)) & 0xFFu;
                const double wl = al * static_cast<double>(byte & 15u) - bl;   // exact
                const double wh = ah * static_cast<double>(byte >> 4) - bh;     // exact
                acc = fma(wl, static_cast<double>(xlo[t]), acc);
                acc = fma(wh, static_cast<double>(xhi[t]), acc);
            }
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// The rigorous check of a batch-1 row sum t with error bound E (rounded up)
// and S <= sum_k |w_k x_k| (rounded down): true when the fixed-point result is
// already within the contract.  With the other roundings (fp64 combine, fp32
// partials and output, each below 2^-23 S) it needs
//   E (1 + 1e-4) <= (1e-4 - 2^-22) S + 1e-6.
__device__ __forceinline__ bool fx_bound_ok(float E, float S)
{
    return __fmul_ru(E, 1.0001f) <= __fmaf_rd(9.99e-5f, S, 0.999e-6f);
}

// For the lanes holding a row (valid) whose sum t fails fx_bound_ok, the warp
// recomputes the row exactly; wrow is that lane's row.  Non-finite sums (an
// infinity or a NaN in x) are left as they are.  All 32 lanes must call it.
__device__ __forceinline__ double fx_fix_rows(double t, float E, float S, bool valid, const uint8_t *wrow, int nb,
                                              int soa, const float *x)
{
    const bool redo = valid && isfinite(t) && !fx_bound_ok(E, S);
    unsigned fail = __ballot_sync(0xffffffffu, redo);
    while (fail != 0) {
        const int src = __ffs(fail) - 1;
        fail &= fail - 1;
        const unsigned long long wr =
            __shfl_sync(0xffffffffu, static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(wrow)), src);
        const double v = q4k_exact_row(reinterpret_cast<const uint8_t *>(static_cast<uintptr_t>(wr)), nb, soa, x);
        if ((threadIdx.x & 31) == src)
            t = v;
    }
    return t;
}

}  // namespace dq
