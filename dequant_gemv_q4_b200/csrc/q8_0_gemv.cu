// q8_0_gemv.cu -- fused Q8_0 dequantize + GEMV for sm_100a (the pages' CUDA
// lane Q8_0 GEMV: qualiaDB cuda_lane, try_q8_0_cuda_gemv; the design below is
// this library's own).
//
// A Q8_0 block is 34 bytes, so blocks (and rows, unless K % 256 == 0) are only
// 2-byte aligned.  A CTA stages a tile of 16 rows x one K-chunk of 32 blocks in
// shared memory with 16-byte loads for the aligned body of each row range and
// 2-byte loads for its ragged ends, placing every byte at the same address
// modulo 16 as in global memory.  Lane l then reads block l of two rows,
// realigns the quant words with a funnel shift, forms each weight exactly
// (q8_decode.cuh) and accumulates weight*x in fp32 (units of 2^-64, scaled back
// at the end); the row sums are reduced across the warp with shuffles.
#include <cuda_fp16.h>
#include <cstdint>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "q8_decode.cuh"

namespace dq {

constexpr int kQ8Threads = 256;
constexpr int kQ8RowsPerWarp = 2;
constexpr int kQ8Rows = (kQ8Threads / 32) * kQ8RowsPerWarp;  // 16 rows per tile
constexpr int kQ8ChunkBlocks = 32;                             // one block per lane
constexpr int kQ8RowPitch = kQ8ChunkBlocks * kQ8BlockBytes + 32;  // 1120, 16-byte multiple

template <int O, int M>
struct WarpReduceT {
    static __device__ __forceinline__ void run(float *v, int lane)
    {
        if constexpr (M > 1) {
            const bool up = (lane & O) != 0;
#pragma unroll
            for (int i = 0; i < M / 2; ++i) {
                const float send = up ? v[i] : v[i + M / 2];
                const float keep = up ? v[i + M / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
            }
            if constexpr (O > 1)
                WarpReduceT<O / 2, M / 2>::run(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
            if constexpr (O > 1)
                WarpReduceT<O / 2, 1>::run(v, lane);
        }
    }
};

template <int B>
__global__ void __launch_bounds__(kQ8Threads) q8_0_gemv_kernel(const Q8Params p)
{
    pdl_wait();
    pdl_launch_dependents();
    constexpr int MV = kQ8RowsPerWarp * B;
    constexpr int MP = (MV <= 2) ? 2 : (MV <= 4) ? 4 : (MV <= 8) ? 8 : 16;
    __shared__ __align__(16) uint8_t tile[kQ8Rows * kQ8RowPitch];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long row_bytes = static_cast<long long>(p.nb) * kQ8BlockBytes;
    const int nchunk = (p.nb + kQ8ChunkBlocks - 1) / kQ8ChunkBlocks;
    const long long ntiles = (p.N + kQ8Rows - 1) / kQ8Rows;

    for (long long ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
        const long long row0 = ti * kQ8Rows;
        // each chunk's products are summed in fp32 (16 per accumulator) and then
        // added into fp64, so the rounding error stays that of 16 + 7 additions
        // whatever K is
        double dacc[kQ8RowsPerWarp][B];
#pragma unroll
        for (int rr = 0; rr < kQ8RowsPerWarp; ++rr)
#pragma unroll
            for (int b = 0; b < B; ++b)
                dacc[rr][b] = 0.0;

        for (int ch = 0; ch < nchunk; ++ch) {
            const int kb0 = ch * kQ8ChunkBlocks;
            const int nblk = min(kQ8ChunkBlocks, p.nb - kb0);
            const int cbytes = nblk * kQ8BlockBytes;
            __syncthreads();  // the previous chunk has been consumed
#pragma unroll
            for (int rr = 0; rr < kQ8RowsPerWarp; ++rr) {
                const int r = warp * kQ8RowsPerWarp + rr;
                const long long n = row0 + r;
                if (n >= p.N)
                    continue;
                const uint8_t *g = p.w + n * row_bytes + static_cast<long long>(kb0) * kQ8BlockBytes;
                const int mis = static_cast<int>(reinterpret_cast<uintptr_t>(g) & 15);  // even
                uint8_t *s = tile + r * kQ8RowPitch + mis;
                const int head = min(cbytes, (16 - mis) & 15);
                const int body = ((cbytes - head) / 16) * 16;
                const int tail = cbytes - head - body;
                if (lane < head / 2)
                    reinterpret_cast<uint16_t *>(s)[lane] = reinterpret_cast<const uint16_t *>(g)[lane];
                for (int i = lane; i < body / 16; i += 32)
                    reinterpret_cast<uint4 *>(s + head)[i] = reinterpret_cast<const uint4 *>(g + head)[i];
                if (lane < tail / 2)
                    reinterpret_cast<uint16_t *>(s + head + body)[lane] =
                        reinterpret_cast<const uint16_t *>(g + head + body)[lane];
            }
            __syncthreads();

            float2 acc[kQ8RowsPerWarp][B];
#pragma unroll
            for (int rr = 0; rr < kQ8RowsPerWarp; ++rr)
#pragma unroll
                for (int b = 0; b < B; ++b)
                    acc[rr][b] = make_float2(0.f, 0.f);
            if (lane < nblk) {
                const int kb = kb0 + lane;
                uint32_t q[kQ8RowsPerWarp][8];
                float2 s01[kQ8RowsPerWarp], s23[kQ8RowsPerWarp], off[kQ8RowsPerWarp];
#pragma unroll
                for (int rr = 0; rr < kQ8RowsPerWarp; ++rr) {
                    const int r = warp * kQ8RowsPerWarp + rr;
                    const long long n = row0 + r;
                    const uint8_t *g = p.w + min(n, p.N - 1) * row_bytes + static_cast<long long>(kb0) * kQ8BlockBytes;
                    const int mis = static_cast<int>(reinterpret_cast<uintptr_t>(g) & 15);
                    const uint8_t *blk = tile + r * kQ8RowPitch + mis + lane * kQ8BlockBytes;
                    const float d = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t *>(blk)));
                    q8_scales(d, s01[rr], s23[rr], off[rr]);
                    const uintptr_t qa = reinterpret_cast<uintptr_t>(blk + 2);
                    const uint32_t *wb = reinterpret_cast<const uint32_t *>(qa & ~static_cast<uintptr_t>(3));
                    const uint32_t sh = static_cast<uint32_t>(qa & 3) * 8;  // 0 or 16
                    uint32_t v[9];
#pragma unroll
                    for (int j = 0; j < 9; ++j)
                        v[j] = wb[j];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        q[rr][j] = __funnelshift_r(v[j], v[j + 1], sh);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
#pragma unroll
                    for (int b = 0; b < B; ++b) {
                        const float4 xv = ldg_nc_f4(reinterpret_cast<const float4 *>(
                            p.x + static_cast<long long>(b) * p.K + static_cast<long long>(kb) * kQ8BlockElems + 4 * j));
#pragma unroll
                        for (int rr = 0; rr < kQ8RowsPerWarp; ++rr) {
                            float2 wv[2];
                            q8_word_weights(q[rr][j], s01[rr], s23[rr], off[rr], wv);
                            acc[rr][b] = __ffma2_rn(wv[0], make_float2(xv.x, xv.y), acc[rr][b]);
                            acc[rr][b] = __ffma2_rn(wv[1], make_float2(xv.z, xv.w), acc[rr][b]);
                        }
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < kQ8RowsPerWarp; ++rr)
#pragma unroll
                for (int b = 0; b < B; ++b)
                    dacc[rr][b] += static_cast<double>(acc[rr][b].x) + static_cast<double>(acc[rr][b].y);
        }

        // reduce the 32 lanes' partial sums of each (row, batch)
        float v[MP];
#pragma unroll
        for (int rr = 0; rr < kQ8RowsPerWarp; ++rr)
#pragma unroll
            for (int b = 0; b < B; ++b)
                v[rr * B + b] = static_cast<float>(dacc[rr][b]);
#pragma unroll
        for (int j = MV; j < MP; ++j)
            v[j] = 0.f;
        WarpReduceT<16, MP>::run(v, lane);
        int offi = 0;
        bool writer = true;
        {
            int m = MP;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                if (m > 1) {
                    if (lane & o)
                        offi += m / 2;
                    m /= 2;
                } else if (lane & o) {
                    writer = false;
                }
            }
        }
        constexpr int VPL = (MP > 32) ? MP / 32 : 1;
        if (writer) {
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int idx = offi + j;
                if (idx >= MV)
                    continue;
                const int rr = idx / B;
                const int b = idx % B;
                const long long n = row0 + warp * kQ8RowsPerWarp + rr;
                if (n < p.N)
                    p.y[static_cast<long long>(b) * p.N + n] = v[j] * 0x1p64f;
            }
        }
    }
}

Q8Plan q8_plan(long long N, int K, int B, int sm_count, int smem_optin)
{
    (void)K;
    (void)B;
    (void)smem_optin;
    Q8Plan pl{};
    const long long ntiles = (N + kQ8Rows - 1) / kQ8Rows;
    long long g = static_cast<long long>(sm_count) * 6;
    if (g > ntiles)
        g = ntiles;
    pl.grid = static_cast<int>(g < 1 ? 1 : g);
    pl.block = kQ8Threads;
    pl.smem = 0;
    pl.ok = true;
    return pl;
}

cudaError_t q8_0_gemv_launch(const Q8Params &p, const Q8Plan &pl, int B, cudaStream_t s)
{
    switch (B) {
    case 1: return launch_pdl(q8_0_gemv_kernel<1>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    case 2: return launch_pdl(q8_0_gemv_kernel<2>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    case 3: return launch_pdl(q8_0_gemv_kernel<3>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    case 4: return launch_pdl(q8_0_gemv_kernel<4>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    case 5: return launch_pdl(q8_0_gemv_kernel<5>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    case 6: return launch_pdl(q8_0_gemv_kernel<6>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    case 7: return launch_pdl(q8_0_gemv_kernel<7>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    case 8: return launch_pdl(q8_0_gemv_kernel<8>, dim3(pl.grid), dim3(pl.block), 0, s, p);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dq
