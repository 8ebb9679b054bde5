// aux_kernels.cu -- debug dequantization, the SoA repack, the split-K
// reduction (with the SwiGLU epilogue and argmax candidates) and the argmax
// finalisation, plus the per-device error flag.
#include <cuda_fp16.h>
#include <cstdint>
#include <mutex>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "q4k_decode.cuh"
#include "q8_decode.cuh"
#include "q4k_exact.cuh"

namespace dq {

// Set by kernels whose bounded waits gave up (see dq_device_error in dqgemv.h).
__device__ int g_dq_error_flag;

CUcontext current_context()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
        else
            cudaGetLastError();
    });
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS)
        c = nullptr;
    return c;
}

// Device address of the error flag on `device` (the current device), looked up
// once per context.
int *device_error_flag(int device)
{
    static std::mutex mu;
    static CUcontext ctx[64] = {};
    static int *addr[64] = {};
    if (device < 0 || device >= 64)
        return nullptr;
    const CUcontext cur = current_context();
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[device] || ctx[device] != cur) {
        void *a = nullptr;
        if (cudaGetSymbolAddress(&a, g_dq_error_flag) != cudaSuccess)
            return nullptr;
        addr[device] = static_cast<int *>(a);
        ctx[device] = cur;
    }
    return addr[device];
}

// ---------------------------------------------------------------------------
// Q4_K debug dequant: one thread per (row, super-block, 16-byte quant slice)
// writes that slice's 32 weights with the GEMV's own weight formation
// (q4k_decode.cuh); vector stores when `out` is 16-byte aligned.
// ---------------------------------------------------------------------------

// Byte offset within a row of the header (byte < 16) or of quant slice s of
// super-block kb in the SoA layout (groups of kQ4KSoaGroup super-blocks; see dqgemv.h).
__device__ __forceinline__ long long soa_hdr_off(int nb, int kb)
{
    const int first = (kb / kQ4KSoaGroup) * kQ4KSoaGroup;
    return static_cast<long long>(first) * kQ4KBlockBytes + 16 * (kb - first);
}
__device__ __forceinline__ long long soa_slice_off(int nb, int kb, int s)
{
    const int first = (kb / kQ4KSoaGroup) * kQ4KSoaGroup;
    const int g = min(kQ4KSoaGroup, nb - first);
    return static_cast<long long>(first) * kQ4KBlockBytes + 16 * g + 16 * g * s + 16 * (kb - first);
}

__global__ void q4k_dequant_kernel(const uint8_t *__restrict__ w, int soa, float *__restrict__ out,
                                   long long N, int K)
{
    const int nb = K / kQ4KBlockElems;
    const long long total = N * nb * 8;
    const long long row_bytes = static_cast<long long>(nb) * kQ4KBlockBytes;
    const bool vec = (reinterpret_cast<uintptr_t>(out) & 15) == 0;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int s = static_cast<int>(i % 8);
        const long long blk = i / 8;
        const int kb = static_cast<int>(blk % nb);
        const long long n = blk / nb;
        const uint8_t *row = w + n * row_bytes;
        const uint8_t *hp = soa ? row + soa_hdr_off(nb, kb) : row + static_cast<long long>(kb) * kQ4KBlockBytes;
        const uint8_t *qp = soa ? row + soa_slice_off(nb, kb, s)
                                : row + static_cast<long long>(kb) * kQ4KBlockBytes + 16 + 16 * s;
        const Hdr h = decode_hdr(*reinterpret_cast<const uint4 *>(hp));
        const uint4 q = *reinterpret_cast<const uint4 *>(qp);
        const ChunkScales cs = chunk_scales(h, s / 2);
        // lo weights of this slice start at L, hi weights at L + 32
        const long long L = n * K + static_cast<long long>(kb) * kQ4KBlockElems + 64 * (s / 2) + 16 * (s % 2);
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float2 wv[4];
            q4_word_weights(words[t], cs, wv);
            if (vec) {
                *reinterpret_cast<float4 *>(out + L + 4 * t) =
                    make_float4(wv[0].x * 0x1p64f, wv[1].x * 0x1p64f, wv[2].x * 0x1p64f, wv[3].x * 0x1p64f);
                *reinterpret_cast<float4 *>(out + L + 32 + 4 * t) =
                    make_float4(wv[0].y * 0x1p64f, wv[1].y * 0x1p64f, wv[2].y * 0x1p64f, wv[3].y * 0x1p64f);
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    out[L + 4 * t + k] = wv[k].x * 0x1p64f;
                    out[L + 32 + 4 * t + k] = wv[k].y * 0x1p64f;
                }
            }
        }
    }
}

static int grid_for(long long work, int block)
{
    long long g = (work + block - 1) / block;
    if (g > 65535LL * 16)
        g = 65535LL * 16;
    if (g < 1)
        g = 1;
    return static_cast<int>(g);
}

cudaError_t q4k_dequant_launch(const uint8_t *w, int soa, float *out, long long N, int K, cudaStream_t s)
{
    const long long total = N * (K / kQ4KBlockElems) * 8;
    q4k_dequant_kernel<<<grid_for(total, 256), 256, 0, s>>>(w, soa, out, N, K);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Q8_0 debug dequant: one thread per block, the GEMV's weight formation.
// ---------------------------------------------------------------------------
__global__ void q8_0_dequant_kernel(const uint8_t *__restrict__ w, float *__restrict__ out, long long N, int K)
{
    const int nb = K / kQ8BlockElems;
    const long long total = N * nb;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const uint8_t *blk = w + i * kQ8BlockBytes;  // blocks are contiguous over rows
        const uint16_t *h = reinterpret_cast<const uint16_t *>(blk);
        const float d = __half2float(__ushort_as_half(h[0]));
        float2 s01, s23, off;
        q8_scales(d, s01, s23, off);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t wq = static_cast<uint32_t>(h[1 + 2 * j]) | (static_cast<uint32_t>(h[2 + 2 * j]) << 16);
            float2 wv[2];
            q8_word_weights(wq, s01, s23, off, wv);
            float *o = out + i * kQ8BlockElems + 4 * j;
            o[0] = wv[0].x * 0x1p64f;
            o[1] = wv[0].y * 0x1p64f;
            o[2] = wv[1].x * 0x1p64f;
            o[3] = wv[1].y * 0x1p64f;
        }
    }
}

cudaError_t q8_0_dequant_launch(const uint8_t *w, float *out, long long N, int K, cudaStream_t s)
{
    const long long total = N * (K / kQ8BlockElems);
    q8_0_dequant_kernel<<<grid_for(total, 256), 256, 0, s>>>(w, out, N, K);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// AoS -> SoA repack: one thread per (row, super-block, 16-byte piece).
// Piece 0 is the header, pieces 1..8 the quant slices 0..7.
// ---------------------------------------------------------------------------
__global__ void q4k_repack_soa_kernel(const uint8_t *__restrict__ aos, uint8_t *__restrict__ soa, long long N,
                                      int K)
{
    const int nb = K / kQ4KBlockElems;
    const long long total = N * nb * 9;
    const long long row_bytes = static_cast<long long>(nb) * kQ4KBlockBytes;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int piece = static_cast<int>(i % 9);
        const long long blk = i / 9;
        const int kb = static_cast<int>(blk % nb);
        const long long n = blk / nb;
        const uint4 v = *reinterpret_cast<const uint4 *>(aos + n * row_bytes + static_cast<long long>(kb) * kQ4KBlockBytes +
                                                         16 * piece);
        const long long dst = n * row_bytes + (piece == 0 ? soa_hdr_off(nb, kb) : soa_slice_off(nb, kb, piece - 1));
        *reinterpret_cast<uint4 *>(soa + dst) = v;
    }
}

cudaError_t q4k_repack_soa_launch(const uint8_t *aos, uint8_t *soa, long long N, int K, cudaStream_t s)
{
    const long long total = N * (K / kQ4KBlockElems) * 9;
    q4k_repack_soa_kernel<<<grid_for(total, 256), 256, 0, s>>>(aos, soa, N, K);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Split-K reduction: out = sum over splits in split order (in fp64), with the
// batch-1 bound check and exact recomputation of a failing row; SwiGLU epilogue when
// NS == 2; per-CTA argmax candidates when cand != nullptr (B == 1).
// ---------------------------------------------------------------------------
constexpr int kReduceThreads = 256;

int reduce_grid(long long N, int B)
{
    long long g = (N * B + kReduceThreads - 1) / kReduceThreads;
    if (g > 1024)
        g = 1024;
    return static_cast<int>(g < 1 ? 1 : g);
}

__global__ void __launch_bounds__(kReduceThreads) splitk_reduce_kernel(const float *__restrict__ part, int splits,
                                                                       int NS, int B, long long N,
                                                                       float *y, float *__restrict__ g_out,
                                                                       int qg_hd, const GroupOut grp,
                                                                       const float *res, ArgmaxCand *cand,
                                                                       const ExactArgs ex)
{
    pdl_wait();
    pdl_launch_dependents();
    float best_v = -INFINITY;
    long long best_i = 0x7fffffffffffffffLL;
    const int lane = threadIdx.x & 31;
    const long long total = N * B;
    const long long P = static_cast<long long>(splits) * NS * B * N;   // one plane of partials
    const long long row_bytes = static_cast<long long>(ex.nb) * kQ4KBlockBytes;
    // whole warps step together (the exact recomputation of a row is warp-wide)
    for (long long base = blockIdx.x * static_cast<long long>(blockDim.x) + (threadIdx.x & ~31); base < total;
         base += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long i = base + lane;
        const bool in = i < total;
        const long long n = in ? i % N : 0;
        const int b = in ? static_cast<int>(i / N) : 0;
        // the fp32 partials are added in fp64 (in split order), so the sum adds
        // no rounding beyond the partials' own and the final one; batch-1 bounds
        // are added rounded outwards
        double gd = 0.0, ud = 0.0;
        float ge = 0.f, gs = 0.f, ue = 0.f, us = 0.f;
        if (in) {
            for (int s = 0; s < splits; ++s) {
                const long long ig = ((static_cast<long long>(s) * NS + 0) * B + b) * N + n;
                gd += part[ig];
                if (ex.bounds) {
                    ge = __fadd_ru(ge, part[P + ig]);
                    gs = __fadd_rd(gs, part[2 * P + ig]);
                }
                if (NS == 2) {
                    const long long iu = ig + static_cast<long long>(B) * N;
                    ud += part[iu];
                    if (ex.bounds) {
                        ue = __fadd_ru(ue, part[P + iu]);
                        us = __fadd_rd(us, part[2 * P + iu]);
                    }
                }
            }
        }
        // padded row n of a grouped GEMV: the matrix holding it, and its row there
        int m = 0;
        long long row = n;
        bool valid = in;
        float *ym = nullptr;
        if (grp.n > 0) {
#pragma unroll
            for (int k = 1; k < kMaxGroup; ++k)
                if (k < grp.n && n >= grp.base[k])
                    m = k;
            const long long gbase = m == 0 ? grp.base[0] : m == 1 ? grp.base[1] : m == 2 ? grp.base[2] : grp.base[3];
            const long long rows = m == 0 ? grp.N[0] : m == 1 ? grp.N[1] : m == 2 ? grp.N[2] : grp.N[3];
            ym = m == 0 ? grp.y[0] : m == 1 ? grp.y[1] : m == 2 ? grp.y[2] : grp.y[3];
            row = n - gbase;
            valid = in && row < rows;
        }
        if (ex.bounds) {
            const uint8_t *w0 = grp.n > 0 ? (m == 0 ? ex.gw[0] : m == 1 ? ex.gw[1] : m == 2 ? ex.gw[2] : ex.gw[3])
                                          : ex.w[0];
            gd = fx_fix_rows(gd, ge, gs, valid, w0 + row * row_bytes, ex.nb, ex.soa, ex.x);
            if (NS == 2)
                ud = fx_fix_rows(ud, ue, us, valid, ex.w[1] + row * row_bytes, ex.nb, ex.soa, ex.x);
        }
        if (!valid)
            continue;
        const float g = static_cast<float>(gd), u = static_cast<float>(ud);
        const float out = (NS == 2) ? g / (1.0f + expf(-g)) * u : (res ? g + res[i] : g);
        if (grp.n > 0) {
            ym[row] = out;
            continue;
        }
        *gemv_out_addr(y, g_out, qg_hd, N, b, n) = out;
        if (cand && cand_better(out, n, best_v, best_i)) {
            best_v = out;
            best_i = n;
        }
    }
    if (cand) {
        __shared__ ArgmaxCand red[kReduceThreads / 32];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
            const long long oi = __shfl_xor_sync(0xffffffffu, best_i, o);
            if (cand_better(ov, oi, best_v, best_i)) {
                best_v = ov;
                best_i = oi;
            }
        }
        if ((threadIdx.x & 31) == 0) {
            red[threadIdx.x >> 5].v = best_v;
            red[threadIdx.x >> 5].idx = best_i;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            ArgmaxCand c = red[0];
            for (int w = 1; w < kReduceThreads / 32; ++w)
                if (cand_better(red[w].v, red[w].idx, c.v, c.idx))
                    c = red[w];
            cand[blockIdx.x] = c;
        }
    }
}

cudaError_t splitk_reduce_launch(const float *part, int splits, int NS, int B, long long N, float *y, float *g,
                                 int qg_hd, const GroupOut &grp, const float *res, ArgmaxCand *cand,
                                 const ExactArgs &ex, int grid, cudaStream_t s)
{
    return launch_pdl(splitk_reduce_kernel, dim3(grid), dim3(kReduceThreads), 0, s, part, splits, NS, B, N, y, g,
                      qg_hd, grp, res, cand, ex);
}

// One CTA folds all candidates into the final index.
__global__ void __launch_bounds__(1024) argmax_finalize_kernel(const ArgmaxCand *__restrict__ cand, int ncand,
                                                               long long *out)
{
    pdl_wait();
    pdl_launch_dependents();
    float best_v = -INFINITY;
    long long best_i = 0x7fffffffffffffffLL;
    for (int i = threadIdx.x; i < ncand; i += blockDim.x)
        if (cand_better(cand[i].v, cand[i].idx, best_v, best_i)) {
            best_v = cand[i].v;
            best_i = cand[i].idx;
        }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
        const long long oi = __shfl_xor_sync(0xffffffffu, best_i, o);
        if (cand_better(ov, oi, best_v, best_i)) {
            best_v = ov;
            best_i = oi;
        }
    }
    __shared__ ArgmaxCand red[32];
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5].v = best_v;
        red[threadIdx.x >> 5].idx = best_i;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        ArgmaxCand c = red[0];
        for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w)
            if (cand_better(red[w].v, red[w].idx, c.v, c.idx))
                c = red[w];
        // every value NaN leaves no candidate: report -1
        *out = (c.idx == 0x7fffffffffffffffLL) ? -1 : c.idx;
    }
}

cudaError_t argmax_finalize_launch(const ArgmaxCand *cand, int ncand, long long *out, cudaStream_t s)
{
    return launch_pdl(argmax_finalize_kernel, dim3(1), dim3(1024), 0, s, cand, ncand, out);
}

}  // namespace dq
