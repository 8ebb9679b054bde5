// dq_internal.h -- declarations shared between the C-ABI layer (api.cu) and the
// kernel translation units of libdqgemv.  Not installed, not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace dq {

struct ArgmaxCand;

constexpr int kMaxGroup = 4;

// Outputs of a grouped GEMV: n > 0 matrices whose row tiles follow each other;
// matrix m holds padded rows base[m] .. base[m] + N[m] - 1 (base[m] a multiple of
// the tile height) and writes y[m][0 .. N[m]-1].  n == 0: not a group.
struct GroupOut {
    int n;
    float *y[kMaxGroup];
    long long N[kMaxGroup];
    long long base[kMaxGroup];
};

// Q4_K GEMV kernel arguments (one weight stream, or gate + up for SwiGLU).
struct Q4KParams {
    const uint8_t *w[2];
    const float *x;        // B x K
    float *y;              // B x N final output (splits == 1); Q when qg_hd > 0
    float *g;              // G output of the fused Q/gate split (qg_hd > 0), else null
    const float *res;      // B x N residual added to the plain output (may alias y), or null
    int qg_hd;             // head dim of the fused Q/gate split, 0 for a plain output
    float *part;           // [splits][NS][B][N] partial sums (splits > 1)
    ArgmaxCand *cand;      // per-CTA argmax candidates (argmax, splits == 1)
    int *err;              // device error flag
    long long N;
    int K;
    int nb;                // K / 256
    int splits;
    int chunks_per_split;  // K-chunks (of LPR super-blocks) per split
    int ctas_per_split;
    int depth;             // ring slots per warp
    int soa;
    int argmax;
    long long tiles;       // row tiles
    int cluster;           // fx kernel: split partials are added inside each cluster of `splits` CTAs
    GroupOut grp;          // grouped GEMV (fx kernel, batch 1): N is then the padded total
    const uint8_t *gw[kMaxGroup];   // weights of the grouped matrices
    unsigned long long wait_ns;     // limit of every bounded wait (kWaitNanos unless a test lowers it)
    int lost_copy;         // test hook: warp 0 of CTA 0 arms its first slot but issues no copy
};

struct Q4KPlan {
    bool ok;
    bool tma;              // slots moved by TMA tile copies (else one bulk copy per row)
    bool cluster;          // batch 1: K splits reduced in-kernel across a CTA cluster (no workspace)
    int R;                 // rows per lane
    int warps;             // warps per CTA
    long long tiles;
    int splits;
    int chunks_per_split;
    int ctas_per_split;
    int grid;
    int depth;
    int smem;
};

Q4KPlan q4k_plan(long long N, int K, int B, int NS, int soa, int sm_count, int smem_optin);
cudaError_t q4k_gemv_launch(const Q4KParams &p, const Q4KPlan &pl, int B, int NS, cudaStream_t s);
int q4k_fx_tile_rows();

// Q8_0 GEMV
struct Q8Params {
    const uint8_t *w;
    const float *x;
    float *y;
    int *err;
    long long N;
    int K;
    int nb;                // K / 32
};
struct Q8Plan {
    bool ok;
    int grid;
    int block;
    int smem;
};
Q8Plan q8_plan(long long N, int K, int B, int sm_count, int smem_optin);
cudaError_t q8_0_gemv_launch(const Q8Params &p, const Q8Plan &pl, int B, cudaStream_t s);

// split-K reduction (+ SwiGLU epilogue, + argmax candidates), argmax finalisation.
// Batch-1 partials carry error-bound planes; a row whose bound fails is
// recomputed exactly from these:
struct ExactArgs {
    const uint8_t *w[2];           // the matrix (gate and up for SwiGLU)
    const uint8_t *gw[kMaxGroup];  // grouped matrices
    const float *x;
    int nb;                        // K / 256
    int soa;
    int bounds;                    // 1: partials are [sums][bounds][|y| sums] planes (batch 1)
};
int reduce_grid(long long N, int B);
cudaError_t splitk_reduce_launch(const float *part, int splits, int NS, int B, long long N, float *y, float *g,
                                 int qg_hd, const GroupOut &grp, const float *res, ArgmaxCand *cand,
                                 const ExactArgs &ex, int grid, cudaStream_t s);
cudaError_t argmax_finalize_launch(const ArgmaxCand *cand, int ncand, long long *out, cudaStream_t s);

// debug dequant, repack
cudaError_t q4k_dequant_launch(const uint8_t *w, int soa, float *out, long long N, int K, cudaStream_t s);
cudaError_t q8_0_dequant_launch(const uint8_t *w, float *out, long long N, int K, cudaStream_t s);
cudaError_t q4k_repack_soa_launch(const uint8_t *aos, uint8_t *soa, long long N, int K, cudaStream_t s);

// The driver's tensor-map encoder, looked up once (null when unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// W4A16 prefill (tcgen05): Y = X W^T, X binary16, W Q4_K
struct PrefillPlan {
    bool ok;
    int th;                // accumulators of 128 tokens per CTA (1 or 2)
    int mtiles;            // token tiles of 128 * th
    int ntiles;            // 256-row weight tiles
    int splits;            // K splits (partials reduced by a second kernel when > 1)
    int sb_per_split;      // super-blocks per split
    int raw_depth;         // raw weight ring (super-blocks)
    int depth;             // operand ring (stages of 64 K)
    int tmem_cols;         // tensor-memory columns allocated per CTA
    int grid;
    int smem;
};
PrefillPlan q4k_prefill_plan(long long N, int K, long long M, int sm_count, int smem_optin);
cudaError_t q4k_prefill_launch(const uint8_t *w, int soa, const uint16_t *x16, float *y, float *part, int *err,
                               long long N, int K, long long M, const PrefillPlan &pl, cudaStream_t s);

// device error flag
int *device_error_flag(int device);

// The calling thread's current driver context (null if none or unknown): the
// key under which device addresses of this library's __device__ arrays are
// cached, so that a new context (after a device reset) looks them up again.
CUcontext current_context();

}  // namespace dq
