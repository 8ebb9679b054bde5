/*
 * dqgemv.h -- C ABI of libdqgemv.so: fused block-quantized dequantize + GEMV
 * for NVIDIA B200 (sm_100a).
 *
 * The operation.  y = W x for one decode step, where W (N rows x K columns) is
 * stored as GGML-style quantized blocks and x is fp32.  The pages this library
 * follows call it the fused dequant+GEMV ("upload raw Q4K weight bytes for
 * fused dequant+GEMV on GPU": trueno WgslForwardPass, upload_q4k_weight) and
 * ship it as a CUDA lane with a Q4_K structure-of-arrays GEMV, a fused SwiGLU
 * variant and a Q8_0 GEMV (qualiaDB cuda_lane module map: try_q4k_soa_gemv,
 * try_q4k_soa_fused_swiglu, try_q8_0_cuda_gemv, preload_q4k_soa_weights).
 *
 * Block formats (little-endian):
 *   Q8_0  34 bytes / 32 weights:  d (fp16) | q[32] (int8)         w = d*q
 *   Q4_K 144 bytes / 256 weights: d (fp16) | dmin (fp16) | 12 scale bytes
 *         (8 six-bit scale/min pairs, GGML get_scale_min_k4 packing)
 *         | 128 quant bytes (4-bit; chunk c = bytes 32c..32c+31 holds weights
 *         64c..64c+31 in its low nibbles and 64c+32..64c+63 in its high ones)
 *         w = d*scale_j*q - dmin*min_j  for sub-block j = weight/32.
 *   A row is K/32 (Q8_0) or K/256 (Q4_K) consecutive blocks; rows follow each
 *   other without padding, so W occupies N*K*34/32 or N*K*144/256 bytes.
 *
 * Numerics.  Results satisfy
 *     |y - y_exact| <= 1e-4 * sum_k |W[n][k] * x[k]| + 1e-6
 * (y_exact: the exact sum over the exact dequantized weights) for every finite
 * input, up to fp32 overflow of the result.
 *   - Q8_0 and Q4_K with B >= 2: every weight is formed exactly as the fp32
 *     value nearest to its dequantized value (the bits the *_dequant entry
 *     points return) and the products are accumulated in fp32, at most 1024
 *     products per accumulator (Q4_K: K is split so; Q8_0: each 1024-wide
 *     chunk of K is summed in fp32 and the chunks in fp64), then in fp64.
 *   - Q4_K with B == 1 (q4k_gemv, q4k_swiglu_gemv, q4k_gemv_split_qg,
 *     q4k_gemv_group, q4k_gemv_residual, q4k_ffn_block): each activation is
 *     rounded to a 30-bit fixed point shared by its super-block of 256
 *     activations, and the dot products over the exact quants, scales and mins
 *     are then exact (integers, fp64).  Beside every output the kernel keeps an
 *     upper bound on the error that rounding caused and a lower bound on
 *     sum_k |W[n][k] x[k]|; an output whose bound does not prove the inequality
 *     above (possible only when a super-block mixes activations of very
 *     different sizes and its large ones meet near-zero weights) is recomputed
 *     with exact weights in fp64 before it is stored.  An infinity or NaN in x
 *     makes every result that reads it NaN.
 *   - Environment: DQGEMV_NO_TMA=1 makes the batch-1 kernel fill its shared
 *     memory with per-row bulk copies instead of TMA tile copies (bitwise
 *     identical results; a debugging aid).
 *
 * Conventions shared by every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller (for example
 *     allocated by PyTorch).  The library never allocates or frees memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous: they enqueue work and return without synchronizing.
 *     Inputs must stay alive, and outputs untouched, until the stream reaches
 *     the call.
 *   - Every argument is validated on the host before anything is enqueued.
 *     On any error status nothing is launched and no memory is touched.
 *   - The device of the call is the current CUDA device of the calling thread.
 *   - Batched activations are row-major: x is B x K (row b at x + b*K) and y is
 *     B x N (row b at y + b*N).
 */
#ifndef DQGEMV_H
#define DQGEMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dq_status {
    DQ_OK = 0,
    DQ_ERR_NULL = 1,      /* a required pointer is NULL                              */
    DQ_ERR_SHAPE = 2,     /* N < 1, K not a positive multiple of the block size,
                             K above the supported maximum, or B outside [1, 8]      */
    DQ_ERR_ALIGN = 3,     /* w or x is not 16-byte aligned, y not 4-byte aligned     */
    DQ_ERR_WORKSPACE = 4, /* workspace NULL or smaller than dq_workspace_bytes()     */
    DQ_ERR_LAYOUT = 5,    /* layout is not DQ_LAYOUT_AOS / DQ_LAYOUT_SOA             */
    DQ_ERR_CUDA = 6,      /* a CUDA runtime call failed; see dq_last_cuda_error()    */
    DQ_ERR_ARG = 7        /* any other invalid argument (e.g. argmax with B != 1)    */
} dq_status;

typedef enum dq_layout {
    DQ_LAYOUT_AOS = 0,    /* GGML block order: 144-byte super-blocks back to back    */
    DQ_LAYOUT_SOA = 1     /* q4k_repack_soa() order (see there)                      */
} dq_layout;

typedef enum dq_op {
    DQ_OP_Q8_0_GEMV = 0,
    DQ_OP_Q4K_GEMV = 1,
    DQ_OP_Q4K_SWIGLU = 2,
    DQ_OP_Q4K_PREFILL = 3,  /* q4k_prefill_gemm; the `B` argument is M */
    DQ_OP_Q4K_FFN = 4       /* q4k_ffn_block; the `N`, `K` arguments are H, F */
} dq_op;

/* Largest K accepted by the GEMV entry points (fp32 activations of one split
 * of K are staged in shared memory). */
#define DQ_MAX_K 1048576

/*
 * Q8_0 GEMV:  y[b][n] = sum_k W[n][k] * x[b][k].
 *   w   N*(K/32) Q8_0 blocks (34 bytes each), 16-byte aligned.
 *   x   B x K fp32, 16-byte aligned.       y  B x N fp32, 4-byte aligned.
 *   K   positive multiple of 32.           B  1..8.
 *   workspace / ws_bytes: scratch of at least
 *       dq_workspace_bytes(DQ_OP_Q8_0_GEMV, N, K, B, 0) bytes (may be NULL/0
 *       when that is 0).  Contents on entry are ignored; the library keeps no
 *       state in it between calls.
 */
dq_status q8_0_gemv(const void *w, const float *x, float *y, int64_t N, int64_t K, int B,
                    void *workspace, size_t ws_bytes, void *stream);

/*
 * Q4_K GEMV:  y[b][n] = sum_k W[n][k] * x[b][k],  optionally with argmax.
 *   w          N*(K/256) Q4_K super-blocks, 16-byte aligned, in `layout`.
 *   x, y, B    as for q8_0_gemv.           K  positive multiple of 256.
 *   argmax_out NULL, or (B == 1 only) a device int64: receives the index n of
 *              the largest y[0][n]; among equal largest values the lowest n.
 *              (The LM-head epilogue; NaN outputs make it unspecified.)
 *   workspace  at least dq_workspace_bytes(DQ_OP_Q4K_GEMV, N, K, B,
 *              argmax_out != NULL) bytes.
 */
dq_status q4k_gemv(const void *w, int layout, const float *x, float *y, int64_t N, int64_t K,
                   int B, int64_t *argmax_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * Q4_K GEMV with a fused residual add, the down projection of a decoder
 * layer's FFN block (qualiaDB cuda_lane: try_q4k_soa_ffn_block_residual):
 *   y[b][n] = sum_k W[n][k] * x[b][k] + residual[b][n].
 *   residual  B x N fp32, 4-byte aligned; it may be y itself (y += W x).
 *   Other arguments, the workspace and argmax (over the sums) as for q4k_gemv.
 * The product is formed exactly as q4k_gemv forms it, rounded to fp32, and the
 * residual is then added in fp32.
 */
dq_status q4k_gemv_residual(const void *w, int layout, const float *x, const float *residual, float *y, int64_t N,
                            int64_t K, int B, int64_t *argmax_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * A decoder layer's FFN block in one call (qualiaDB cuda_lane:
 * try_q4k_soa_ffn_block, try_q4k_soa_ffn_block_residual):
 *   h = silu(W_gate x) * (W_up x)        (B x F)
 *   y = W_down h [+ residual]            (B x H)
 * as two launches on `stream`, the second chained to the first by programmatic
 * dependent launch; h (B x F fp32) is left at the start of the workspace.
 *   w_gate, w_up  F x H Q4_K matrices;  w_down  H x F;  all in `layout`,
 *                 16-byte aligned.
 *   x             B x H fp32, 16-byte aligned.   y  B x H fp32, 4-byte aligned.
 *   residual      NULL, or B x H fp32, 4-byte aligned; it may be x or y
 *                 (y = x + FFN(x) in place is allowed).
 *   H, F          positive multiples of 256.     B  1..8.
 *   workspace     at least dq_workspace_bytes(DQ_OP_Q4K_FFN, H, F, B, 0) bytes.
 * Every argument is checked before the first launch.  The results are exactly
 * those of the two separate calls.
 */
dq_status q4k_ffn_block(const void *w_gate, const void *w_up, const void *w_down, int layout, const float *x,
                        const float *residual, float *y, int64_t H, int64_t F, int B, void *workspace, size_t ws_bytes,
                        void *stream);

/*
 * Q4_K GEMV of a q-projection-with-gate matrix with the Q/gate de-interleave
 * fused into the store (Doppler 0.1.8, split_qg.wgsl: "attentionOutputGate"
 * models interleave, per head, head_dim Q rows and head_dim gate rows):
 *   with y = W x (B x N) and h, d such that n = h*2*head_dim + d,
 *     q[b][h*head_dim + d]            = y[b][n]  for d <  head_dim,
 *     g[b][h*head_dim + d - head_dim] = y[b][n]  for d >= head_dim.
 *   q, g      B x N/2 fp32 each, 4-byte aligned, not overlapping (q takes the
 *             place of y; x as for q4k_gemv).
 *   N         a positive multiple of 2*head_dim.
 *   workspace at least dq_workspace_bytes(DQ_OP_Q4K_GEMV, N, K, B, 0) bytes.
 * The values are exactly those q4k_gemv writes for the same call, stored in
 * the split order; no argmax.
 */
dq_status q4k_gemv_split_qg(const void *w, int layout, const float *x, float *q, float *g, int64_t N, int64_t K,
                            int B, int64_t head_dim, void *workspace, size_t ws_bytes, void *stream);

/*
 * Grouped batch-1 Q4_K GEMV: up to DQ_MAX_GROUP matrices that share one
 * activation vector (for example the Q, K and V projections of a layer) in one
 * launch (qualiaDB cuda_lane: try_q4k_soa_qkv):
 *   y[m][n] = sum_k W_m[n][k] * x[k],  m < count, n < N[m].
 *   count       1..DQ_MAX_GROUP.
 *   w, N, y     HOST arrays of `count` entries, read during the call: device
 *               pointers to each matrix (N[m] x K Q4_K super-blocks, 16-byte
 *               aligned, all in `layout`), row counts (>= 1), and device
 *               outputs of N[m] fp32 (4-byte aligned).
 *   x           K fp32, 16-byte aligned.   K  positive multiple of 256.
 *   workspace   at least dq_workspace_bytes(DQ_OP_Q4K_GEMV, P, K, 1, 0) bytes,
 *               P = sum over m of N[m] rounded up to a multiple of 16.
 * Numerics as for q4k_gemv with B == 1.
 */
#define DQ_MAX_GROUP 4
dq_status q4k_gemv_group(int count, const void *const *w, const int64_t *N, float *const *y, int layout,
                         const float *x, int64_t K, void *workspace, size_t ws_bytes, void *stream);

/*
 * Fused gate/up SwiGLU GEMV (qualiaDB cuda_lane: try_q4k_soa_fused_swiglu;
 * trueno WgslForwardPass: silu_mul_shader, here fused into the GEMV):
 *   out[b][n] = silu(g) * u,  g = (W_gate x_b)[n],  u = (W_up x_b)[n],
 *   silu(g) = g / (1 + exp(-g)).
 *   w_gate, w_up  two N x K Q4_K matrices in the same `layout`, 16-byte aligned.
 *   out           B x N fp32.  Other arguments as for q4k_gemv.
 *   workspace     at least dq_workspace_bytes(DQ_OP_Q4K_SWIGLU, N, K, B, 0).
 */
dq_status q4k_swiglu_gemv(const void *w_gate, const void *w_up, int layout, const float *x,
                          float *out, int64_t N, int64_t K, int B, void *workspace,
                          size_t ws_bytes, void *stream);

/*
 * W4A16 prefill GEMM: 4-bit weights, 16-bit activations, M tokens at once
 * (qualiaDB qwen3_attention, prefill_weights: "W4A16 M128 dispatcher"; the
 * pages name the operation and its operand widths, nothing more).
 *   y[m][n] = sum_k W16[n][k] * x16[m][k],  m < M, n < N,
 * where W16[n][k] is the Q4_K weight rounded to fp32 (exactly the value
 * q4k_dequant returns) and then to binary16 (round to nearest even), and x16
 * holds binary16 values.  The products are summed in fp32 on the tensor cores
 * (K split across CTAs when there are few tiles; the splits' partial sums are
 * then added in a fixed order, so results are deterministic).
 *   w          N x K Q4_K matrix in `layout`, 16-byte aligned.
 *   x16        M x K binary16 bit patterns, row-major, 16-byte aligned.
 *   y          M x N fp32, row-major, 16-byte aligned.
 *   N >= 1;  K a positive multiple of 256, at most DQ_MAX_K;
 *   M in [1, DQ_MAX_PREFILL_M].
 *   workspace  at least dq_workspace_bytes(DQ_OP_Q4K_PREFILL, N, K, M, 0) bytes.
 * Needs the driver's tensor-map encoder; without it the call returns
 * DQ_ERR_CUDA (dq_last_cuda_error() = cudaErrorNotSupported) and enqueues
 * nothing.
 */
#define DQ_MAX_PREFILL_M 65536
dq_status q4k_prefill_gemm(const void *w, int layout, const uint16_t *x16, float *y, int64_t N, int64_t K,
                           int64_t M, void *workspace, size_t ws_bytes, void *stream);

/*
 * Offline repack of a Q4_K matrix from GGML block order (AoS) into this
 * library's structure-of-arrays order (qualiaDB cuda_lane:
 * preload_q4k_soa_weights; the pages do not define the SoA layout, this is the
 * library's own).  Every row keeps its byte range and size.  Within a row the
 * super-blocks are taken in groups of 4 (the last group holds the remaining
 * g <= 4); a group of g blocks is stored as g 16-byte headers (d, dmin, 12
 * scale bytes of block t at 16*t) followed by 8 slices, slice s holding quant
 * bytes 16s..16s+15 of each block t at 16*g + 16*g*s + 16*t.
 *   w_aos, w_soa  N*(K/256)*144 bytes each, 16-byte aligned, not overlapping.
 */
dq_status q4k_repack_soa(const void *w_aos, void *w_soa, int64_t N, int64_t K, void *stream);

/*
 * Scratch bytes the GEMV entry points need for this shape on the current
 * device (split-K partial sums, argmax candidates).  0 means none.
 * `op` is a dq_op; `with_argmax` is nonzero when argmax_out will be passed.
 * Returns (size_t)-1 for an invalid op or shape.
 */
size_t dq_workspace_bytes(int op, int64_t N, int64_t K, int B, int with_argmax);

/*
 * Debug dequantization (the bit-exact check of the weights the GEMVs use):
 * out[n][k] = the fp32 value nearest to the exact dequantized W[n][k]
 * (round to nearest even).  out is N x K fp32, 4-byte aligned.  Rows are
 * independent, so a row slice is a pointer offset on w and out.
 */
dq_status q8_0_dequant(const void *w, float *out, int64_t N, int64_t K, void *stream);
dq_status q4k_dequant(const void *w, int layout, float *out, int64_t N, int64_t K, void *stream);

/*
 * q4k_gemv without a workspace argument, for callers that cannot allocate
 * device memory (code that runs where no allocator is reachable, or that must
 * not allocate once set up, such as a decode loop whose memory budget is fixed
 * in advance).  No counterpart on the pages: this is a packaging of q4k_gemv.
 *   Arguments and results are exactly those of q4k_gemv minus the workspace.
 *   The scratch it needs (split-K partial sums, argmax candidates) lives in a
 *   fixed array of dq_noalloc_scratch_bytes() bytes (4 MiB) inside the library,
 *   held by every GPU that loads the library until the process exits.  A shape
 *   whose q4k_gemv workspace (dq_workspace_bytes) is larger than that returns
 *   DQ_ERR_WORKSPACE and launches nothing.
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   The address is cached per device and driver context: after a device
 *   reset (a new context) the next call looks it up again.
 *   It never calls cudaMalloc, cudaFree or any allocating routine.
 *   Every call shares the one array and nothing in it needs to start at zero;
 *   calls that may overlap on the GPU (other streams, other host threads)
 *   race on it, so serialize them.
 */
dq_status q4k_gemv_noalloc(const void *w, int layout, const float *x, float *y, int64_t N, int64_t K,
                           int B, int64_t *argmax_out, void *stream);

/* Size in bytes of the fixed scratch array q4k_gemv_noalloc uses. */
size_t dq_noalloc_scratch_bytes(void);

/*
 * Test of the bounded waits (no counterpart on the pages; this library's
 * failure detection, see dq_device_error).  A batch-1 q4k_gemv call (AoS
 * layout, no argmax) in which warp 0 of the first CTA arms the mbarrier of its
 * first slot but issues no copy into it, so that its wait runs out; every
 * bounded wait of the launch gives up after wait_ns nanoseconds instead of the
 * usual 2 s.  The kernel then sets the device error flag, waits (bounded) for
 * its other copies in flight and returns; the rows of that slot's tile are not
 * written correctly, the others are.  No fault, trap or hang is involved.
 *   wait_ns    1,000 .. 2,000,000,000.   Other arguments as for q4k_gemv.
 * Returns DQ_ERR_ARG for a wait_ns outside that range; otherwise as q4k_gemv.
 */
dq_status dq_test_lost_copy(const void *w, const float *x, float *y, int64_t N, int64_t K, uint64_t wait_ns,
                            void *workspace, size_t ws_bytes, void *stream);

/* Static string naming a status code. */
const char *dq_status_string(int status);

/* cudaError_t of the most recent DQ_ERR_CUDA returned on this thread (0 if none). */
int dq_last_cuda_error(void);

/*
 * Device-side error flag of the current device.  Kernels that wait for their
 * own asynchronous copies give up after a bounded wait instead of hanging;
 * when that happens they set this flag (and their output is invalid).
 * Synchronizes `stream`, writes the flag value to *flag (0 = no error) and,
 * when `clear` is nonzero, resets it.
 */
dq_status dq_device_error(int *flag, int clear, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DQGEMV_H */
