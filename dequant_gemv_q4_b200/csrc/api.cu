// api.cu -- the C ABI of libdqgemv (declared and documented in dqgemv.h):
// argument validation, launch planning, workspace carving and kernel launch.
// Nothing here allocates device memory; every pointer comes from the caller.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <cuda_runtime.h>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "dqgemv.h"

namespace {

thread_local int g_last_cuda_error = 0;

dq_status cuda_fail(cudaError_t e)
{
    g_last_cuda_error = static_cast<int>(e);
    return DQ_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct DevInfo {
    int device;
    int sm_count;
    int smem_optin;
};

dq_status dev_info(DevInfo &di)
{
    static int cached_sm[64] = {};
    static int cached_smem[64] = {};
    cudaError_t e = cudaGetDevice(&di.device);
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (di.device >= 0 && di.device < 64 && cached_sm[di.device] > 0) {
        di.sm_count = cached_sm[di.device];
        di.smem_optin = cached_smem[di.device];
        return DQ_OK;
    }
    e = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, di.device);
    if (e != cudaSuccess)
        return cuda_fail(e);
    e = cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, di.device);
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (di.device >= 0 && di.device < 64) {
        cached_sm[di.device] = di.sm_count;
        cached_smem[di.device] = di.smem_optin;
    }
    return DQ_OK;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }


// Workspace layout of the Q4_K GEMV for a plan: [split partials][argmax candidates].
struct Q4KWorkspace {
    size_t part_bytes;
    size_t cand_bytes;
    int ncand;
    size_t total() const { return part_bytes + cand_bytes; }
};

Q4KWorkspace q4k_ws(const dq::Q4KPlan &pl, long long N, int B, int NS, bool argmax)
{
    Q4KWorkspace ws{};
    const bool reduce_kernel = pl.splits > 1 && !pl.cluster;
    // batch 1 adds two planes of per-row bounds (error, sum of |y|) to the sums
    const size_t planes = (B == 1) ? 3 : 1;
    if (reduce_kernel)
        ws.part_bytes = round_up(planes * pl.splits * NS * B * N * sizeof(float), 256);
    if (argmax) {
        ws.ncand = reduce_kernel ? dq::reduce_grid(N, B) : pl.grid;
        ws.cand_bytes = round_up(static_cast<size_t>(ws.ncand) * sizeof(dq::ArgmaxCand), 256);
    }
    return ws;
}

dq_status check_q4k_shape(int64_t N, int64_t K, int B)
{
    if (N < 1 || K < 256 || K % 256 != 0 || K > DQ_MAX_K || B < 1 || B > 8)
        return DQ_ERR_SHAPE;
    return DQ_OK;
}

// Scratch of one Q4_K GEMV (NS = 1) or SwiGLU pair (NS = 2) on the current
// device, for either layout; (size_t)-1 if the shape has no plan.
size_t q4k_gemv_ws_bytes(int64_t N, int64_t K, int B, int NS, bool argmax)
{
    const size_t bad = static_cast<size_t>(-1);
    if (check_q4k_shape(N, K, B) != DQ_OK)
        return bad;
    DevInfo di;
    if (dev_info(di) != DQ_OK)
        return bad;
    size_t need = 0;
    for (int soa = 0; soa < 2; ++soa) {
        const dq::Q4KPlan pl = dq::q4k_plan(N, static_cast<int>(K), B, NS, soa, di.sm_count, di.smem_optin);
        if (!pl.ok)
            return bad;
        const size_t t = q4k_ws(pl, N, B, NS, argmax).total();
        if (t > need)
            need = t;
    }
    return need;
}

// FFN block scratch: the SwiGLU output h (B x F) and then the larger of the two
// GEMVs' own scratch.
size_t ffn_ws_bytes(int64_t H, int64_t F, int B)
{
    const size_t bad = static_cast<size_t>(-1);
    const size_t a = q4k_gemv_ws_bytes(F, H, B, 2, false);
    const size_t b = q4k_gemv_ws_bytes(H, F, B, 1, false);
    if (a == bad || b == bad)
        return bad;
    return round_up(static_cast<size_t>(B) * F * sizeof(float), 256) + (a > b ? a : b);
}

dq_status check_prefill_shape(int64_t N, int64_t K, int64_t M)
{
    if (N < 1 || N > 0x7FFFFFFFLL || K < 256 || K % 256 != 0 || K > DQ_MAX_K || M < 1 || M > DQ_MAX_PREFILL_M)
        return DQ_ERR_SHAPE;
    return DQ_OK;
}

size_t prefill_ws_bytes(const dq::PrefillPlan &pl, int64_t N, int64_t M)
{
    return pl.splits > 1 ? round_up(static_cast<size_t>(pl.splits) * M * N * sizeof(float), 256) : 0;
}

dq_status q4k_common(const void *w0, const void *w1, int layout, const float *x, float *y, int64_t N, int64_t K,
                     int B, int NS, int64_t *argmax_out, void *workspace, size_t ws_bytes, void *stream,
                     float *g_out = nullptr, int64_t qg_hd = 0, const dq::GroupOut *grp = nullptr,
                     const void *const *gw = nullptr, const float *res = nullptr,
                     unsigned long long wait_ns = dq::kWaitNanos, int lost_copy = 0)
{
    if (!w0 || (NS == 2 && !w1) || !x || !y)
        return DQ_ERR_NULL;
    if (layout != DQ_LAYOUT_AOS && layout != DQ_LAYOUT_SOA)
        return DQ_ERR_LAYOUT;
    dq_status st = check_q4k_shape(N, K, B);
    if (st != DQ_OK)
        return st;
    if (argmax_out && (B != 1 || NS != 1))
        return DQ_ERR_ARG;
    if (!aligned(w0, 16) || (w1 && !aligned(w1, 16)) || !aligned(x, 16) || !aligned(y, 4) ||
        (argmax_out && !aligned(argmax_out, 8)))
        return DQ_ERR_ALIGN;
    DevInfo di;
    st = dev_info(di);
    if (st != DQ_OK)
        return st;
    const dq::Q4KPlan pl = dq::q4k_plan(N, static_cast<int>(K), B, NS, layout == DQ_LAYOUT_SOA, di.sm_count,
                                        di.smem_optin);
    if (!pl.ok)
        return DQ_ERR_SHAPE;
    const Q4KWorkspace ws = q4k_ws(pl, N, B, NS, argmax_out != nullptr);
    if (ws.total() > 0 && (!workspace || ws_bytes < ws.total()))
        return DQ_ERR_WORKSPACE;
    if (ws.total() > 0 && !aligned(workspace, 16))
        return DQ_ERR_ALIGN;

    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    dq::Q4KParams p{};
    p.w[0] = static_cast<const uint8_t *>(w0);
    p.w[1] = static_cast<const uint8_t *>(NS == 2 ? w1 : w0);
    p.x = x;
    p.y = y;
    p.g = g_out;
    p.res = res;
    p.qg_hd = static_cast<int>(qg_hd);
    if (grp) {
        p.grp = *grp;
        for (int m = 0; m < grp->n; ++m)
            p.gw[m] = static_cast<const uint8_t *>(gw[m]);
    }
    p.part = (pl.splits > 1 && !pl.cluster) ? reinterpret_cast<float *>(wsb) : nullptr;
    p.cand = argmax_out ? reinterpret_cast<dq::ArgmaxCand *>(wsb + ws.part_bytes) : nullptr;
    p.err = dq::device_error_flag(di.device);
    p.N = N;
    p.K = static_cast<int>(K);
    p.nb = static_cast<int>(K / 256);
    p.splits = pl.splits;
    p.chunks_per_split = pl.chunks_per_split;
    p.ctas_per_split = pl.ctas_per_split;
    p.depth = pl.depth;
    p.soa = layout == DQ_LAYOUT_SOA;
    p.argmax = argmax_out != nullptr;
    p.tiles = pl.tiles;
    p.cluster = pl.cluster ? 1 : 0;
    p.wait_ns = wait_ns;
    p.lost_copy = lost_copy;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = dq::q4k_gemv_launch(p, pl, B, NS, s);
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (pl.splits > 1 && !pl.cluster) {
        dq::ExactArgs ex{};
        ex.w[0] = p.w[0];
        ex.w[1] = p.w[1];
        for (int m = 0; m < dq::kMaxGroup; ++m)
            ex.gw[m] = p.gw[m];
        ex.x = x;
        ex.nb = p.nb;
        ex.soa = p.soa;
        ex.bounds = B == 1;
        e = dq::splitk_reduce_launch(p.part, pl.splits, NS, B, N, y, p.g, p.qg_hd, p.grp, p.res, p.cand, ex,
                                     dq::reduce_grid(N, B), s);
        if (e != cudaSuccess)
            return cuda_fail(e);
    }
    if (argmax_out) {
        e = dq::argmax_finalize_launch(p.cand, ws.ncand, reinterpret_cast<long long *>(argmax_out), s);
        if (e != cudaSuccess)
            return cuda_fail(e);
    }
    return DQ_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for q4k_gemv_noalloc: a fixed device array in this library's own
// image, for callers that cannot allocate device memory themselves.  Every GPU
// that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
#define DQ_NOALLOC_SCRATCH_BYTES (4u << 20)
static __device__ __align__(256) uint8_t g_noalloc_scratch[DQ_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[64] = {};
CUcontext g_noalloc_ctx[64] = {};

// Device address of g_noalloc_scratch on the current device.  The symbol's
// host-side name is only a stand-in, so the address is looked up with the
// device current, once per device and context (a device reset makes a new
// context, and the next call looks the address up again), and cached.
dq_status noalloc_scratch(int device, void **ptr)
{
    if (device < 0 || device >= 64)
        return DQ_ERR_ARG;
    const CUcontext cur = dq::current_context();
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[device] || g_noalloc_ctx[device] != cur) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return cuda_fail(e);
        g_noalloc_ptr[device] = p;
        g_noalloc_ctx[device] = cur;
    }
    *ptr = g_noalloc_ptr[device];
    return DQ_OK;
}

}  // namespace

extern "C" {

dq_status q4k_gemv_noalloc(const void *w, int layout, const float *x, float *y, int64_t N, int64_t K, int B,
                           int64_t *argmax_out, void *stream)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e);
    void *scratch = nullptr;
    dq_status st = noalloc_scratch(dev, &scratch);
    if (st != DQ_OK)
        return st;
    return q4k_common(w, nullptr, layout, x, y, N, K, B, 1, argmax_out, scratch, DQ_NOALLOC_SCRATCH_BYTES, stream);
}

size_t dq_noalloc_scratch_bytes(void) { return DQ_NOALLOC_SCRATCH_BYTES; }

dq_status dq_test_lost_copy(const void *w, const float *x, float *y, int64_t N, int64_t K, uint64_t wait_ns,
                            void *workspace, size_t ws_bytes, void *stream)
{
    if (wait_ns < 1000 || wait_ns > dq::kWaitNanos)
        return DQ_ERR_ARG;
    return q4k_common(w, nullptr, DQ_LAYOUT_AOS, x, y, N, K, 1, 1, nullptr, workspace, ws_bytes, stream, nullptr, 0,
                      nullptr, nullptr, nullptr, static_cast<unsigned long long>(wait_ns), 1);
}


dq_status q4k_gemv(const void *w, int layout, const float *x, float *y, int64_t N, int64_t K, int B,
                   int64_t *argmax_out, void *workspace, size_t ws_bytes, void *stream)
{
    return q4k_common(w, nullptr, layout, x, y, N, K, B, 1, argmax_out, workspace, ws_bytes, stream);
}

dq_status q4k_ffn_block(const void *w_gate, const void *w_up, const void *w_down, int layout, const float *x,
                        const float *residual, float *y, int64_t H, int64_t F, int B, void *workspace, size_t ws_bytes,
                        void *stream)
{
    if (!w_gate || !w_up || !w_down || !x || !y)
        return DQ_ERR_NULL;
    if (layout != DQ_LAYOUT_AOS && layout != DQ_LAYOUT_SOA)
        return DQ_ERR_LAYOUT;
    dq_status st = check_q4k_shape(F, H, B);
    if (st != DQ_OK)
        return st;
    if ((st = check_q4k_shape(H, F, B)) != DQ_OK)
        return st;
    if (!aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) || !aligned(x, 16) || !aligned(y, 4) ||
        (residual && !aligned(residual, 4)))
        return DQ_ERR_ALIGN;
    // everything either GEMV could reject is checked here, before the first launch
    const size_t need = ffn_ws_bytes(H, F, B);
    if (need == static_cast<size_t>(-1))
        return DQ_ERR_SHAPE;
    if (!workspace || ws_bytes < need)
        return DQ_ERR_WORKSPACE;
    if (!aligned(workspace, 16))
        return DQ_ERR_ALIGN;
    const size_t hbytes = round_up(static_cast<size_t>(B) * F * sizeof(float), 256);
    float *h = static_cast<float *>(workspace);
    void *rest = static_cast<uint8_t *>(workspace) + hbytes;
    const size_t rest_bytes = ws_bytes - hbytes;
    st = q4k_common(w_gate, w_up, layout, x, h, F, H, B, 2, nullptr, rest, rest_bytes, stream);
    if (st != DQ_OK)
        return st;
    if (residual)
        return q4k_common(w_down, nullptr, layout, h, y, H, F, B, 1, nullptr, rest, rest_bytes, stream, nullptr, 0,
                          nullptr, nullptr, residual);
    return q4k_common(w_down, nullptr, layout, h, y, H, F, B, 1, nullptr, rest, rest_bytes, stream);
}

dq_status q4k_gemv_residual(const void *w, int layout, const float *x, const float *residual, float *y, int64_t N,
                            int64_t K, int B, int64_t *argmax_out, void *workspace, size_t ws_bytes, void *stream)
{
    if (!residual)
        return DQ_ERR_NULL;
    if (!aligned(residual, 4))
        return DQ_ERR_ALIGN;
    return q4k_common(w, nullptr, layout, x, y, N, K, B, 1, argmax_out, workspace, ws_bytes, stream, nullptr, 0,
                      nullptr, nullptr, residual);
}

dq_status q4k_prefill_gemm(const void *w, int layout, const uint16_t *x16, float *y, int64_t N, int64_t K, int64_t M,
                           void *workspace, size_t ws_bytes, void *stream)
{
    if (!w || !x16 || !y)
        return DQ_ERR_NULL;
    if (layout != DQ_LAYOUT_AOS && layout != DQ_LAYOUT_SOA)
        return DQ_ERR_LAYOUT;
    dq_status st = check_prefill_shape(N, K, M);
    if (st != DQ_OK)
        return st;
    if (!aligned(w, 16) || !aligned(x16, 16) || !aligned(y, 16))
        return DQ_ERR_ALIGN;
    DevInfo di;
    st = dev_info(di);
    if (st != DQ_OK)
        return st;
    if (!dq::tensor_map_encoder())
        return cuda_fail(cudaErrorNotSupported);
    const dq::PrefillPlan pl = dq::q4k_prefill_plan(N, static_cast<int>(K), M, di.sm_count, di.smem_optin);
    if (!pl.ok)
        return DQ_ERR_SHAPE;
    const size_t need = prefill_ws_bytes(pl, N, M);
    if (need > 0 && (!workspace || ws_bytes < need))
        return DQ_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 16))
        return DQ_ERR_ALIGN;
    const cudaError_t e = dq::q4k_prefill_launch(static_cast<const uint8_t *>(w), layout == DQ_LAYOUT_SOA, x16, y,
                                                 static_cast<float *>(workspace), dq::device_error_flag(di.device), N,
                                                 static_cast<int>(K), M, pl, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

dq_status q4k_gemv_split_qg(const void *w, int layout, const float *x, float *q, float *g, int64_t N, int64_t K,
                            int B, int64_t head_dim, void *workspace, size_t ws_bytes, void *stream)
{
    if (!q || !g)
        return DQ_ERR_NULL;
    if (head_dim < 1 || N < 2 || N % (2 * head_dim) != 0 || head_dim > (1LL << 30))
        return DQ_ERR_SHAPE;
    if (!aligned(g, 4))
        return DQ_ERR_ALIGN;
    // Q and G must not overlap: each is B x N/2 floats
    const uintptr_t qa = reinterpret_cast<uintptr_t>(q), ga = reinterpret_cast<uintptr_t>(g);
    const uintptr_t span = static_cast<uintptr_t>(B > 0 ? B : 0) * static_cast<uintptr_t>(N / 2) * sizeof(float);
    if (qa < ga + span && ga < qa + span)
        return DQ_ERR_ARG;
    return q4k_common(w, nullptr, layout, x, q, N, K, B, 1, nullptr, workspace, ws_bytes, stream, g, head_dim);
}

dq_status q4k_gemv_group(int count, const void *const *w, const int64_t *N, float *const *y, int layout,
                         const float *x, int64_t K, void *workspace, size_t ws_bytes, void *stream)
{
    if (!w || !N || !y)
        return DQ_ERR_NULL;
    if (count < 1 || count > dq::kMaxGroup)
        return DQ_ERR_ARG;
    dq::GroupOut grp{};
    grp.n = count;
    int64_t total = 0;
    for (int m = 0; m < count; ++m) {
        if (!w[m] || !y[m])
            return DQ_ERR_NULL;
        if (N[m] < 1 || N[m] > (int64_t(1) << 40))
            return DQ_ERR_SHAPE;
        if (!aligned(w[m], 16))
            return DQ_ERR_ALIGN;
        if (!aligned(y[m], 4))
            return DQ_ERR_ALIGN;
        grp.y[m] = y[m];
        grp.N[m] = N[m];
        grp.base[m] = total;
        // each matrix's rows are padded to the batch-1 kernel's row tile
        const int64_t tile = dq::q4k_fx_tile_rows();
        total += (N[m] + tile - 1) / tile * tile;
    }
    // y is only a stand-in here: every output goes through the group map
    return q4k_common(w[0], nullptr, layout, x, y[0], total, K, 1, 1, nullptr, workspace, ws_bytes, stream, nullptr, 0,
                      &grp, w);
}

dq_status q4k_swiglu_gemv(const void *w_gate, const void *w_up, int layout, const float *x, float *out, int64_t N,
                          int64_t K, int B, void *workspace, size_t ws_bytes, void *stream)
{
    if (!w_up)
        return DQ_ERR_NULL;
    return q4k_common(w_gate, w_up, layout, x, out, N, K, B, 2, nullptr, workspace, ws_bytes, stream);
}

dq_status q8_0_gemv(const void *w, const float *x, float *y, int64_t N, int64_t K, int B, void *workspace,
                    size_t ws_bytes, void *stream)
{
    (void)workspace;
    (void)ws_bytes;
    if (!w || !x || !y)
        return DQ_ERR_NULL;
    if (N < 1 || K < 32 || K % 32 != 0 || K > DQ_MAX_K || B < 1 || B > 8)
        return DQ_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(x, 16) || !aligned(y, 4))
        return DQ_ERR_ALIGN;
    DevInfo di;
    dq_status st = dev_info(di);
    if (st != DQ_OK)
        return st;
    const dq::Q8Plan pl = dq::q8_plan(N, static_cast<int>(K), B, di.sm_count, di.smem_optin);
    if (!pl.ok)
        return DQ_ERR_SHAPE;
    dq::Q8Params p{};
    p.w = static_cast<const uint8_t *>(w);
    p.x = x;
    p.y = y;
    p.err = dq::device_error_flag(di.device);
    p.N = N;
    p.K = static_cast<int>(K);
    p.nb = static_cast<int>(K / 32);
    cudaError_t e = dq::q8_0_gemv_launch(p, pl, B, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

dq_status q4k_repack_soa(const void *w_aos, void *w_soa, int64_t N, int64_t K, void *stream)
{
    if (!w_aos || !w_soa)
        return DQ_ERR_NULL;
    if (N < 1 || K < 256 || K % 256 != 0 || K > DQ_MAX_K)
        return DQ_ERR_SHAPE;
    if (!aligned(w_aos, 16) || !aligned(w_soa, 16))
        return DQ_ERR_ALIGN;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(w_aos), b0 = reinterpret_cast<uintptr_t>(w_soa);
    const uintptr_t bytes = static_cast<uintptr_t>(N) * static_cast<uintptr_t>(K / 256) * 144u;
    if (a0 < b0 + bytes && b0 < a0 + bytes)
        return DQ_ERR_ARG;
    cudaError_t e = dq::q4k_repack_soa_launch(static_cast<const uint8_t *>(w_aos), static_cast<uint8_t *>(w_soa), N,
                                              static_cast<int>(K), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

size_t dq_workspace_bytes(int op, int64_t N, int64_t K, int B, int with_argmax)
{
    const size_t bad = static_cast<size_t>(-1);
    if (op == DQ_OP_Q4K_FFN)
        return with_argmax ? bad : ffn_ws_bytes(N, K, B);
    if (op == DQ_OP_Q4K_PREFILL) {
        if (with_argmax || check_prefill_shape(N, K, B) != DQ_OK)
            return bad;
        DevInfo di;
        if (dev_info(di) != DQ_OK)
            return bad;
        const dq::PrefillPlan pl = dq::q4k_prefill_plan(N, static_cast<int>(K), B, di.sm_count, di.smem_optin);
        return pl.ok ? prefill_ws_bytes(pl, N, B) : bad;
    }
    if (op == DQ_OP_Q8_0_GEMV) {
        if (N < 1 || K < 32 || K % 32 != 0 || K > DQ_MAX_K || B < 1 || B > 8 || with_argmax)
            return bad;
        return 0;
    }
    if (op != DQ_OP_Q4K_GEMV && op != DQ_OP_Q4K_SWIGLU)
        return bad;
    const int NS = (op == DQ_OP_Q4K_SWIGLU) ? 2 : 1;
    if (with_argmax && (B != 1 || NS != 1))
        return bad;
    // the plan does not depend on the layout except through the chunk width,
    // so take the larger of the two requirements
    return q4k_gemv_ws_bytes(N, K, B, NS, with_argmax != 0);
}

dq_status q8_0_dequant(const void *w, float *out, int64_t N, int64_t K, void *stream)
{
    if (!w || !out)
        return DQ_ERR_NULL;
    if (N < 1 || K < 32 || K % 32 != 0 || K > DQ_MAX_K)
        return DQ_ERR_SHAPE;
    if (!aligned(w, 2) || !aligned(out, 4))
        return DQ_ERR_ALIGN;
    cudaError_t e = dq::q8_0_dequant_launch(static_cast<const uint8_t *>(w), out, N, static_cast<int>(K),
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

dq_status q4k_dequant(const void *w, int layout, float *out, int64_t N, int64_t K, void *stream)
{
    if (!w || !out)
        return DQ_ERR_NULL;
    if (layout != DQ_LAYOUT_AOS && layout != DQ_LAYOUT_SOA)
        return DQ_ERR_LAYOUT;
    if (N < 1 || K < 256 || K % 256 != 0 || K > DQ_MAX_K)
        return DQ_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(out, 4))
        return DQ_ERR_ALIGN;
    cudaError_t e = dq::q4k_dequant_launch(static_cast<const uint8_t *>(w), layout == DQ_LAYOUT_SOA, out, N,
                                           static_cast<int>(K), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

const char *dq_status_string(int status)
{
    switch (status) {
    case DQ_OK: return "DQ_OK";
    case DQ_ERR_NULL: return "DQ_ERR_NULL: a required pointer is NULL";
    case DQ_ERR_SHAPE: return "DQ_ERR_SHAPE: N, K or B outside the supported range";
    case DQ_ERR_ALIGN: return "DQ_ERR_ALIGN: a pointer is not suitably aligned";
    case DQ_ERR_WORKSPACE: return "DQ_ERR_WORKSPACE: workspace missing or too small";
    case DQ_ERR_LAYOUT: return "DQ_ERR_LAYOUT: unknown weight layout";
    case DQ_ERR_CUDA: return "DQ_ERR_CUDA: a CUDA runtime call failed";
    case DQ_ERR_ARG: return "DQ_ERR_ARG: invalid argument combination";
    default: return "unknown dq_status";
    }
}

int dq_last_cuda_error(void) { return g_last_cuda_error; }

dq_status dq_device_error(int *flag, int clear, void *stream)
{
    if (!flag)
        return DQ_ERR_NULL;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e);
    int *d = dq::device_error_flag(dev);
    if (!d)
        return cuda_fail(cudaErrorInvalidSymbol);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cuda_fail(e);
    e = cudaMemcpy(flag, d, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (clear) {
        e = cudaMemset(d, 0, sizeof(int));
        if (e != cudaSuccess)
            return cuda_fail(e);
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess)
            return cuda_fail(e);
    }
    return DQ_OK;
}

}  // extern "C"
