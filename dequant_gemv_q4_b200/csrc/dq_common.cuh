// dq_common.cuh -- device helpers shared by the sm_100a kernels of libdqgemv.
//
// mbarrier + bulk-copy (cp.async.bulk, the TMA engine's 1-D form) wrappers,
// the bounded wait that replaces an unbounded spin, and the device error flag.
// Bulk copies here always read this GPU's own global memory into the issuing
// CTA's shared memory; no multicast form is used anywhere.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace dq {

constexpr int kQ4KBlockElems = 256;
constexpr int kQ4KBlockBytes = 144;
// Q4_K structure-of-arrays layout: groups of this many super-blocks, each
// group holding its headers and then its eight 16-byte quant slices.
constexpr int kQ4KSoaGroup = 4;
constexpr int kQ8BlockElems = 32;
constexpr int kQ8BlockBytes = 34;

// Address of GEMV output (b, n) for rows of length N: y[b][n]; or, with the
// fused Q/gate split (hd > 0; Doppler split_qg.wgsl), the de-interleaved place
// in Q (= y) or G, each B x N/2: row n = h*2*hd + d goes to Q[b][h*hd + d] when
// d < hd and to G[b][h*hd + d - hd] otherwise.
__device__ __forceinline__ float *gemv_out_addr(float *y, float *g, int hd, long long N, int b, long long n)
{
    if (hd == 0)
        return y + static_cast<long long>(b) * N + n;
    const long long hd2 = 2LL * hd;
    const long long h = n / hd2;
    const long long d = n - h * hd2;
    const long long base = static_cast<long long>(b) * (N / 2) + h * hd;
    return d < hd ? y + base + d : g + base + (d - hd);
}

// Error codes written to the device error flag.
constexpr int kDevErrWaitTimeout = 1;

// A wait for one of the kernel's own bulk copies is declared lost after this
// many nanoseconds of the global timer (a legitimate wait is microseconds), or
// after kWaitLimit polls, whichever comes first.
constexpr unsigned long long kWaitNanos = 2000000000ull;
constexpr uint32_t kWaitLimit = 1u << 26;

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Adds v to a shared-memory counter and returns its old value, ordered after
// this thread's earlier accesses (release) and before its later ones (acquire)
// at block scope.
__device__ __forceinline__ uint32_t atom_add_acq_rel_shared_u32(uint32_t addr, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}

// Programmatic dependent launch.  The GEMV-path kernels are launched with the
// programmatic stream-serialization attribute (launch_pdl below), so a grid may
// be scheduled while the previous kernel of the stream is still running: each
// such kernel calls pdl_wait() before its first global-memory access, which
// returns once the previous grid has completed and its writes are visible.
// pdl_launch_dependents() lets the next grid of the stream be scheduled early
// in the same way (it, too, waits before touching memory).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <class... KArgs, class... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async proxy (the bulk-copy unit).
__device__ __forceinline__ void mbar_fence_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of barrier `bar`: at most limit_ns of the
// global timer (and kWaitLimit polls).  Returns false (after setting the
// device error flag, when err is given) if the phase did not complete in time.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int *err,
                                                  unsigned long long limit_ns = kWaitNanos)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 63) == 63 && global_ns() - t0 > limit_ns)
            break;
    }
    if (err)
        atomicExch(err, kDevErrWaitTimeout);
    return false;
}

// Orders this thread's earlier generic-proxy shared-memory accesses before its
// later async-proxy ones (a bulk copy about to overwrite a consumed slot).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared, completing `bytes` of transaction count on
// barrier `bar`.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// An L2 policy under which the lines a load brings in are the first to be
// evicted: for data read once (the weights a GEMV streams), so that they do not
// push data that is read again (activations, outputs) out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// bulk_g2s with an L2 cache policy (l2_evict_first_policy).
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(pol)
        : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ float4 lds128f(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ float4 ldg_nc_f4(const float4 *p)
{
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// fp16 bit pattern -> fp32 (exact; subnormals included).
__device__ __forceinline__ float half_bits_to_float(uint32_t h)
{
    float f;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.f32.f16 %0, t; }" : "=f"(f) : "r"(h));
    return f;
}

// Argmax candidate: the largest value seen and its (lowest) index.
struct ArgmaxCand {
    float v;
    int pad;
    long long idx;
};

__device__ __forceinline__ bool cand_better(float v, long long i, float bv, long long bi)
{
    return v > bv || (v == bv && i < bi);
}

}  // namespace dq
