// q4k_prefill.cu -- W4A16 prefill GEMM for sm_100a: Y (M x N, fp32) = X (M x K,
// binary16) * W^T, with W an N x K Q4_K matrix, on the fifth-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory).
//
// The operation is the pages' batched-prefill projection with 4-bit weights and
// 16-bit activations (qualiaDB qwen3_attention: prefill_weights, "W4A16 M128
// dispatcher"); the pages give no more than its name and operand widths.  The
// reading taken: each weight is the Q4_K weight rounded to fp32 (the same value
// the dequantize entry point produces) and then to binary16, and the products
// of those binary16 weights with the binary16 activations are summed.
//
// Work decomposition.  A CTA owns a tile of 256 weight rows (the MMA's N) by
// up to 256 tokens (two accumulators of 128 tokens, the MMA's M; tokens past M
// are zeros from the TMA unit's out-of-bounds fill) and a range of K.  Putting
// the tokens on M keeps every MMA a full 128 x 256 x 16 operation even for a
// handful of tokens, so the issuing thread never limits the rate.  Per
// super-block the raw bytes of the 256 rows (36 KB) arrive by one TMA tile copy.
// Sixteen dequantizing warps, in two groups that take alternate stages, turn
// each quarter super-block (64 weights per row) into a 256 x 64 binary16 tile in the tensor cores' K-major, 128-byte swizzled
// shared-memory layout, while the activation tile(s) of the same 64 columns
// arrive by TMA in that same layout.  Every CTA starts its K range at a
// different super-block (rotated by its tile index), so that the CTAs, which
// all read the same activations, do not all ask L2 for the same tile at once.
// One thread issues four (or eight) MMAs per stage into the fp32 accumulators
// in tensor memory and, through tcgen05.commit, releases the stage when they
// have read it.  After the last stage the same sixteen warps read the
// accumulators back (tcgen05.ld) and store Y, or the split's partial sums when
// K is split across CTAs.
//
//   warp 0      weight TMA producer (one lane)
//   warp 1      tensor-memory allocation, MMA issue (one lane)
//   warp 2      activation TMA producer (one lane)
//   warp 3      idle
//   warps 4-19  dequantization, then the epilogue
//
// Dequantization of one weight: the GEMV's exact fp32 weight formation
// (q4k_decode.cuh: the quant read in place as a subnormal, one fma with the
// scaled d*scale and dmin*min, giving the fp32-rounded weight times 2^-64), a
// multiplication by 2^64 (exact), and cvt.rn to binary16.  So the tensor cores
// see exactly the binary16 rounding of the weights the dequantize entry point
// returns.
//
// All waits are bounded; a wait that runs out sets the device error flag and
// the shared abort word, every role then stops issuing work, waits (bounded)
// for its own copies and MMAs in flight, and the tensor memory is released.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "dq_common.cuh"
#include "dq_internal.h"
#include "q4k_decode.cuh"

namespace dq {

constexpr int kPfRows = 256;                              // weight rows per tile (MMA N)
constexpr int kPfTok = 128;                               // tokens per accumulator (MMA M)
constexpr int kPfK = 64;                                  // K per stage: one 128-byte row of binary16
constexpr int kPfRawBytes = kPfRows * kQ4KBlockBytes;     // one super-block of 256 rows: 36 KB
constexpr int kPfWTileBytes = kPfRows * kPfK * 2;         // 32 KB
constexpr int kPfXTileBytes = kPfTok * kPfK * 2;          // 16 KB
constexpr int kPfWarps = 20;
constexpr int kPfDqWarp0 = 4;                             // first dequantizing warp
constexpr int kPfDqWarps = kPfWarps - kPfDqWarp0;
constexpr int kPfMaxRaw = 4;                              // raw weight ring, super-blocks
constexpr int kPfMaxStages = 4;                           // operand ring, stages
constexpr int kPfEpiPitch = kPfRows + 4;                  // epilogue tile: floats per token row

struct PrefillMaps {
    CUtensorMap w;        // raw weight rows (AoS: 2-D bytes; SoA: 5-D gather of one block)
    CUtensorMap w_tail;   // SoA only: the last, partial group of each row
    CUtensorMap x;        // activations, binary16, 128-byte swizzle
};

// --- tcgen05 / TMA wrappers --------------------------------------------------

// Shared-memory matrix descriptor of a K-major operand tile in the 128-byte
// swizzled layout: rows of 128 bytes, 8-row groups 1024 bytes apart (stride
// byte offset), the leading byte offset unused for this layout (set to 16).
__device__ __forceinline__ uint64_t pf_desc_sw128(uint32_t saddr)
{
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(16 >> 4) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) /* descriptor version */ |
           (2ull << 61) /* 128-byte swizzle */;
}

__device__ __forceinline__ void pf_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void pf_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void pf_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void pf_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void pf_tma_2d(uint32_t dst, const CUtensorMap *m, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(m), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void pf_tma_5d(uint32_t dst, const CUtensorMap *m, int c0, int c1, int c2, int c3, int c4,
                                          uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
        "%6}], [%7];" ::"r"(dst),
        "l"(m), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
        : "memory");
}

// Eight consecutive fp32 accumulator columns of this warp's 32 lanes.
__device__ __forceinline__ void pf_tmem_ld8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
    for (int i = 0; i < 8; ++i)
        v[i] = __uint_as_float(r[i]);
}

// One try of an mbarrier phase wait that suspends the thread in hardware until
// the phase completes or kPfSleepNs pass, instead of returning at once: the
// waiting warps then take no issue slots and no shared-memory bandwidth from the
// single threads that issue the copies and the MMAs.
constexpr uint32_t kPfSleepNs = 10000000u;

__device__ __forceinline__ bool pf_try_wait_sleep(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kPfSleepNs)
        : "memory");
    return ok != 0;
}

// Bounded wait (kWaitNanos of the global timer in all) that also gives up once
// another role has aborted; a timeout sets the device error flag and the abort
// word.
__device__ __forceinline__ bool pf_wait(uint32_t bar, uint32_t parity, int *err, volatile int *abort)
{
    if (pf_try_wait_sleep(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 <= kWaitNanos) {
        if (abort && *abort)
            return false;
        if (pf_try_wait_sleep(bar, parity))
            return true;
    }
    atomicExch(err, kDevErrWaitTimeout);
    if (abort)
        *abort = 1;
    return false;
}

// Position in a ring of `depth` slots: the slot and the parity of the pass over
// the ring (the mbarrier phase a full-barrier wait expects; an empty-barrier
// wait on a later pass expects the other one).
struct Ring {
    int slot;
    uint32_t phase;
    int depth;
    __device__ __forceinline__ void next()
    {
        if (++slot == depth) {
            slot = 0;
            phase ^= 1u;
        }
    }
    __device__ __forceinline__ void prev()
    {
        if (slot == 0) {
            slot = depth;
            phase ^= 1u;
        }
        --slot;
    }
};

// Bounded wait for the single threads on the pipeline's critical path (the
// producers, the MMA issuer and the group leaders): mbarrier.try_wait with the
// system's own suspend limit, so that the thread resumes as soon as the phase
// completes.  Otherwise as pf_wait.
__device__ __forceinline__ bool pf_wait_fast(uint32_t bar, uint32_t parity, int *err, volatile int *abort)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 15) == 15) {
            if (abort && *abort)
                return false;
            if (global_ns() - t0 > kWaitNanos)
                break;
        }
    }
    atomicExch(err, kDevErrWaitTimeout);
    if (abort)
        *abort = 1;
    return false;
}

// pf_wait by lane 0 of a warp for the whole warp (one sleeping waiter instead of
// 32); the outcome is the same for every lane, and __syncwarp orders the lanes'
// later shared-memory accesses after lane 0's observation of the phase.
__device__ __forceinline__ bool pf_wait_warp(uint32_t bar, uint32_t parity, int *err, volatile int *abort)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0)
        ok = pf_wait(bar, parity, err, abort) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Two fp32 values -> one binary16 pair (round to nearest even), lo in bits 0..15.
__device__ __forceinline__ uint32_t pf_pack_f16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Binary16 weights of the 8 quant bytes of one row in `qv` (bytes 32c + 8e ..
// 32c + 8e + 7 of the super-block): lo holds the 8 low-nibble weights
// (k = 64c + 8e + 0..7), hi the 8 high-nibble weights (k = 64c + 32 + 8e + 0..7).
__device__ __forceinline__ void pf_dequant8(uint2 qv, const ChunkScales &cs, uint4 &lo, uint4 &hi)
{
    const float2 up = make_float2(0x1p64f, 0x1p64f);   // q4_word_weights forms w * 2^-64
    const uint32_t words[2] = {qv.x, qv.y};
    uint32_t plo[4], phi[4];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        float2 wv[4];   // {lo, hi} weights of bytes 4t .. 4t+3
        q4_word_weights(words[t], cs, wv);
#pragma unroll
        for (int b = 0; b < 4; ++b)
            wv[b] = __fmul2_rn(wv[b], up);
        plo[2 * t] = pf_pack_f16x2(wv[0].x, wv[1].x);
        plo[2 * t + 1] = pf_pack_f16x2(wv[2].x, wv[3].x);
        phi[2 * t] = pf_pack_f16x2(wv[0].y, wv[1].y);
        phi[2 * t + 1] = pf_pack_f16x2(wv[2].y, wv[3].y);
    }
    lo = make_uint4(plo[0], plo[1], plo[2], plo[3]);
    hi = make_uint4(phi[0], phi[1], phi[2], phi[3]);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

struct PrefillParams {
    float *out;        // Y (splits == 1) or the partial sums [splits][M][N]
    int *err;          // device error flag
    long long N;
    long long M;
    int nb;            // super-blocks per row (K / 256)
    int th;            // accumulators (token halves of 128) per CTA: 1 or 2
    int mtiles;        // token tiles of 128 * th
    int ntiles;        // weight-row tiles of 256
    int sb_per_split;
    int raw_depth;
    int depth;         // operand ring stages
    int soa;
    int soa_full;      // complete 4-block groups per row (SoA)
    uint32_t idesc;    // MMA instruction descriptor
    uint32_t tmem_cols;
};

__global__ void __launch_bounds__(kPfWarps * 32, 1)
    q4k_prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps maps)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_epi_bad;   // a dequantizing warp saw an abort before the epilogue
    __shared__ int s_go[4];
    __shared__ __align__(8) uint64_t s_bars[2 * (kPfMaxRaw + kPfMaxStages) + 1];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int SD = p.depth;
    const int RD = p.raw_depth;
    const int TH = p.th;
    const uint32_t x_bytes = static_cast<uint32_t>(TH) * kPfXTileBytes;
    const uint32_t stage_bytes = kPfWTileBytes + x_bytes;

    // stage slot s: [binary16 weight tile, 32 KB][activation tile(s), 16 KB each]
    const uint32_t st_s = (smem_u32(smem) + 1023u) & ~1023u;
    const uint32_t raw_s = st_s + SD * stage_bytes;                 // RD x 256 rows x 144 raw bytes
    const uint32_t raw_full = smem_u32(s_bars);
    const uint32_t raw_empty = raw_full + 8 * kPfMaxRaw;
    const uint32_t full = raw_empty + 8 * kPfMaxRaw;               // stage: weights formed + activations landed
    const uint32_t empty = full + 8 * kPfMaxStages;                // stage: MMAs done reading it
    const uint32_t acc_full = empty + 8 * kPfMaxStages;

    // tile: consecutive CTAs share one weight tile (mt fastest), then row tiles, then splits
    const int mt = static_cast<int>(blockIdx.x % p.mtiles);
    const int rest = static_cast<int>(blockIdx.x / p.mtiles);
    const int nt = rest % p.ntiles;
    const int split = rest / p.ntiles;
    const long long row0 = static_cast<long long>(nt) * kPfRows;
    const long long m0 = static_cast<long long>(mt) * kPfTok * TH;
    const int kb0 = split * p.sb_per_split;
    const int nsb = min(p.sb_per_split, p.nb - kb0);
    const int nst = 4 * nsb;
    const int rot = nt % nsb;   // first super-block of this CTA's K range, relative to kb0

    if (threadIdx.x == 0) {
        for (int i = 0; i < RD; ++i) {
            mbar_init(raw_full + 8 * i, 1);
            mbar_init(raw_empty + 8 * i, kPfDqWarps);
        }
        for (int i = 0; i < SD; ++i) {
            mbar_init(full + 8 * i, kPfDqWarps / 2 + 1);   // one arrival per warp of a group + the activation copy
            mbar_init(empty + 8 * i, 1);
        }
        mbar_init(acc_full, 1);
        s_abort = 0;
        s_epi_bad = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    pf_fence_before();
    __syncthreads();
    pf_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort = &s_abort;

    pdl_wait();
    pdl_launch_dependents();

    if (warp == 0) {
        // ---- weight producer: one TMA tile copy per super-block of the tile's rows
        if (lane == 0) {
            Ring r{0, 0, RD};
            int kbi = rot;    // super-block, relative to kb0
            int issued = 0;
            for (; issued < nsb; ++issued) {
                if (issued >= RD && !pf_wait_fast(raw_empty + 8 * r.slot, r.phase ^ 1, p.err, abort))
                    break;
                const uint32_t bar = raw_full + 8 * r.slot;
                const uint32_t dst = raw_s + r.slot * kPfRawBytes;
                const int kb = kb0 + kbi;
                mbar_arrive_expect_tx(bar, kPfRawBytes);
                if (!p.soa)
                    pf_tma_2d(dst, &maps.w, kb * kQ4KBlockBytes, static_cast<int>(row0), bar);   // x: 144 kb bytes
                else if (kb < 4 * p.soa_full)
                    pf_tma_5d(dst, &maps.w, 0, kb & 3, 0, kb >> 2, static_cast<int>(row0), bar);
                else
                    pf_tma_5d(dst, &maps.w_tail, 0, kb - 4 * p.soa_full, 0, 0, static_cast<int>(row0), bar);
                r.next();
                if (++kbi == nsb)
                    kbi = 0;
            }
            // own copies still in flight complete before the CTA may exit
            for (int u = 0; u < issued && u < RD; ++u) {
                r.prev();
                pf_wait(raw_full + 8 * r.slot, r.phase, p.err, nullptr);
            }
        }
    } else if (warp == 2) {
        // ---- activation producer: TH TMA tile copies (128 tokens x 64, swizzled) per stage, completing
        // on the stage's full barrier together with the dequantizing warps' arrivals
        if (lane == 0) {
            Ring r{0, 0, SD};
            int kbi = rot, quarter = 0;
            int issued = 0;
            for (; issued < nst; ++issued) {
                if (issued >= SD && !pf_wait_fast(empty + 8 * r.slot, r.phase ^ 1, p.err, abort))
                    break;
                const uint32_t bar = full + 8 * r.slot;
                const uint32_t dst = st_s + r.slot * stage_bytes + kPfWTileBytes;
                const int k = (kb0 + kbi) * kQ4KBlockElems + quarter * kPfK;
                mbar_arrive_expect_tx(bar, x_bytes);
                for (int t = 0; t < TH; ++t)
                    pf_tma_2d(dst + t * kPfXTileBytes, &maps.x, k, static_cast<int>(m0) + t * kPfTok, bar);
                r.next();
                if (++quarter == 4) {
                    quarter = 0;
                    if (++kbi == nsb)
                        kbi = 0;
                }
            }
            for (int u = 0; u < issued && u < SD; ++u) {
                r.prev();
                pf_wait(full + 8 * r.slot, r.phase, p.err, nullptr);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue: per stage and accumulator, four K = 16 steps (128 tokens x 256 rows each).
        // Descriptors advance by whole stages (and by 32 bytes per K step) in their 16-byte address field.
        if (lane == 0) {
            Ring r{0, 0, SD};
            const uint64_t w_desc0 = pf_desc_sw128(st_s);
            const uint64_t x_desc0 = pf_desc_sw128(st_s + kPfWTileBytes);
            const uint32_t idesc = p.idesc;
            for (int j = 0; j < nst; ++j) {
                if (!pf_wait_fast(full + 8 * r.slot, r.phase, p.err, abort))
                    break;
                pf_fence_after();
                const uint64_t soff = static_cast<uint64_t>(r.slot * (stage_bytes >> 4));
                for (int t = 0; t < TH; ++t) {
                    const uint64_t xd = x_desc0 + soff + static_cast<uint64_t>(t * (kPfXTileBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < kPfK / 16; ++kk)
                        pf_mma_f16(tmem + t * kPfRows, xd + 2 * kk, w_desc0 + soff + 2 * kk, idesc, (j | kk) != 0);
                }
                pf_commit(empty + 8 * r.slot);
                r.next();
            }
            // arrives once every MMA issued above has completed
            pf_commit(acc_full);
        }
    } else if (warp >= kPfDqWarp0) {
        // ---- dequantization: the sixteen warps form two groups of eight that take alternate stages
        // (group g the stages j with j % 2 == g, i.e. chunks g and g + 2 of each super-block), so
        // two stages are formed at once.  Warp d = warp - 4 of group g = d / 8 forms row
        // 32 (d % 8) + lane: all 32 quant bytes of the stage's chunk, written into the K-major
        // 128-byte swizzled weight tile (16-byte unit u of row r at position u ^ (r % 8) of the
        // row's 128 bytes; 8-row groups 1024 bytes apart): low nibbles are units 0-3, high
        // nibbles units 4-7.
        const int d = warp - kPfDqWarp0;
        const int g = d >> 3;
        const int r = 32 * (d & 7) + lane;
        const uint32_t row_off = static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128);
        const int sw = r & 7;
        // One leader thread per group waits on the mbarriers for the group's eight warps and passes
        // its outcome through s_go (two slots per group, alternating per barrier, so that a slot is
        // rewritten only after every warp of the group has read it); the warps meet at the group's
        // named hardware barrier, where waiting takes no issue slots.
        const bool leader = (d & 7) == 0 && lane == 0;
        int nb_sync = 0;
        auto gate = [&](uint32_t bar, uint32_t parity) -> bool {
            volatile int *go = s_go + 2 * g + (nb_sync & 1);
            if (leader)
                *go = pf_wait_fast(bar, parity, p.err, abort) ? 1 : 0;
            asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(kPfDqWarps * 16) : "memory");
            ++nb_sync;
            return *go != 0;
        };
        Ring rr{0, 0, RD}, rs{0, 0, SD};
        if (g == 1)
            rs.next();   // the group's first stage is stage 1
        int j = g;       // stage
        bool ok = true;
        for (int i = 0; i < nsb && ok; ++i) {
            if (!gate(raw_full + 8 * rr.slot, rr.phase))
                break;
            const uint32_t raw = raw_s + rr.slot * kPfRawBytes + r * kQ4KBlockBytes;
            const Hdr hd = decode_hdr(lds128(raw));
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = g + 2 * cc;
                if (j >= SD && !gate(empty + 8 * rs.slot, rs.phase ^ 1)) {
                    ok = false;
                    break;
                }
                const ChunkScales cs = chunk_scales(hd, c);
                const uint4 qa = lds128(raw + 16 + 32 * c);
                const uint4 qb = lds128(raw + 16 + 32 * c + 16);
                uint4 lo[4], hi[4];
                pf_dequant8(make_uint2(qa.x, qa.y), cs, lo[0], hi[0]);
                pf_dequant8(make_uint2(qa.z, qa.w), cs, lo[1], hi[1]);
                pf_dequant8(make_uint2(qb.x, qb.y), cs, lo[2], hi[2]);
                pf_dequant8(make_uint2(qb.z, qb.w), cs, lo[3], hi[3]);
                const uint32_t at = st_s + rs.slot * stage_bytes + row_off;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    sts128(at + ((u ^ sw) << 4), lo[u]);
                    sts128(at + (((4 + u) ^ sw) << 4), hi[u]);
                }
                fence_proxy_async_smem();   // generic-proxy stores -> visible to the tensor cores
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(full + 8 * rs.slot);   // one arrival per warp of the group
                rs.next();
                rs.next();
                j += 2;
            }
            if (!ok)
                break;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(raw_empty + 8 * rr.slot);
            rr.next();
        }

        // ---- epilogue, per accumulator: warp (q = warp % 4, e = d / 4) reads accumulator lanes
        // 32q .. 32q+31 (tokens) and columns 64e .. 64e+63 (weight rows) into a token-major tile in
        // the now idle rings (rows of 256 floats at a 260-float pitch); then warp d stores tokens
        // d, d + 16, ...: each token's 256 outputs are one contiguous run of Y (or of the split's
        // partial sums), written 512 bytes per instruction.  Every dequantizing warp passes both
        // named barriers; if any of them saw an abort, nothing is stored.
        const bool done = pf_wait_warp(acc_full, 0, p.err, nullptr);
        pf_fence_after();
        // tcgen05.ld is warp-collective: the whole warp reads, or none of it
        const bool ok_w = __all_sync(0xFFFFFFFFu, done && !*abort);
        if (!ok_w && lane == 0)
            s_epi_bad = 1;
        const int q = warp & 3;
        const int e = d >> 2;
        float *out = p.out + static_cast<long long>(split) * p.M * p.N;
        const bool vec = (p.N & 3) == 0;
        float *tile = reinterpret_cast<float *>(smem + (st_s - smem_u32(smem)));
        for (int t = 0; t < TH; ++t) {
            if (ok_w) {
                float *trow = tile + (32 * q + lane) * kPfEpiPitch;
                for (int c0 = 64 * e; c0 < 64 * e + 64; c0 += 8) {
                    float v[8];
                    pf_tmem_ld8(tmem + (static_cast<uint32_t>(32 * q) << 16) + t * kPfRows + c0, v);
                    reinterpret_cast<float4 *>(trow + c0)[0] = make_float4(v[0], v[1], v[2], v[3]);
                    reinterpret_cast<float4 *>(trow + c0)[1] = make_float4(v[4], v[5], v[6], v[7]);
                }
            }
            asm volatile("bar.sync 3, %0;" ::"n"(kPfDqWarps * 32) : "memory");
            if (!s_epi_bad) {
                for (int mm = d; mm < kPfTok; mm += kPfDqWarps) {
                    const long long m = m0 + t * kPfTok + mm;
                    if (m >= p.M)
                        break;
                    const float *trow = tile + mm * kPfEpiPitch;
                    float *o = out + m * p.N + row0;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c = 128 * h + 4 * lane;
                        const float4 v = reinterpret_cast<const float4 *>(trow + c)[0];
                        if (vec && row0 + c + 4 <= p.N) {
                            reinterpret_cast<float4 *>(o + c)[0] = v;
                        } else {
                            const float vv[4] = {v.x, v.y, v.z, v.w};
                            for (int u = 0; u < 4 && row0 + c + u < p.N; ++u)
                                o[c + u] = vv[u];
                        }
                    }
                }
            }
            // the tile is rewritten by the next accumulator only after every warp has stored it
            asm volatile("bar.sync 3, %0;" ::"n"(kPfDqWarps * 32) : "memory");
        }
    }

    pf_fence_before();
    __syncthreads();
    if (warp == 1) {
        pf_fence_after();
        // every MMA has completed once acc_full's phase 0 has (bounded; normally it has long since)
        pf_wait(acc_full, 0, p.err, nullptr);
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols)
                     : "memory");
    }
}

// Sum of the K-split partial sums, in split order: y[i] = sum_s part[s][i].
__global__ void __launch_bounds__(256) prefill_reduce_kernel(const float *part, int splits, long long count, float *y)
{
    pdl_wait();
    pdl_launch_dependents();
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const long long first = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if ((count & 3) == 0) {
        const long long n4 = count >> 2;
        const float4 *p4 = reinterpret_cast<const float4 *>(part);
        for (long long i = first; i < n4; i += stride) {
            const float4 a = __ldg(p4 + i);
            float ax = a.x, ay = a.y, az = a.z, aw = a.w;
            for (int s = 1; s < splits; ++s) {
                const float4 b = __ldg(p4 + s * n4 + i);
                ax += b.x;
                ay += b.y;
                az += b.z;
                aw += b.w;
            }
            reinterpret_cast<float4 *>(y)[i] = make_float4(ax, ay, az, aw);
        }
    } else {
        for (long long i = first; i < count; i += stride) {
            float a = part[i];
            for (int s = 1; s < splits; ++s)
                a += part[s * count + i];
            y[i] = a;
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Tiles of 256 weight rows by 128 tokens (M <= 128) or 256 tokens (two
// accumulators), one CTA per SM (the rings take most of shared memory).  K is
// split into the number of parts that minimises (waves of CTAs) x (super-blocks
// per CTA + a fixed cost of about six for the pipeline fill and the epilogue);
// ties go to fewer parts.  Rings: as many operand stages as fit next to two raw
// super-blocks, up to 4; the raw ring grows into what is left, up to 4.
PrefillPlan q4k_prefill_plan(long long N, int K, long long M, int sm_count, int smem_optin)
{
    PrefillPlan pl{};
    if (N < 1 || M < 1 || K < kQ4KBlockElems || K % kQ4KBlockElems != 0 || sm_count < 1 ||
        tensor_map_encoder() == nullptr)
        return pl;
    const int nb = K / kQ4KBlockElems;
    const int th = M <= kPfTok ? 1 : 2;
    const long long mtiles = (M + th * kPfTok - 1) / (th * kPfTok);
    const long long ntiles = (N + kPfRows - 1) / kPfRows;
    const long long tiles = ntiles * mtiles;
    int splits = 1, sbps = nb;
    long long best = -1;
    for (int s = 1; s <= nb && s <= 64; ++s) {
        const int per_split = (nb + s - 1) / s;
        const int used = (nb + per_split - 1) / per_split;
        const long long waves = (tiles * used + sm_count - 1) / sm_count;
        const long long cost = waves * (per_split + 6);
        if (best < 0 || cost < best) {
            best = cost;
            splits = used;
            sbps = per_split;
        }
    }
    if (tiles * splits > 0x7FFFFFFFLL)
        return pl;
    const int stage = kPfWTileBytes + th * kPfXTileBytes;
    const int budget = smem_optin - 1024 /*static shared memory*/ - 1024 /*alignment of the tiles*/;
    int depth = (budget - 2 * kPfRawBytes) / stage;
    if (depth > kPfMaxStages)
        depth = kPfMaxStages;
    if (depth < 2)
        return pl;
    int rd = (budget - depth * stage) / kPfRawBytes;
    if (rd > kPfMaxRaw)
        rd = kPfMaxRaw;
    // the epilogue stages one accumulator as a token-major tile in the rings
    if (depth * stage + rd * kPfRawBytes < kPfTok * kPfEpiPitch * 4)
        return pl;
    pl.th = th;
    pl.mtiles = static_cast<int>(mtiles);
    pl.ntiles = static_cast<int>(ntiles);
    pl.splits = splits;
    pl.sb_per_split = sbps;
    pl.raw_depth = rd;
    pl.depth = depth;
    pl.tmem_cols = 256 * th;
    pl.grid = static_cast<int>(tiles * splits);
    pl.smem = 1024 + depth * stage + rd * kPfRawBytes;
    pl.ok = true;
    return pl;
}

static cudaError_t encode(CUtensorMap *m, CUtensorMapDataType t, cuuint32_t rank, const void *base,
                          const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
                          CUtensorMapSwizzle swz)
{
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    const CUresult r = tensor_map_encoder()(m, t, rank, const_cast<void *>(base), dims, strides, box, es,
                                            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t q4k_prefill_launch(const uint8_t *w, int soa, const uint16_t *x16, float *y, float *part, int *err,
                               long long N, int K, long long M, const PrefillPlan &pl, cudaStream_t s)
{
    const int nb = K / kQ4KBlockElems;
    const cuuint64_t row = static_cast<cuuint64_t>(nb) * kQ4KBlockBytes;
    PrefillMaps maps;
    memset(&maps, 0, sizeof(maps));
    cudaError_t e = cudaSuccess;
    int soa_full = 0;
    if (!soa) {
        // raw rows as bytes: box = one super-block (144 bytes) of 256 rows
        const cuuint64_t dims[2] = {row, static_cast<cuuint64_t>(N)};
        const cuuint64_t strides[1] = {row};
        const cuuint32_t box[2] = {kQ4KBlockBytes, kPfRows};
        e = encode(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        // SoA group of g blocks: 16-byte piece u (0: header, 1..8: quant slices) of block t at
        // 64u... = 16 g u + 16 t.  Viewed as [row][group][u][t][16 bytes], a box of one t and all
        // nine u gathers one block back into its 144-byte AoS order.
        soa_full = nb / kQ4KSoaGroup;
        const cuuint32_t box[5] = {16, 1, 9, 1, kPfRows};
        if (soa_full > 0) {
            const cuuint64_t dims[5] = {16, kQ4KSoaGroup, 9, static_cast<cuuint64_t>(soa_full),
                                        static_cast<cuuint64_t>(N)};
            const cuuint64_t strides[4] = {16, 16 * kQ4KSoaGroup, kQ4KSoaGroup * kQ4KBlockBytes, row};
            e = encode(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, w, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
        }
        const int g = nb - soa_full * kQ4KSoaGroup;
        if (e == cudaSuccess && g > 0) {
            const cuuint64_t dims[5] = {16, static_cast<cuuint64_t>(g), 9, 1, static_cast<cuuint64_t>(N)};
            const cuuint64_t strides[4] = {16, static_cast<cuuint64_t>(16 * g),
                                           static_cast<cuuint64_t>(g * kQ4KBlockBytes), row};
            e = encode(&maps.w_tail, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5,
                       w + static_cast<size_t>(soa_full) * kQ4KSoaGroup * kQ4KBlockBytes, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
        }
    }
    if (e != cudaSuccess)
        return e;
    {
        // activations: box of 64 binary16 (128 bytes) x 128 tokens, 128-byte swizzle
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
        const cuuint32_t box[2] = {kPfK, kPfTok};
        e = encode(&maps.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess)
            return e;
    }
    PrefillParams p{};
    p.out = pl.splits > 1 ? part : y;
    p.err = err;
    p.N = N;
    p.M = M;
    p.nb = nb;
    p.th = pl.th;
    p.mtiles = pl.mtiles;
    p.ntiles = pl.ntiles;
    p.sb_per_split = pl.sb_per_split;
    p.raw_depth = pl.raw_depth;
    p.depth = pl.depth;
    p.soa = soa;
    p.soa_full = soa_full;
    // kind::f16 instruction descriptor: D fp32 (bits 4-5 = 1), A and B binary16 (bits 7-9, 10-12 = 0),
    // both K-major (bits 15, 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28; A = 128 tokens,
    // B = 256 weight rows
    p.idesc = (1u << 4) | (static_cast<uint32_t>(kPfRows >> 3) << 17) | (static_cast<uint32_t>(kPfTok >> 4) << 24);
    p.tmem_cols = static_cast<uint32_t>(pl.tmem_cols);
    e = cudaFuncSetAttribute(q4k_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess)
        return e;
    e = launch_pdl(q4k_prefill_kernel, dim3(pl.grid), dim3(kPfWarps * 32), pl.smem, s, p, maps);
    if (e != cudaSuccess || pl.splits == 1)
        return e;
    const long long count = M * N;
    long long blocks = (count / 4 + 255) / 256;
    if (blocks > 4LL * 148)
        blocks = 4LL * 148;
    if (blocks < 1)
        blocks = 1;
    return launch_pdl(prefill_reduce_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                      static_cast<const float *>(part), pl.splits, count, y);
}

}  // namespace dq
