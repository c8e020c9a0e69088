// common.cuh -- shared definitions for the paged-attention kernels (sm_100a).
//
// Inline-PTX wrappers for the pieces of the Blackwell memory pipeline the
// kernels use: mbarriers with transaction counts, and bulk (TMA engine)
// copies from global to shared memory that complete on an mbarrier.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tfp {

// Device-side status bits (mirrors the public TF_DEV_* values).
constexpr uint32_t kDevBadLen = 1u;
constexpr uint32_t kDevBadPage = 2u;
constexpr uint32_t kDevTimeout = 4u;

// The workspace starts with a 256-byte header; word 0 is the status word.
constexpr size_t kWsHeaderBytes = 256;

// Per-device bookkeeping on the host (kernel attributes set once per device).
constexpr int kMaxDevices = 64;

// A pipeline wait gives up after this many SM clock cycles (about two
// seconds at B200 clocks; an internal error: every wait in these kernels is
// satisfied by work issued earlier in the same CTA).  The SM's own cycle
// counter is used because it only moves forward.  A call carries its limit
// in AttnParams::wait_limit (this value unless a test asks for a shorter
// one).
constexpr long long kWaitLimitCycles = 4000000000ll;

// Word 1 of the workspace header records which wait gave up (one bit per
// site), for diagnosis; word 0 is the status word.
enum WaitSite : uint32_t {
    kWaitFull = 1u, kWaitEmpty = 2u, kWaitQFull = 4u, kWaitQEmpty = 8u, kWaitFree = 16u,
    kWaitTag = 32u
};

struct AttnParams {
    const __nv_bfloat16 *k_pool;
    const __nv_bfloat16 *v_pool;
    const int32_t *table;
    const int32_t *lens;
    const __nv_bfloat16 *q;
    const uint8_t *tree;  // tree-verify row masks [S][W] (bit c: the row sees window row c), or null
    float *out;
    float *part;        // split-context partials (workspace past the header)
    uint32_t *flags;    // workspace status word
    int32_t n_pages, Hkv, P, D;
    int32_t table_stride, S, max_len;
    int32_t Hq, G, W, M;        // M = G * W query rows per (stream, KV head)
    int32_t RB, n_rblk;         // rows per row block, row blocks per (stream, KV head)
    int32_t SR;                 // rows per partial slot: min(RB, M)
    int32_t n_cta;              // persistent CTAs of the partial kernel (the work split)
    int32_t VT;                 // entry tiles of work in front of every unit
    int32_t whole;              // 1: CTA c takes unit c whole (no split, no partials)
    int32_t has_tree;           // 1: tree-verify call (the tree pointer holds the masks)
    // Test switch (0 in every library call): 1 makes CTA 0 withhold one
    // synchronous arrival that no copy or MMA completes -- the softmax warps'
    // P-ready arrival of their first tile (tensor-core kernels), or the
    // consumer's release of the first ring stage (CUDA-core kernel) -- so
    // that a bounded wait runs out and the failure path runs.
    int32_t withhold;
    long long wait_limit;       // cycles a pipeline wait may take (kWaitLimitCycles)
    long long *first_tile;      // workspace: where each stream's work starts in the launch
    long long *total_tiles;     // workspace: work tiles of the launch
    float scale_log2;           // scale * log2(e): scores are kept in log2 units
};

// Floats per partial slot: SR rows of O (D floats each), then SR running
// maxima and SR running sums, rounded up to 16 bytes so every slot (and every
// row of O in it) starts 16-byte aligned.
__host__ __device__ __forceinline__ size_t part_slot_floats(const AttnParams &p)
{
    return ((size_t)p.SR * (p.D + 2) + 3) & ~(size_t)3;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Counts `bytes` of the barrier's expected transaction bytes as arrived
// without a copy (a copy that is not made).
__device__ __forceinline__ void mbar_complete_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete; false after the
// time limit (the caller records kDevTimeout and winds down).  A phase that
// has already completed costs one non-blocking test.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          long long limit = kWaitLimitCycles)
{
    if (mbar_test_wait(bar, parity))
        return true;
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 255u) == 0 && clock64() - t0 > limit)
            return false;
    }
}

// Bulk copy (TMA engine, no tensor map) of `bytes` from global to this
// CTA's shared memory; completion is counted on `bar` in bytes.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Bulk copy (TMA engine) of `bytes` from this CTA's shared memory to global
// memory, in the issuing thread's current bulk group.  Both addresses 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(static_cast<uint32_t>(__cvta_generic_to_shared(src))), "r"(bytes)
                 : "memory");
}

// Closes the issuing thread's current bulk group.
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Waits until at most N of the thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Waits until all of the thread's bulk groups are complete (writes performed).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// L2 policy for data read once per call (K/V streams): evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// max(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Maximum of v[0 .. N) (N >= 4, N even) in four independent chains of
// three-input maxima: N / 2 instructions, a dependency depth of about N / 8.
template <int N>
__device__ __forceinline__ float max_tree(const float (&v)[N])
{
    static_assert(N >= 4 && N % 2 == 0, "max_tree");
    float c[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
    for (int k = 4; k < N; k += 2)
        c[(k / 2) & 3] = fmax3(c[(k / 2) & 3], v[k], v[k + 1]);
    return fmaxf(fmax3(c[0], c[1], c[2]), c[3]);
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// bf16 pair (packed in a 32-bit word, low element first) to two floats.
// bf16 is the upper half of an IEEE binary32, so widening is a shift/mask.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void named_barrier(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Lets the next kernel in the stream, if it was launched as a programmatic
// dependent (the merge), be scheduled now; it waits for this grid itself.
__device__ __forceinline__ void allow_dependent_launch()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Waits until the previous kernel in the stream has completed and its writes
// are visible, when this grid was launched as its programmatic dependent (a
// no-op otherwise).  Nothing a previous kernel may have written (lens, tables,
// pools, queries) is read before it.
__device__ __forceinline__ void wait_prior_grid()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void set_flag(uint32_t *flags, uint32_t bit)
{
    atomicOr(flags, bit);
}

}  // namespace tfp
