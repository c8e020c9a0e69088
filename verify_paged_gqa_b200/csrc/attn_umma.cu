// attn_umma.cu -- split-context paged attention on the 5th-generation tensor
// cores (tcgen05 / TMEM) for row blocks of up to 128 query rows: draft-verify
// windows and chunked prompt rows, head dim 128.
//
// TensorFold #1620 ("Kolibri-1's full layers take their K/V from pages of
// the core pool"), opening comment, "Reads": prompt rows and drafted verify
// rows attend over keys read through the page table; TensorFold #2730 ("an
// eight-row verify window"), "What this changes": a window holds up to eight
// rows.  With G query heads per KV head and W window rows, the G * W rows of
// one (stream, KV head) form a dense tile that shares every K and V row, so
// QK^T and PV run as tensor-core MMAs here.
//
// One persistent CTA per SM, six warps:
//   warp 0     producer (one lane): for each 64-position tile, one page id
//              (read one page early) and four TMA loads (K and V, two
//              64-dim halves each, 128-byte swizzle) into a 7-stage ring.
//   warp 1     MMA issuer (one lane): S = Q K^T (M 128, N 64, K 128) into
//              one of two TMEM S buffers; O += P_hi V + P_lo V (M 128, N 128,
//              K 64) into the TMEM O accumulator.  Also owns the TMEM
//              allocation, and zeroes V rows past the stream's end before PV
//              (so no NaN from unused slots reaches the MMA: 0 * NaN = NaN).
//   warps 2-5  softmax (one query row per thread, the row's TMEM lane): write
//              the row's query into the swizzled Q tile at the start of each
//              segment; per tile, read the S row from TMEM, select masked
//              positions to -inf, update the running max m and sum l in log2
//              units, and write P into TMEM as two bf16 parts (P = hi + lo,
//              each the truncated upper half of a float, so the PV product
//              keeps ~15 bits of each probability, close to the fp32 CUDA
//              core path).  Q and P live in TMEM and both MMAs
//              read their A operand from there, so shared memory holds only
//              the K/V ring (7 stages).  O in TMEM is rescaled only when the row max
//              grows by more than 2^8 (exact: the final O / l does not depend
//              on the reference max).  At the end of the segment the row is
//              normalised and stored, or left as a partial for the merge.
#include "launch.cuh"
#include "plan.cuh"
#include "umma.cuh"

namespace tfp {

namespace {

constexpr int UD = 128;        // head dim of this kernel
constexpr int UM = 128;        // MMA rows (the row block, padded)
constexpr int UN = 128;        // positions per tile
constexpr int NST = 3;         // K/V ring stages (64 KB each)
constexpr int kUmmaThreads = 192;
constexpr float kRescaleLog2 = 8.f;  // rescale O only when the max grows by more

// Shared memory (SW128 regions are 1024-byte aligned).
struct UmmaSmem {
    // per stage: K half 0, K half 1, V half 0, V half 1; each [128 pos][64 dims] bf16
    alignas(1024) uint8_t kv[NST][4][UN * 128];
    uint64_t kv_full[NST];
    uint64_t kv_empty[NST];
    uint64_t q_full;       // softmax warps wrote the segment's Q tile
    uint64_t q_free;       // the segment's last QK MMA is done with Q
    uint64_t s_full[2];
    uint64_t p_full[2];    // softmax warps wrote P into buffer b
    uint64_t o_done[2];    // the PV reading P buffer b finished (and every MMA before it)
    uint64_t fin;          // every MMA this CTA issued has completed
    CtaRange range;        // this CTA's tiles
    uint32_t tmem_base;
    volatile int abort_flag;
};

constexpr size_t kUmmaSmemBytes = sizeof(UmmaSmem) + 1024;  // + alignment slack

struct UmmaArgs {
    AttnParams p;
    CUtensorMap kmap;
    CUtensorMap vmap;
};

__device__ __forceinline__ bool uwait(UmmaSmem &sm, uint64_t *bar, uint32_t parity, uint32_t *flags,
                                      uint32_t site)
{
    if (sm.abort_flag)
        return false;
    if (mbar_wait(bar, parity))
        return true;
    set_flag(flags, kDevTimeout);
    set_flag(flags + 1, site);
    sm.abort_flag = 1;
    return false;
}

// ---- roles -------------------------------------------------------------------

__device__ __forceinline__ void umma_producer(const UmmaArgs &a, UmmaSmem &sm)
{
    const AttnParams &p = a.p;
    const uint64_t pol = l2_evict_first_policy();
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it, nx;
    uint32_t T = 0;
    bool have = cur.next(p, it);
    int32_t page_next = have ? __ldg(p.table + (int64_t)it.s * p.table_stride + it.key0 / p.P) : 0;
    while (have && !sm.abort_flag) {
        SegCursor ahead = cur;
        const bool have_nx = ahead.next(p, nx);
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        const int lp_end = (it.key1 + p.P - 1) / p.P;
        for (int lp = it.key0 / p.P; lp < lp_end && !sm.abort_flag; ++lp) {
            const int32_t page = page_next;
            if (lp + 1 < lp_end)
                page_next = __ldg(trow + lp + 1);
            else if (have_nx)
                page_next = __ldg(p.table + (int64_t)nx.s * p.table_stride + nx.key0 / p.P);
            const bool page_ok = page >= 0 && page < p.n_pages;
            if (!page_ok)
                set_flag(p.flags, kDevBadPage);
            const int pos0 = max(it.key0, lp * p.P);
            const int pos1 = min(it.key1, (lp + 1) * p.P);
            const int row0 = ((page_ok ? page : 0) * p.Hkv + it.kh) * p.P - lp * p.P;
            for (int t0 = pos0; t0 < pos1; t0 += UN, ++T) {
                const int st = T % NST;
                if (!uwait(sm, &sm.kv_empty[st], ((T / NST) & 1u) ^ 1u, p.flags, kWaitEmpty))
                    break;
                if (page_ok) {
                    mbar_arrive_expect_tx(&sm.kv_full[st], 4u * UN * 128u);
                    const int y = row0 + t0;
                    tma_load_2d(sm.kv[st][0], &a.kmap, 0, y, &sm.kv_full[st], pol);
                    tma_load_2d(sm.kv[st][1], &a.kmap, 64, y, &sm.kv_full[st], pol);
                    tma_load_2d(sm.kv[st][2], &a.vmap, 0, y, &sm.kv_full[st], pol);
                    tma_load_2d(sm.kv[st][3], &a.vmap, 64, y, &sm.kv_full[st], pol);
                } else {
                    mbar_arrive(&sm.kv_full[st]);
                }
            }
        }
        have = have_nx;
        it = nx;
        cur = ahead;
    }
    if (sm.abort_flag) {
        const uint32_t n = T < (uint32_t)NST ? T : (uint32_t)NST;
        for (uint32_t k = 1; k <= n; ++k) {
            const uint32_t t = T - k;
            (void)mbar_wait(&sm.kv_full[t % NST], (t / NST) & 1u);
        }
    }
}

// Tensor-memory columns (448 used of 512):
//   [0, 256)    two S buffers of 128 fp32 columns.  Once the softmax has read
//               the 32 columns of S(t) for positions 32c..32c+31, it writes
//               P_hi of those positions (16 columns of bf16 pairs) and P_lo
//               (16 more) over them; PV(t) reads them there, and QK(t+2)
//               overwrites the buffer only after PV(t) in the MMA's issue
//               order.  S and P are thus both double-buffered.
//   [256, 384)  O, fp32
//   [384, 448)  Q, the row's 128 query dims as bf16 pairs
constexpr uint32_t kColSP = 0;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColQ = 384;
constexpr uint32_t kTmemCols = 512;

// Column of the P part (0: hi, 1: lo) holding positions 16s..16s+15.
__host__ __device__ constexpr uint32_t p_col(int s, int part)
{
    return (uint32_t)(32 * (s >> 1) + 16 * part + 8 * (s & 1));
}

// One lane runs this: the ring's only consumer, in order, so its parity
// waits are unambiguous.  It does as little as possible between MMA batches:
// the tensor pipe takes a tcgen05.mma about every 100 cycles and idles
// whenever this thread does anything else.
// MR is the MMA's M: 128, or 64 for row blocks of at most 64 rows (their
// accumulator rows sit in lanes m % 16 + 32 * (m / 16) of tensor memory).
template <int MR>
__device__ __forceinline__ void umma_issuer(const UmmaArgs &a, UmmaSmem &sm)
{
    const AttnParams &p = a.p;
    const uint32_t tmem = sm.tmem_base;
    constexpr uint32_t idQK = f16_idesc(MR, UN, 0, 0);
    constexpr uint32_t idPV = f16_idesc(MR, UD, 0, 1);
    const uint32_t kv0 = smem_addr(sm.kv[0][0]);
    constexpr uint32_t kHalf = UN * 128;          // one [UN][64] bf16 box
    constexpr uint32_t kStageBytes = 4 * kHalf;

    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t T0 = 0, j = 0;
    bool ok = true;
    for (; cur.next(p, it); ++j) {
        const int ntiles = (it.key1 - it.key0 + UN - 1) / UN;
        ok = ok && uwait(sm, &sm.q_full, j & 1u, p.flags, kWaitQFull);
        tc_fence_after();
        auto issue_qk = [&](int t) {
            const uint32_t T = T0 + t;  // CTA-wide tile count (S / P buffer phases too)
            const int st = T % NST;
            ok = ok && uwait(sm, &sm.kv_full[st], (T / NST) & 1u, p.flags, kWaitFull);
            tc_fence_after();
            if (!ok)
                return;
            // positions past the stream's end: zero those V rows (both halves)
            const int tpos = it.key0 + t * UN;
            const int nvalid = min(UN, it.len - tpos);
            if (nvalid < UN) {
                for (int r = nvalid; r < UN; ++r)
                    for (int c = 0; c < 8; ++c) {
                        *reinterpret_cast<uint4 *>(sm.kv[st][2] + sw128_off(r, c)) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(sm.kv[st][3] + sw128_off(r, c)) = make_uint4(0, 0, 0, 0);
                    }
                fence_async_smem();
            }
            const uint32_t ka = kv0 + st * kStageBytes;
#pragma unroll
            for (int s = 0; s < UD / 16; ++s) {
                const uint32_t koff = (uint32_t)((s >> 2) * kHalf + (s & 3) * 32);
                umma_f16_ts(tmem + kColSP + 128 * (T & 1), tmem + kColQ + s * 8,
                            sw128_desc(ka + koff, 16, 1024), idQK, s > 0);
            }
            umma_commit(&sm.s_full[T & 1]);
            if (t == ntiles - 1)
                umma_commit(&sm.q_free);
        };
        issue_qk(0);
        for (int t = 0; t < ntiles; ++t) {
            const uint32_t T = T0 + t;
            const int st = T % NST;
            if (t + 1 < ntiles)
                issue_qk(t + 1);
            ok = ok && uwait(sm, &sm.p_full[T & 1], (T >> 1) & 1u, p.flags, kWaitQEmpty);
            tc_fence_after();
            if (ok) {
                const uint32_t va = kv0 + st * kStageBytes + 2 * kHalf;
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint32_t tp = tmem + kColSP + 128 * (T & 1);
#pragma unroll
                    for (int s = 0; s < UN / 16; ++s)
                        umma_f16_ts(tmem + kColO, tp + p_col(s, part),
                                    sw128_desc(va + s * 2048, kHalf, 1024), idPV,
                                    (t > 0 || part > 0 || s > 0) ? 1u : 0u);
                }
                umma_commit(&sm.o_done[T & 1]);
                umma_commit(&sm.kv_empty[st]);
            }
        }
        T0 += ntiles;
    }
    // every MMA issued by this thread has completed once `fin` flips
    umma_commit(&sm.fin);
    (void)mbar_wait(&sm.fin, 0);
}

// Softmax warpgroup: one query row per thread (the row's TMEM lane).  With
// MR = 64 only lanes 0-15 of each warp hold rows (row 16 * (warp % 4) + lane).
template <int MR>
__device__ __forceinline__ void umma_softmax(const UmmaArgs &a, UmmaSmem &sm, int warp, int lane)
{
    const AttnParams &p = a.p;
    const int row = MR == 128 ? (warp & 3) * 32 + lane : (warp & 3) * 16 + (lane & 15);
    const bool lane_rows = MR == 128 || lane < 16;
    const uint32_t lane_base = sm.tmem_base + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t tO = lane_base + kColO;
    const float NEG_INF = -__int_as_float(0x7f800000);

    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t j = 0, tt = 0;
    for (; cur.next(p, it); ++j) {
        const int m = it.b * MR + row;
        const bool live = lane_rows && m < p.M;
        const int lim = row_lim(p, it.len, m);
        // the first row of the block sees the fewest positions
        const int lim_lo = row_lim(p, it.len, it.b * MR);
        // --- the row's query into the swizzled Q tile ----------------------
        bool ok;
        {
            // load the row first (overlaps the wait for the previous segment's last QK)
            const int mm = min(m, p.M - 1);
            const int wr = mm / p.G;
            const int h = it.kh * p.G + (mm - wr * p.G);
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.q + (((size_t)it.s * p.W + wr) * p.Hq + h) * UD);
            uint32_t qr[2][32];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 v = live ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                qr[c >> 3][(c & 7) * 4 + 0] = v.x;
                qr[c >> 3][(c & 7) * 4 + 1] = v.y;
                qr[c >> 3][(c & 7) * 4 + 2] = v.z;
                qr[c >> 3][(c & 7) * 4 + 3] = v.w;
            }
            ok = uwait(sm, &sm.q_free, (j & 1u) ^ 1u, p.flags, kWaitQEmpty);
            tc_fence_after();
            tmem_st32(lane_base + kColQ, qr[0]);
            tmem_st32(lane_base + kColQ + 32, qr[1]);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.q_full);

        float m_run = NEG_INF, l_run = 0.f;
        const int ntiles = (it.key1 - it.key0 + UN - 1) / UN;
        for (int t = 0; t < ntiles; ++t) {
            const uint32_t u = tt + t;
            const int tpos = it.key0 + t * UN;
            const uint32_t tS = lane_base + kColSP + 128 * (u & 1);
            ok = uwait(sm, &sm.s_full[u & 1], (u >> 1) & 1u, p.flags, kWaitFull) && ok;
            tc_fence_after();
            // a tile every row of the block sees whole needs no mask; in a
            // partial tile a row sees positions [tpos, vis_end)
            const bool whole = tpos + UN <= lim_lo && tpos + UN <= it.key1;
            const int vis_n = live ? max(0, min(min(lim, it.key1) - tpos, UN)) : 0;
            const float sl = p.scale_log2;
            // pass 1: the tile's row max (log2 units)
            float tmax = NEG_INF;
#pragma unroll
            for (int c = 0; c < UN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tS + 32 * c, r);
                tmem_wait_ld();
                float m0 = NEG_INF, m1 = NEG_INF;
                if (whole) {
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        m0 = fmaxf(m0, __uint_as_float(r[e]));
                        m1 = fmaxf(m1, __uint_as_float(r[e + 1]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        m0 = fmaxf(m0, 32 * c + e < vis_n ? __uint_as_float(r[e]) : NEG_INF);
                        m1 = fmaxf(m1, 32 * c + e + 1 < vis_n ? __uint_as_float(r[e + 1]) : NEG_INF);
                    }
                }
                tmax = fmaxf(tmax, fmaxf(m0, m1));
            }
            tmax = (live && tmax != NEG_INF) ? tmax * sl : NEG_INF;
            // a new reference max only when the row max grows by more than 2^8
            const bool grow = tmax > m_run + kRescaleLog2 || (m_run == NEG_INF && tmax != NEG_INF);
            const float m_new = grow ? tmax : m_run;
            const float m_use = m_new == NEG_INF ? 0.f : m_new;
            const float alpha = fast_exp2(m_run - m_use);   // 0 when m_run is -inf
            const bool need = grow && t > 0 && m_run != NEG_INF;
            if (__any_sync(0xffffffffu, need)) {   // warp-collective TMEM traffic
                // S(u) is in, so PV(u - 2) is done (MMAs complete in issue
                // order): this wait for PV(u - 1) cannot alias an older phase
                ok = uwait(sm, &sm.o_done[(u - 1) & 1], ((u - 1) >> 1) & 1u, p.flags, kWaitEmpty) && ok;
                tc_fence_after();
                const float f = need ? alpha : 1.f;
#pragma unroll 1
                for (int c = 0; c < UD / 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(tO + c * 16, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
                    tmem_st16(tO + c * 16, r);
                }
                tmem_wait_st();
            }
            if (grow)
                l_run *= alpha;
            m_run = m_new;
            // pass 2: P = exp2(s * scale - m) as hi + lo bf16 parts, written over
            // the S chunk just read (hi to columns 32c..32c+15, lo after it)
            float lsum0 = 0.f, lsum1 = 0.f;
            const float neg_m = -m_use;
#pragma unroll
            for (int c = 0; c < UN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tS + 32 * c, r);
                tmem_wait_ld();
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float x0 = fmaf(__uint_as_float(r[2 * e]), sl, neg_m);
                    float x1 = fmaf(__uint_as_float(r[2 * e + 1]), sl, neg_m);
                    if (!whole) {
                        x0 = 32 * c + 2 * e < vis_n ? x0 : NEG_INF;
                        x1 = 32 * c + 2 * e + 1 < vis_n ? x1 : NEG_INF;
                    }
                    const float p0 = fast_exp2(x0);
                    const float p1 = fast_exp2(x1);
                    lsum0 += p0;
                    lsum1 += p1;
                    // P = hi + lo, both bf16 by truncation (upper 16 bits):
                    // |p - hi - lo| < 2^-14 p.  Packed with byte permutes.
                    const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
                    hi[e] = __byte_perm(b0, b1, 0x7632);
                    const float r0 = p0 - __uint_as_float(b0 & 0xffff0000u);
                    const float r1 = p1 - __uint_as_float(b1 & 0xffff0000u);
                    lo[e] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
                }
                tmem_st16(tS + 32 * c, hi);
                tmem_st16(tS + 32 * c + 16, lo);
            }
            const float lsum = lsum0 + lsum1;
            tmem_wait_st();
            l_run += lsum;
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.p_full[u & 1]);
        }
        // --- the segment's last PV, then the row's result ----------------------
        const uint32_t ulast = tt + ntiles - 1;
        ok = uwait(sm, &sm.o_done[ulast & 1], (ulast >> 1) & 1u, p.flags, kWaitEmpty) && ok;
        tc_fence_after();
        const bool write = live && ok && !sm.abort_flag;
        float *dst = nullptr;
        float sc = 1.f;
        if (write) {
            if (it.fin) {
                const int wr = m / p.G;
                const int h = it.kh * p.G + (m - wr * p.G);
                dst = p.out + (((size_t)it.s * p.W + wr) * p.Hq + h) * UD;
                sc = 1.f / l_run;
            } else {
                float *slot =
                    p.part + (size_t)it.slot * (p.SR * (UD + 2));
                dst = slot + (size_t)row * UD;
                slot[(size_t)p.SR * UD + row] = m_run;
                slot[(size_t)p.SR * UD + p.SR + row] = l_run;
            }
        }
#pragma unroll 1
        for (int c = 0; c < UD / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(tO + c * 16, r);   // warp-collective: every lane loads
            tmem_wait_ld();
            if (write) {
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4 *>(dst + c * 16 + e) =
                        make_float4(__uint_as_float(r[e]) * sc, __uint_as_float(r[e + 1]) * sc,
                                    __uint_as_float(r[e + 2]) * sc, __uint_as_float(r[e + 3]) * sc);
            }
        }
        tc_fence_before();
        tt += ntiles;
    }
}

template <int MR>
__global__ void __launch_bounds__(kUmmaThreads, 1) attn_umma_kernel(const __grid_constant__ UmmaArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    UmmaSmem &sm = *reinterpret_cast<UmmaSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
        }
        mbar_init(&sm.q_full, 4);
        mbar_init(&sm.q_free, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.s_full[s], 1);
            mbar_init(&sm.p_full[s], 4);
            mbar_init(&sm.o_done[s], 1);
        }
        mbar_init(&sm.fin, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0)
        find_range(a.p, sm.range, lane);
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&sm.tmem_base)), "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        if (lane == 0)
            umma_producer(a, sm);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0)
            umma_issuer<MR>(a, sm);
        __syncwarp();
    } else {
        umma_softmax<MR>(a, sm, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sm.tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

// Rows of a row block.  (An M = 64 MMA costs about as much time as M = 128
// on this hardware, so small row counts are padded to 128.)
int umma_rows(int64_t) { return UM; }

// Tiles stay inside a page.
bool umma_supported(const AttnParams &p) { return p.D == UD && p.P % UN == 0 && pool_rows_fit(p); }

cudaError_t launch_attn_umma(const AttnParams &p, int grid, cudaStream_t stream)
{
    UmmaArgs a;
    a.p = p;
    if (!make_pool_map(&a.kmap, p.k_pool, p, UN) || !make_pool_map(&a.vmap, p.v_pool, p, UN))
        return cudaErrorInvalidValue;
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        for (auto fn : {attn_umma_kernel<64>, attn_umma_kernel<128>}) {
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kUmmaSmemBytes);
            if (e != cudaSuccess)
                return e;
        }
        configured[dev] = true;
    }
    if (p.RB == 64)
        attn_umma_kernel<64><<<grid, kUmmaThreads, kUmmaSmemBytes, stream>>>(a);
    else
        attn_umma_kernel<128><<<grid, kUmmaThreads, kUmmaSmemBytes, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tfp
