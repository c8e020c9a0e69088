// attn_prompt.cu -- split-context paged attention on the 5th-generation
// tensor cores for row blocks of 128 query rows at head dim 128: chunked
// prompt rows (and any call with more than 64 rows per KV head).
//
// TensorFold #1620 ("Kolibri-1's full layers take their K/V from pages of
// the core pool"), opening comment, "Reads": prompt rows attend over keys
// read through the page table, causally.  Such a block is tensor bound.  Per
// 128-position tile the kernel issues 16 MMAs, which the tensor pipe runs at
// its peak rate in 1,536 cycles (N / 2 cycles per K = 16 step at M = 128):
//
//   S    = Q K^T                  M = 128 rows, N = 128 positions, 8 MMAs,
//                                 Q in tensor memory
//   O^T += V^T [P_hi ; P_lo]^T    M = 128 dims, N = 256 (P_hi rows, then
//                                 P_lo rows), 8 MMAs, P in shared memory as
//                                 the K-major B operand
//
// P = hi + lo (each the truncated upper half of a float) keeps about 15 bits
// of every probability; the two halves land in separate O^T columns that the
// epilogue adds.  16 instructions per tile instead of 24 for a row-major PV
// run once per half.
//
// One persistent CTA per SM, ten warps:
//   warp 0     producer (one lane): the K/V ring (ring.cuh).
//   warp 1     MMA issuer (one lane): QK(t + 1) before PV(t).  S has one
//              tensor-memory buffer: QK(t + 1) starts once the softmax has
//              read S(t) into registers.  Owns the tensor-memory allocation.
//   warps 2-9  softmax, two threads per query row (its lane of S), one per
//              64-position half of the tile: per tile, read the half's 64
//              scores, mask, and compare the half's max with the row's
//              reference max; a block-wide vote moves the references of rows
//              whose max grew by more than 2^8 (and then the O^T columns are
//              rescaled).  Write the half row of P into the shared P tile;
//              keep the half row's sum.  At a segment's end the same threads
//              read O^T by head dim (their lane) and store the rows, or leave
//              partials for the merge.
#include "launch.cuh"
#include "ring.cuh"

namespace tfp {

namespace {

constexpr int PT = kRingTile;          // positions per tile
constexpr int RR = 128;                // rows per row block (the QK MMA's M)
constexpr int DD = 128;                // head dim
constexpr int NU = 4;                  // ring units (K or V of a tile each)
constexpr int kThreads = 320;      // producer, issuer, 8 softmax warps
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kPAtom = 32768;     // P: [256 rows][64 positions] bf16, SW128 K-major
constexpr uint32_t kPBytes = 2 * kPAtom;
// tensor memory: S (128 columns), O^T (hi rows 128, lo rows 128), Q (64)
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 128;
constexpr uint32_t kColQ = 384;
constexpr uint32_t kTmemCols = 512;

struct PrSmem {
    alignas(1024) uint8_t ring[NU][kRingUnit];
    alignas(1024) uint8_t pbuf[kPBytes];
    alignas(16) float alpha[RR];   // factor of the last reference change, per row
    alignas(16) float hmax[2][RR]; // tile max of each half row (slow path)
    alignas(16) float lhalf[2][RR]; // row sums of each half at a segment's end
    int rowoff[RR];                // output row of row r; -1 past M
    uint64_t full[NU];
    uint64_t empty[NU];
    uint64_t q_full;   // the softmax warps wrote the segment's Q
    uint64_t q_free;   // the segment's last QK is done with Q
    uint64_t s_full;   // S(u) is in tensor memory
    uint64_t s_free;   // the softmax warps read S(u)
    uint64_t p_full;   // the softmax warps wrote P(u)
    uint64_t o_done;   // PV(u) (and every MMA before it) completed
    uint64_t fin;
    CtaRange range;
    uint32_t tmem_base;
    volatile int abort_flag;
    long long wait_limit;  // cycles a pipeline wait may take (the call's)
};

constexpr size_t kPrSmemBytes = sizeof(PrSmem) + 1024;  // + alignment slack
static_assert(kPrSmemBytes <= 232448, "shared memory");

// Kernel arguments: the call's parameters and the K and V pools' tensor maps
// (one 128-row box, or for tiles assembled from pages one map per box height).
template <bool kG>
struct PrArgs {
    AttnParams p;
    CUtensorMap kmap[kG ? kBoxHeights : 1];
    CUtensorMap vmap[kG ? kBoxHeights : 1];
};

// ---- MMA issuer --------------------------------------------------------------

// S(u) = Q K^T for tile u of the CTA: the K unit's 8 MMAs (K = 16 dims each),
// A (Q) read from tensor memory.  S has one buffer: it is free once the
// softmax warps read S(u - 1).
__device__ __forceinline__ bool pr_qk(PrSmem &sm, uint32_t &U, uint32_t u, uint32_t tmem,
                                      uint32_t ring0, uint32_t *flags)
{
    constexpr uint32_t idQK = f16_idesc(128, PT, 0, 0);
    if (u > 0 && !pwait(sm, &sm.s_free, (u - 1) & 1u, flags, kWaitTag))
        return false;
    const int st = (int)(U % NU);
    if (!pwait(sm, &sm.full[st], (U / NU) & 1u, flags, kWaitFull))
        return false;
    tc_fence_after();
    const uint32_t ka = ring0 + st * kRingUnit;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const uint32_t koff = (uint32_t)((s >> 2) * kRingBox + (s & 3) * 32);
        umma_f16_ts(tmem + kColS, tmem + kColQ + s * 8, sw128_desc(ka + koff, 16, 1024), idQK,
                    s > 0 ? 1u : 0u);
    }
    umma_commit(&sm.empty[st]);
    umma_commit(&sm.s_full);
    ++U;
    return true;
}

// One lane.  Per segment: QK(0), then per tile t: QK(t + 1), PV(t).
template <class A>
__device__ __forceinline__ void pr_issuer(const A &a, PrSmem &sm)
{
    const AttnParams &p = a.p;
    const uint32_t tmem = sm.tmem_base;
    // O^T += V^T P^T: A = V^T (MN-major, from the V unit), B = P (K-major,
    // [256 rows: hi then lo][positions]), N = 256
    constexpr uint32_t idPV = f16_idesc(128, 2 * RR, 1, 0);
    const uint32_t ring0 = smem_addr(sm.ring[0]);
    const uint32_t pb = smem_addr(sm.pbuf);

    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t U = 0, T0 = 0, j = 0;
    bool ok = true;
    for (; ok && cur.next(p, it); ++j) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        ok = pwait(sm, &sm.q_full, j & 1u, p.flags, kWaitQFull);
        tc_fence_after();
        ok = ok && pr_qk(sm, U, T0, tmem, ring0, p.flags);
        if (!ok)
            break;
        if (n == 1)
            umma_commit(&sm.q_free);
        for (int t = 0; t < n; ++t) {
            const uint32_t T = T0 + t;
            if (t + 1 < n) {
                ok = pr_qk(sm, U, T + 1, tmem, ring0, p.flags);
                if (!ok)
                    break;
                if (t + 2 == n)
                    umma_commit(&sm.q_free);
            }
            ok = pwait(sm, &sm.p_full, T & 1u, p.flags, kWaitQEmpty);
            tc_fence_after();
            if (!ok)
                break;
            const int st = (int)(U % NU);
            ok = pwait(sm, &sm.full[st], (U / NU) & 1u, p.flags, kWaitFull);
            tc_fence_after();
            if (!ok)
                break;
            const uint32_t va = ring0 + st * kRingUnit;
#pragma unroll
            for (int s = 0; s < 8; ++s)
                umma_f16(tmem + kColO, sw128_desc(va + s * 2048, kRingBox, 1024),
                         sw128_desc(pb + (s >> 2) * kPAtom + (s & 3) * 32, 16, 1024), idPV,
                         (t > 0 || s > 0) ? 1u : 0u);
            umma_commit(&sm.empty[st]);
            ++U;
            umma_commit(&sm.o_done);
        }
        T0 += n;
    }
    // every MMA issued by this thread has completed once `fin` flips
    umma_commit(&sm.fin);
    (void)mbar_wait(&sm.fin, 0, sm.wait_limit);
}

// ---- softmax warps -----------------------------------------------------------

// Eight warps (2..9).  Warp w reads tensor-memory lanes 32 (w % 4) .. + 31
// and owns half hh = (w - 2) / 4 of the tile: positions [64 hh, 64 hh + 64),
// which are K-atom hh of the P tile.  During a tile a thread works on its
// row's half; a row's two threads agree on the row's reference max (they
// compute it from the same shared values).  In the epilogue the thread reads
// O^T lane r (head dim r) for rows [64 hh, 64 hh + 64).
template <class A>
__device__ __forceinline__ void pr_softmax(const A &a, PrSmem &sm, int warp, int lane)
{
    const AttnParams &p = a.p;
    const int wq = warp & 3;
    const int hh = (warp - 2) >> 2;
    const int r = wq * 32 + lane;
    const uint32_t lane_base = sm.tmem_base + ((uint32_t)(wq * 32) << 16);
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float sl = p.scale_log2;
    const float2 sl2 = make_float2(sl, sl);
    // this row's lines of K-atom hh of the P tile: hi row r, lo row 128 + r
    uint8_t *const at = sm.pbuf + hh * kPAtom;
    const uint32_t phi = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
    const uint32_t plo = phi + 16 * 1024;
    const int sw = r & 7;

    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it, nx;
    uint32_t j = 0, u0 = 0;
    bool ok = true;
    for (; cur.next(p, it); ++j) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        const int m = it.b * RR + r;
        const bool live = m < p.M;
        // --- the row's query into tensor memory (each half thread its 64
        // dims); the row's output offset ---------------------------------------
        {
            const int mm = min(m, p.M - 1);
            const int wr = mm / p.G;
            const int h = it.kh * p.G + (mm - wr * p.G);
            const size_t row = ((size_t)it.s * p.W + wr) * p.Hq + h;
            if (hh == 0)
                sm.rowoff[r] = live ? (int)row : -1;
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q + row * DD + 64 * hh);
            uint32_t qr[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = live ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                qr[c * 4 + 0] = v.x;
                qr[c * 4 + 1] = v.y;
                qr[c * 4 + 2] = v.z;
                qr[c * 4 + 3] = v.w;
            }
            // (the previous segment's last QK: complete in practice, its S was read)
            ok = pwait(sm, &sm.q_free, (j & 1u) ^ 1u, p.flags, kWaitQEmpty) && ok;
            tc_fence_after();
            tmem_st32(lane_base + kColQ + 32 * hh, qr);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.q_full);
            // the next segment's query rows into L2
            SegCursor ahead = cur;
            if (ahead.next(p, nx)) {
                const int m2 = min(nx.b * RR + r, p.M - 1);
                const int wr2 = m2 / p.G;
                const int h2 = nx.kh * p.G + (m2 - wr2 * p.G);
                const __nv_bfloat16 *q2 =
                    p.q + (((size_t)nx.s * p.W + wr2) * p.Hq + h2) * DD + 64 * hh;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(q2));
            }
        }

        float2 lacc = make_float2(0.f, 0.f);
        float mref = NEG_INF;
        // positions this row sees, and the fewest any row of the block sees
        const int lim = min(row_lim(p, it.len, m), it.key1);
        const int lim_lo = min(row_lim(p, it.len, it.b * RR), it.key1);
        for (int t = 0; t < n; ++t) {
            const uint32_t u = u0 + t;
            const int tpos = it.key0 + t * PT;
            const int hpos = tpos + 64 * hh;  // first position of this half
            ok = pwait(sm, &sm.s_full, u & 1u, p.flags, kWaitFull) && ok;
            tc_fence_after();
            float s[64];
            {
                uint32_t v0[32], v1[32];
                tmem_ld32(lane_base + kColS + 64 * hh, v0);
                tmem_ld32(lane_base + kColS + 64 * hh + 32, v1);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    s[e] = __uint_as_float(v0[e]);
                    s[32 + e] = __uint_as_float(v1[e]);
                }
            }
            // S(u) is in registers: the issuer may run QK(u + 1)
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.s_free);
            // masked positions are selected to -inf (K rows there may be NaN)
            if (hpos + 64 > lim_lo) {
                const int vis = lim - hpos;
#pragma unroll
                for (int k = 0; k < 64; ++k)
                    s[k] = k < vis ? s[k] : NEG_INF;
            }
            const float hmax = max_tree(s);
            const float hm = hmax == NEG_INF ? NEG_INF : hmax * sl;
            // a half that would move the row's reference calls for the slow path
            const bool hgrow = hm != NEG_INF && (mref == NEG_INF || hm > mref + kRescaleLog2);
            if (block_any<256>(hgrow)) {
                // the row's tile max from its two halves; both threads of the
                // row take the same decision from the same values
                sm.hmax[hh][r] = hm;
                named_barrier(1, 256);
                const float tm = fmaxf(sm.hmax[0][r], sm.hmax[1][r]);
                const bool grow = tm != NEG_INF && (mref == NEG_INF || tm > mref + kRescaleLog2);
                float al = 1.f;
                if (grow) {
                    al = mref == NEG_INF ? 0.f : fast_exp2(mref - tm);
                    lacc.x *= al;
                    lacc.y *= al;
                    mref = tm;
                }
                if (hh == 0)
                    sm.alpha[r] = al;
                // rows with an earlier reference moved: rescale their O^T
                // columns (this warp: the hi columns for hh = 0, lo for hh = 1)
                if (block_any<256>(grow && al != 0.f)) {
                    ok = pwait(sm, &sm.o_done, (u - 1) & 1u, p.flags, kWaitEmpty) && ok;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t ta = lane_base + kColO + RR * hh + 32 * c;
                        uint32_t v[32];
                        tmem_ld32(ta, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            v[e] = __float_as_uint(__uint_as_float(v[e]) * sm.alpha[32 * c + e]);
                        tmem_st32(ta, v);
                    }
                    tmem_wait_st();
                }
            }
            // V rows past the stream's end are zeroed (0 * NaN = NaN): the two
            // threads of position r take one 64-dim box each
            if (tpos + PT > it.len) {
                const uint32_t uv = ring_v_unit(1, u0, t, n);
                const int st = (int)(uv % NU);
                ok = pwait(sm, &sm.full[st], (uv / NU) & 1u, p.flags, kWaitFull) && ok;
                if (r >= it.len - tpos) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(sm.ring[st] + hh * kRingBox + sw128_off(r, c)) =
                            make_uint4(0, 0, 0, 0);
                }
            }
            // --- P of this half, 32 positions at a time: the words of the first
            // 32 are computed before the wait for the P tile (PV(u - 1))
            const float negm = mref == NEG_INF ? 0.f : -mref;
            const float2 nm2 = make_float2(negm, negm);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t hw[16], lw[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int k = 32 * q + 2 * e;
                    const float2 x = __ffma2_rn(make_float2(s[k], s[k + 1]), sl2, nm2);
                    const float2 pp = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                    lacc = __fadd2_rn(lacc, pp);
                    // P = hi + lo, both bf16 by truncation: |p - hi - lo| < 2^-14 p
                    const uint32_t b0 = __float_as_uint(pp.x), b1 = __float_as_uint(pp.y);
                    hw[e] = __byte_perm(b0, b1, 0x7632);
                    const float2 tr = make_float2(__uint_as_float(b0 & 0xffff0000u),
                                                  __uint_as_float(b1 & 0xffff0000u));
                    const float2 rs = __ffma2_rn(tr, make_float2(-1.f, -1.f), pp);
                    lw[e] = __byte_perm(__float_as_uint(rs.x), __float_as_uint(rs.y), 0x7632);
                }
                // the P tile is free once PV(u - 1) completed
                if (q == 0 && u > 0)
                    ok = pwait(sm, &sm.o_done, (u - 1) & 1u, p.flags, kWaitEmpty) && ok;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t cofs = (uint32_t)(((4 * q + g) ^ sw) << 4);
                    *reinterpret_cast<uint4 *>(at + phi + cofs) =
                        make_uint4(hw[4 * g], hw[4 * g + 1], hw[4 * g + 2], hw[4 * g + 3]);
                    *reinterpret_cast<uint4 *>(at + plo + cofs) =
                        make_uint4(lw[4 * g], lw[4 * g + 1], lw[4 * g + 2], lw[4 * g + 3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            // (the test switch: every CTA withholds its first tile's arrival)
            if (lane == 0 && !(p.withhold && u == 0))
                mbar_arrive(&sm.p_full);
        }

        // --- the segment's last PV, then the rows' results -----------------------
        const uint32_t ulast = u0 + n - 1;
        ok = pwait(sm, &sm.o_done, ulast & 1u, p.flags, kWaitEmpty) && ok;
        tc_fence_after();
        sm.lhalf[hh][r] = lacc.x + lacc.y;
        named_barrier(1, 256);
        const bool write = ok && !sm.abort_flag;
        float *slot = it.fin ? nullptr : p.part + (size_t)it.slot * part_slot_floats(p);
        // O^T lane r is head dim r; this thread takes rows [64 hh, 64 hh + 64)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            const int r0 = 64 * hh + 32 * c;
            uint32_t hi[32], lo[32];
            tmem_ld32(lane_base + kColO + r0, hi);
            tmem_ld32(lane_base + kColO + RR + r0, lo);
            tmem_wait_ld();
            if (write) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int rr = r0 + e;
                    const float o = __uint_as_float(hi[e]) + __uint_as_float(lo[e]);
                    if (it.fin) {
                        const int orow = sm.rowoff[rr];
                        if (orow >= 0)
                            p.out[(size_t)orow * DD + r] = o / (sm.lhalf[0][rr] + sm.lhalf[1][rr]);
                    } else if (rr < p.SR) {
                        slot[(size_t)rr * DD + r] = o;
                    }
                }
            }
        }
        if (write && !it.fin && hh == 0 && r < p.SR) {
            slot[(size_t)p.SR * DD + r] = mref;
            slot[(size_t)p.SR * DD + p.SR + r] = sm.lhalf[0][r] + sm.lhalf[1][r];
        }
        tc_fence_before();
        // every thread is done with rowoff / lhalf before the next segment writes them
        named_barrier(1, 256);
        u0 += n;
    }
}

template <bool kG>
__global__ void __launch_bounds__(kThreads, 1) attn_prompt_kernel(const __grid_constant__ PrArgs<kG> a)
{
    extern __shared__ uint8_t smem_raw[];
    PrSmem &sm = *reinterpret_cast<PrSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    allow_dependent_launch();
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NU; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.q_full, 8);
        mbar_init(&sm.q_free, 1);
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, 8);
        mbar_init(&sm.p_full, 8);
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.fin, 1);
        sm.abort_flag = 0;
        sm.wait_limit = a.p.wait_limit;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&sm.tmem_base)), "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    wait_prior_grid();
    if (warp == 0)
        find_range(a.p, sm.range, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        if constexpr (kG) {
            ring_producer_pieces<1, NU>(a.p, a.kmap, a.vmap, sm, lane);
        } else {
            if (lane == 0)
                ring_producer<1, NU>(a.p, a.kmap, a.vmap, sm);
            __syncwarp();
        }
    } else if (warp == 1) {
        if (lane == 0)
            pr_issuer(a, sm);
        __syncwarp();
    } else {
        pr_softmax(a, sm, warp, lane);
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

// Rows per row block of this kernel.
int prompt_rows() { return RR; }

// Pool rows are addressed by 32-bit coordinates.  Any page size: tiles that
// straddle pages are gathered row by row.
bool prompt_supported(const AttnParams &p)
{
    return p.D == DD && pool_rows_fit(p);
}

template <bool kG>
cudaError_t launch_prompt(const AttnParams &p, int grid, cudaStream_t stream)
{
    PrArgs<kG> a;
    a.p = p;
    // one box of a whole 128-position tile, or boxes of 1, 2, 4, ..., 128 rows
    // for tiles assembled from page pieces
    for (int h = 0; h < (kG ? kBoxHeights : 1); ++h) {
        const int rows = kG ? 1 << h : PT;
        if (!make_pool_map(&a.kmap[h], p.k_pool, p, rows) ||
            !make_pool_map(&a.vmap[h], p.v_pool, p, rows))
            return cudaErrorInvalidValue;
    }
    static std::atomic<bool> configured[kMaxDevices];
    const cudaError_t e = set_smem_limit_once(attn_prompt_kernel<kG>, kPrSmemBytes, configured);
    if (e != cudaSuccess)
        return e;
    return launch_dependent(attn_prompt_kernel<kG>, dim3(grid), dim3(kThreads), kPrSmemBytes,
                            stream, a);
}

// Pages that are a multiple of 128 positions hold whole tiles (one TMA box);
// other page sizes assemble each tile from page pieces.
cudaError_t launch_attn_prompt(const AttnParams &p, int grid, cudaStream_t stream)
{
    return p.P % PT != 0 ? launch_prompt<true>(p, grid, stream)
                         : launch_prompt<false>(p, grid, stream);
}

}  // namespace tfp
