// attn_pm.cu -- split-context paged attention on the 5th-generation tensor
// cores with the key positions on the MMA's M dimension ("position-major"),
// for row blocks of up to 64 query rows: draft-verify windows, decode at
// head dim 128 (a GQA 4 decode block pads to 32 rows: an MMA instruction
// costs the same for any N up to 128), every head dim 256 call, and head
// dim 512 calls with more than four rows per KV head.
//
// TensorFold #1620 ("Kolibri-1's full layers take their K/V from pages of
// the core pool"), opening comment, "Reads": decode, verify and prompt rows
// attend over keys read through the page table; TensorFold #2730 ("an
// eight-row verify window"), "What this changes": a window holds up to eight
// rows.  The M = G * W rows of one (stream, KV head) share every K and V row.
// With rows on the MMA's M a 64-row verify block would be padded to 128,
// wasting half the tensor and softmax work, so this kernel computes the
// transposed products instead:
//
//   S^T[pos][r]  = sum_d K[pos][d] Q[r][d]       M = 128 positions, N = NR rows
//   O^T[d][r]   += sum_pos V[pos][d] P[r][pos]   M = 128 dims, N = 2 NR
//
// M is always full, and one softmax thread owns one key position of the
// tile: its tensor-memory lane of S^T.  P is fed to the PV MMA from shared
// memory as two bf16 parts (P = hi + lo, each the truncated upper half of a
// float, so the product keeps about 15 bits of every probability); hi and lo
// sit side by side along N and land in separate O^T columns that the
// epilogue adds.
//
// One persistent CTA per SM; 2 + NR / 8 warps (six for 32-row blocks, ten
// for 64):
//   warp 0     producer (one lane): per tile, the K units of the next tile,
//              then the V units of this one (a unit is 128 positions x 128
//              dims, two 64-dim TMA boxes with 128-byte swizzle) into a ring;
//              page ids are read two tiles ahead.
//   warp 1     MMA issuer (one lane): S^T(t+1) = K Q^T before O^T += V^T P^T(t),
//              so the softmax of one tile overlaps the MMAs of the next.
//              Owns the tensor-memory allocation.
//   warps 2-   softmax (NR / 8 warps), one key position per thread (32 rows
//              of it): write the block's query
//              rows into the Q tile at each segment's start; per tile, read the
//              position's scores for all rows, check them against each row's
//              reference max (a block-wide vote; the reference moves only
//              when some row's max grows by more than 2^8, and then O^T is
//              rescaled), write P^T, and keep per-thread row sums.  At the
//              segment's end the sums are reduced across the block and the rows
//              are normalised and stored, or left as partials for the merge.
#include "launch.cuh"
#include "ring.cuh"

namespace tfp {

namespace {

constexpr int PT = kRingTile;            // key positions per tile (the MMA's M)
constexpr uint32_t kBox = kRingBox;      // one [128 positions][64 dims] bf16 SW128 box
constexpr uint32_t kUnit = kRingUnit;    // one ring unit: 128 positions x 128 dims
constexpr float kRescaleLog2 = 8.f;      // move a row's reference max only past this growth
constexpr uint32_t kSmemCap = 232448;    // dynamic shared memory per block

template <int D, int NR>
struct PmCfg {
    static constexpr int DB = D / 128;                         // units per K (or V) tile
    static constexpr uint32_t kQBytes = (uint32_t)NR * D * 2;  // Q tile, 64-dim SW128 boxes
    static constexpr uint32_t kPBytes = (uint32_t)PT * 2 * NR * 2;  // P^T: [128 pos][2 NR] bf16
    // tensor memory: two S^T buffers of NR columns, then DB O^T blocks of 2 NR
    static constexpr uint32_t kColS = 0;
    static constexpr uint32_t kColO = 2 * NR;
    static constexpr uint32_t kCols = 2 * NR + DB * 2 * NR;
    static constexpr uint32_t kTmemCols =
        kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
    static constexpr uint32_t kSmall = 48 * NR + 512;  // per-row arrays, range, barriers
    // P^T buffers: with one, the softmax of tile t + 1 stores P only after
    // PV(t) completed, and the shared memory goes to the K/V ring instead
    static constexpr int kPBufs = 2;
    static constexpr int kFit =
        (int)((kSmemCap - 1024 - kQBytes - kPBufs * kPBytes - kSmall) / kUnit);
    static constexpr int NU = kFit > 6 ? 6 : kFit;     // ring units
    // Head dim 128 has two MMA issuers (QK and PV, see pm_qk_issuer): one
    // thread issues an MMA about every 130 cycles, and the 16 MMAs of a
    // 128-position tile come close to the tile's HBM time when the power cap
    // lowers the clock.  Its ring's slots are then split: K units in slots
    // [0, NK), V units in [NK, NU), each part with one consumer.
    static constexpr bool kDual = D == 128;
    static constexpr int NK = kDual ? 2 : NU;
    static constexpr int NV = kDual ? NU - 2 : NU;
    static_assert(kCols <= 512, "tensor memory");
    static_assert(NU >= 2 && (!kDual || NV >= 2), "ring");
    static_assert(NR == 32 || NR == 64, "row block");
    static constexpr int kSoftThreads = 4 * NR;        // 32 rows per softmax thread
    static constexpr int kPvWarp = 2 + kSoftThreads / 32;  // the PV issuer (dual issue)
    // + producer and MMA issuer warps
    static constexpr int kThreads = (kDual ? 96 : 64) + kSoftThreads;
};

template <int D, int NR>
struct PmSmem {
    using C = PmCfg<D, NR>;
    alignas(1024) uint8_t ring[C::NU][kUnit];
    alignas(1024) uint8_t q[C::kQBytes];
    alignas(1024) uint8_t pt[C::kPBufs][C::kPBytes];
    alignas(16) float mref[NR];   // row reference max, log2 units; -inf while the row saw nothing
    alignas(16) float negm[NR];   // -mref, or +inf while mref is -inf (forces a new reference)
    alignas(16) float alpha[NR];  // factor of the last reference change
    alignas(16) float lsum[NR];   // row sums (inverted for a finished row block)
    alignas(16) float red[4][NR];
    long long rowoff[2][NR];      // output offset of row r (by segment parity); -1 past M
    uint32_t rowvis[NR / 32][8];  // tree masks: bit r of [h][c] -- row 32 h + r sees window row c
    CtaRange range;               // this CTA's tiles
    uint64_t full[C::NU];
    uint64_t empty[C::NU];
    uint64_t q_full;      // the softmax warps wrote the segment's Q tile
    uint64_t q_free;      // the segment's last QK MMA is done with the Q tile
    uint64_t s_full[2];   // S^T(t) is in tensor memory
    uint64_t p_full[2];   // the softmax warps wrote P^T(t)
    uint64_t o_done[2];   // the PV reading P^T buffer b (and every MMA before it) completed
    uint64_t fin;         // every MMA of the (QK) issuer completed
    uint64_t fin_pv;      // every MMA of the PV issuer completed (dual issue)
    uint32_t tmem_base;
    volatile int abort_flag;
    long long wait_limit;  // cycles a pipeline wait may take (the call's)
};

template <int D, int NR>
constexpr size_t pm_smem_bytes()
{
    return sizeof(PmSmem<D, NR>) + 1024;  // + alignment slack
}

static_assert(pm_smem_bytes<128, 32>() <= kSmemCap, "smem");
static_assert(pm_smem_bytes<128, 64>() <= kSmemCap, "smem");
static_assert(pm_smem_bytes<256, 32>() <= kSmemCap, "smem");
static_assert(pm_smem_bytes<512, 32>() <= kSmemCap, "smem");

// Kernel arguments: the call's parameters and the K and V pools' tensor maps
// (one 128-row box, or for tiles assembled from pages one map per box height).
template <bool kG>
struct PmArgs {
    AttnParams p;
    CUtensorMap kmap[kG ? kBoxHeights : 1];
    CUtensorMap vmap[kG ? kBoxHeights : 1];
};

// Reduces v[i] (one value per row, N rows) across the warp: lane l ends up
// holding the reduction of rows [l * N / 32, (l + 1) * N / 32) in v[0 ..].
// Each step sends half of the remaining rows to the partner lane.
template <int N, bool kMax>
__device__ __forceinline__ void xpose_reduce(float (&v)[N], int lane)
{
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int o = 16 >> k;
        const int n = N >> k;
        if (n > 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
                const float send = up ? v[i] : v[i + n / 2];
                const float keep = up ? v[i + n / 2] : v[i];
                const float got = __shfl_xor_sync(0xffffffffu, send, o);
                v[i] = kMax ? fmaxf(keep, got) : keep + got;
            }
        }
    }
}

// The NR scores of this thread's position (its S^T lane), waited for.
template <int NR>
__device__ __forceinline__ void load_scores(uint32_t taddr, float (&x)[NR])
{
#pragma unroll
    for (int c = 0; c < NR / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + 32 * c, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e)
            x[32 * c + e] = __uint_as_float(r[e]);
    }
}

// ---- MMA issuer --------------------------------------------------------------

// S^T = K Q^T for one tile: DB units, 8 MMAs (K = 16 dims) each.
template <int D, int NR>
__device__ __forceinline__ bool pm_qk(PmSmem<D, NR> &sm, uint32_t &U, uint32_t d_tmem,
                                      uint32_t ring0, uint32_t q0, uint32_t *flags)
{
    using C = PmCfg<D, NR>;
    constexpr uint32_t idQK = f16_idesc(128, NR, 0, 0);
    // single issue: U counts every unit of the shared ring; dual: K units of
    // the ring's K part (slots [0, NK))
    constexpr int NRING = C::kDual ? C::NK : C::NU;
#pragma unroll 1
    for (int kb = 0; kb < C::DB; ++kb) {
        const int st = (int)(U % NRING);
        if (!pwait(sm, &sm.full[st], (U / NRING) & 1u, flags, kWaitFull))
            return false;
        tc_fence_after();
        const uint32_t ka = ring0 + st * kUnit;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t koff = (uint32_t)((s >> 2) * kBox + (s & 3) * 32);
            const uint32_t qoff = (uint32_t)((2 * kb + (s >> 2)) * (NR * 128) + (s & 3) * 32);
            umma_f16(d_tmem, sw128_desc(ka + koff, 16, 1024), sw128_desc(q0 + qoff, 16, 1024), idQK,
                     (kb > 0 || s > 0) ? 1u : 0u);
        }
        umma_commit(&sm.empty[st]);
        ++U;
    }
    return true;
}

template <int D, int NR, class A>
__device__ __forceinline__ void pm_issuer(const A &a, PmSmem<D, NR> &sm)
{
    using C = PmCfg<D, NR>;
    const AttnParams &p = a.p;
    const uint32_t tmem = sm.tmem_base;
    constexpr uint32_t idPV = f16_idesc(128, 2 * NR, 1, 1);
    const uint32_t ring0 = smem_addr(sm.ring[0]);
    const uint32_t q0 = smem_addr(sm.q);
    const uint32_t pt0 = smem_addr(sm.pt[0]);

    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t U = 0, T0 = 0, j = 0;
    bool ok = true;
    for (; ok && cur.next(p, it); ++j) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        ok = pwait(sm, &sm.q_full, j & 1u, p.flags, kWaitQFull);
        tc_fence_after();
        ok = ok && pm_qk(sm, U, tmem + C::kColS + (T0 & 1u) * NR, ring0, q0, p.flags);
        if (!ok)
            break;
        umma_commit(&sm.s_full[T0 & 1u]);
        if (n == 1)
            umma_commit(&sm.q_free);
        for (int t = 0; t < n; ++t) {
            const uint32_t T = T0 + t;
            if (t + 1 < n) {
                ok = pm_qk(sm, U, tmem + C::kColS + ((T + 1) & 1u) * NR, ring0, q0,
                                      p.flags);
                if (!ok)
                    break;
                umma_commit(&sm.s_full[(T + 1) & 1u]);
                if (t + 2 == n)
                    umma_commit(&sm.q_free);
            }
            ok = pwait(sm, &sm.p_full[T & 1u], (T >> 1) & 1u, p.flags, kWaitQEmpty);
            tc_fence_after();
            if (!ok)
                break;
            const uint32_t pb = pt0 + (T % C::kPBufs) * C::kPBytes;
#pragma unroll 1
            for (int vb = 0; vb < C::DB; ++vb) {
                const int st = (int)(U % C::NU);
                ok = pwait(sm, &sm.full[st], (U / C::NU) & 1u, p.flags, kWaitFull);
                tc_fence_after();
                if (!ok)
                    break;
                const uint32_t va = ring0 + st * kUnit;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    umma_f16(tmem + C::kColO + vb * 2 * NR, sw128_desc(va + s * 2048, kBox, 1024),
                             sw128_desc(pb + s * 2048, kBox, 1024), idPV, (t > 0 || s > 0) ? 1u : 0u);
                umma_commit(&sm.empty[st]);
                ++U;
            }
            if (!ok)
                break;
            umma_commit(&sm.o_done[T & 1u]);
        }
        T0 += n;
    }
    // every MMA issued by this thread has completed once `fin` flips
    umma_commit(&sm.fin);
    (void)mbar_wait(&sm.fin, 0, sm.wait_limit);
}

// Whether the thread's row R0 + r sees its position (see the tile loop).
template <bool kTree>
__device__ __forceinline__ bool pm_sees(int r, int rvis, uint32_t vis)
{
    if constexpr (kTree)
        return ((vis >> r) & 1u) != 0;
    else
        return r >= rvis;
}

// ---- dual issue (head dim 128) ---------------------------------------------

// One lane: per segment the DB units of K(0), then per tile unit kb of
// K(t + 1) (if any) and unit kb of V(t) in turn; K units into the ring's K
// part, V units into its V part.  Page ids are read two tiles ahead.
template <int D, int NR, class A>
__device__ __forceinline__ void pm_producer_dual(const A &a, PmSmem<D, NR> &sm)
{
    using C = PmCfg<D, NR>;
    const AttnParams &p = a.p;
    const uint64_t pol = l2_evict_first_policy();
    uint32_t UK = 0, UV = 0;
    bool ok = true;
    // unit kb (dims [128 kb, 128 kb + 128)) of page `page`, positions
    // [off, off + 128), into slot st
    auto put = [&](int st, uint32_t parity, const CUtensorMap *map, int page, int kh, int off,
                   int kb) {
        const bool page_ok = page >= 0 && page < p.n_pages;
        if (!page_ok)
            set_flag(p.flags, kDevBadPage);
        if (!pwait(sm, &sm.empty[st], parity, p.flags, kWaitEmpty))
            return false;
        if (page_ok) {
            const int y = (page * p.Hkv + kh) * p.P + off;
            mbar_arrive_expect_tx(&sm.full[st], kUnit);
            tma_load_2d(sm.ring[st], map, 128 * kb, y, &sm.full[st], pol);
            tma_load_2d(sm.ring[st] + kBox, map, 128 * kb + 64, y, &sm.full[st], pol);
        } else {
            mbar_arrive(&sm.full[st]);
        }
        return true;
    };
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    while (ok && cur.next(p, it)) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        int pg0 = __ldg(trow + it.key0 / p.P);
        int pg1 = n > 1 ? __ldg(trow + (it.key0 + PT) / p.P) : 0;
        // (UK and UV count the units actually issued)
#pragma unroll 1
        for (int kb = 0; ok && kb < C::DB; ++kb) {
            ok = put((int)(UK % C::NK), ((UK / C::NK) & 1u) ^ 1u, a.kmap, pg0, it.kh,
                     it.key0 % p.P, kb);
            UK += ok ? 1u : 0u;
        }
        for (int t = 0; ok && t < n; ++t) {
            const int pos = it.key0 + t * PT;
            const int pg2 = t + 2 < n ? __ldg(trow + (pos + 2 * PT) / p.P) : 0;
#pragma unroll 1
            for (int kb = 0; ok && kb < C::DB; ++kb) {
                if (t + 1 < n) {
                    ok = put((int)(UK % C::NK), ((UK / C::NK) & 1u) ^ 1u, a.kmap, pg1, it.kh,
                             (pos + PT) % p.P, kb);
                    UK += ok ? 1u : 0u;
                }
                if (ok) {
                    ok = put(C::NK + (int)(UV % C::NV), ((UV / C::NV) & 1u) ^ 1u, a.vmap, pg0,
                             it.kh, pos % p.P, kb);
                    UV += ok ? 1u : 0u;
                }
            }
            pg0 = pg1;
            pg1 = pg2;
        }
    }
    {
        // Let the copies in flight land before the CTA can exit.  On the
        // normal path every unit was consumed and these phases are complete;
        // after another role gave up, some may still be in flight.
        for (uint32_t k = 1; k <= (UK < (uint32_t)C::NK ? UK : (uint32_t)C::NK); ++k)
            (void)mbar_wait(&sm.full[(UK - k) % C::NK], ((UK - k) / C::NK) & 1u, sm.wait_limit);
        for (uint32_t k = 1; k <= (UV < (uint32_t)C::NV ? UV : (uint32_t)C::NV); ++k)
            (void)mbar_wait(&sm.full[C::NK + (UV - k) % C::NV], ((UV - k) / C::NV) & 1u,
                            sm.wait_limit);
    }
}

// The whole producer warp: the unit order of pm_producer_dual, each unit
// assembled from page pieces (page sizes that are not a multiple of 128;
// ring.cuh).
template <int D, int NR, class A>
__device__ __forceinline__ void pm_producer_dual_pieces(const A &a, PmSmem<D, NR> &sm, int lane)
{
    using C = PmCfg<D, NR>;
    const AttnParams &p = a.p;
    const uint64_t pol = l2_evict_first_policy();
    uint32_t UK = 0, UV = 0;  // units issued
    bool ok = true;
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    while (ok && cur.next(p, it)) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        // rows and page ids of tiles t, t + 1 and t + 2 (the page ids are read
        // two tiles before their first use)
        auto nvalid = [&](int t) { return min(PT, it.len - (it.key0 + t * PT)); };
        TilePages t0 = tile_pages(p, trow, it.key0, nvalid(0), lane);
        TilePages t1 = n > 1 ? tile_pages(p, trow, it.key0 + PT, nvalid(1), lane) : t0;
#pragma unroll 1
        for (int kb = 0; ok && kb < C::DB; ++kb) {
            ok = pieces_unit(p, sm, (int)(UK % C::NK), ((UK / C::NK) & 1u) ^ 1u, a.kmap, t0, trow,
                             it.kh, nvalid(0), kb, lane, pol);
            UK += ok ? 1u : 0u;
        }
        for (int t = 0; ok && t < n; ++t) {
            const int pos = it.key0 + t * PT;
            const TilePages t2 =
                t + 2 < n ? tile_pages(p, trow, pos + 2 * PT, nvalid(t + 2), lane) : t1;
#pragma unroll 1
            for (int kb = 0; ok && kb < C::DB; ++kb) {
                if (t + 1 < n) {
                    ok = pieces_unit(p, sm, (int)(UK % C::NK), ((UK / C::NK) & 1u) ^ 1u, a.kmap, t1,
                                     trow, it.kh, nvalid(t + 1), kb, lane, pol);
                    UK += ok ? 1u : 0u;
                }
                if (ok) {
                    ok = pieces_unit(p, sm, C::NK + (int)(UV % C::NV), ((UV / C::NV) & 1u) ^ 1u,
                                     a.vmap, t0, trow, it.kh, nvalid(t), kb, lane, pol);
                    UV += ok ? 1u : 0u;
                }
            }
            t0 = t1;
            t1 = t2;
        }
    }
    if (lane == 0) {
        // let the copies in flight land before the CTA can exit
        for (uint32_t k = 1; k <= (UK < (uint32_t)C::NK ? UK : (uint32_t)C::NK); ++k)
            (void)mbar_wait(&sm.full[(UK - k) % C::NK], ((UK - k) / C::NK) & 1u, sm.wait_limit);
        for (uint32_t k = 1; k <= (UV < (uint32_t)C::NV ? UV : (uint32_t)C::NV); ++k)
            (void)mbar_wait(&sm.full[C::NK + (UV - k) % C::NV], ((UV - k) / C::NV) & 1u,
                            sm.wait_limit);
    }
    __syncwarp();
}

// One lane: S^T(T) = K Q^T into S^T buffer T % 2 once the softmax arrived on
// p_full for tile T - 2 (it is done reading that buffer then).
template <int D, int NR, class A>
__device__ __forceinline__ void pm_qk_issuer(const A &a, PmSmem<D, NR> &sm)
{
    using C = PmCfg<D, NR>;
    const AttnParams &p = a.p;
    const uint32_t tmem = sm.tmem_base;
    const uint32_t ring0 = smem_addr(sm.ring[0]);
    const uint32_t q0 = smem_addr(sm.q);
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t U = 0, T = 0, j = 0;
    bool ok = true;
    for (; ok && cur.next(p, it); ++j) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        ok = pwait(sm, &sm.q_full, j & 1u, p.flags, kWaitQFull);
        for (int t = 0; ok && t < n; ++t, ++T) {
            if (T >= 2)
                ok = pwait(sm, &sm.p_full[T & 1u], ((T - 2) >> 1) & 1u, p.flags, kWaitQEmpty);
            tc_fence_after();
            ok = ok && pm_qk(sm, U, tmem + C::kColS + (T & 1u) * NR, ring0, q0, p.flags);
            if (!ok)
                break;
            umma_commit(&sm.s_full[T & 1u]);
            if (t + 1 == n)
                umma_commit(&sm.q_free);
        }
    }
    // every MMA issued by this thread has completed once `fin` flips
    umma_commit(&sm.fin);
    (void)mbar_wait(&sm.fin, 0, sm.wait_limit);
}

// The whole warp; lane 0 issues O^T += V^T P^T(T) once the softmax wrote
// P^T(T).  Before the PV of a stream's last tile the warp zeroes the V rows
// past the stream's end (their P is 0, but 0 * NaN = NaN); it is the V
// part's only consumer, so its wait on the slot names the right phase.
template <int D, int NR, class A>
__device__ __forceinline__ void pm_pv_issuer(const A &a, PmSmem<D, NR> &sm, int lane)
{
    using C = PmCfg<D, NR>;
    const AttnParams &p = a.p;
    const uint32_t tmem = sm.tmem_base;
    constexpr uint32_t idPV = f16_idesc(128, 2 * NR, 1, 1);
    const uint32_t pt0 = smem_addr(sm.pt[0]);
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t T = 0, UV = 0;
    bool ok = true;
    while (ok && cur.next(p, it)) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        for (int t = 0; ok && t < n; ++t, ++T) {
            if (lane == 0)
                ok = pwait(sm, &sm.p_full[T & 1u], (T >> 1) & 1u, p.flags, kWaitQEmpty);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            const int nvalid = it.len - (it.key0 + t * PT);
            const uint32_t pb = pt0 + (T % C::kPBufs) * C::kPBytes;
#pragma unroll 1
            for (int vb = 0; ok && vb < C::DB; ++vb, ++UV) {
            const int st = C::NK + (int)(UV % C::NV);
            if (lane == 0)
                ok = pwait(sm, &sm.full[st], (UV / C::NV) & 1u, p.flags, kWaitFull);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok)
                break;
            if (nvalid < PT) {
                // every lane acquires the landed unit (its phase is complete and
                // cannot move on before this warp releases the slot)
                (void)mbar_wait(&sm.full[st], (UV / C::NV) & 1u, sm.wait_limit);
                // rows nvalid .. 127 of both boxes: 16 chunks of 16 bytes a row
                for (int f = lane; f < (PT - nvalid) * 16; f += 32)
                    *reinterpret_cast<uint4 *>(sm.ring[st] + ((f >> 3) & 1) * kBox +
                                               sw128_off(nvalid + (f >> 4), f & 7)) =
                        make_uint4(0, 0, 0, 0);
                fence_async_smem();
                __syncwarp();
            }
            if (lane == 0) {
                tc_fence_after();
                const uint32_t va = smem_addr(sm.ring[st]);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    umma_f16(tmem + C::kColO + vb * 2 * NR, sw128_desc(va + s * 2048, kBox, 1024),
                             sw128_desc(pb + s * 2048, kBox, 1024), idPV, (t > 0 || s > 0) ? 1u : 0u);
                umma_commit(&sm.empty[st]);
            }
            }
            if (ok && lane == 0)
                umma_commit(&sm.o_done[T & 1u]);
        }
    }
    if (lane == 0) {
        umma_commit(&sm.fin_pv);
        (void)mbar_wait(&sm.fin_pv, 0, sm.wait_limit);
    }
    __syncwarp();
}

// ---- softmax warps -----------------------------------------------------------

// NW = 4 * NR / 32 softmax warps: warp w reads tensor-memory lanes
// 32 * (w % 4) .. + 31 (tile positions, or O^T dims), and owns the 32 rows
// [32 h, 32 h + 32) with h = (w - 2) / 4.
template <int D, int NR, bool kTree, class A>
__device__ __forceinline__ void pm_softmax(const A &a, PmSmem<D, NR> &sm, int warp, int lane)
{
    using C = PmCfg<D, NR>;
    constexpr int NT = C::kSoftThreads;
    const AttnParams &p = a.p;
    const int wq = warp & 3;             // tensor-memory lane quarter of this warp
    const int h = (warp - 2) >> 2;       // row half: rows [32 h, 32 h + 32)
    const int tid = wq * 32 + lane;      // position in the tile; O^T lane (dim within a block)
    const int st = (warp - 2) * 32 + lane;  // 0 .. NT - 1
    const uint32_t lane_base = sm.tmem_base + ((uint32_t)(wq * 32) << 16);
    const float NEG_INF = -__int_as_float(0x7f800000);
    const float POS_INF = __int_as_float(0x7f800000);
    const float sl = p.scale_log2;
    // this thread's row of a P^T buffer (SW128: 8-row groups of 1024 bytes)
    const uint32_t prow = (uint32_t)((tid >> 3) * 1024 + (tid & 7) * 128);
    const int sw = tid & 7;
    const int R0 = 32 * h;               // first row of this thread

    bool ok = true;
    // The query rows of segment jj (unit w) into the Q tile, the rows' output
    // offsets, and under tree masks the rows' window masks; then the issuer
    // may run the segment's QK.  `after` is the cursor past segment jj.
    auto load_q = [&](const WorkItem &w, uint32_t jj, const SegCursor &after) {
        constexpr int kPer = NR * D / 8 / NT;  // 16-byte chunks per thread
        static_assert(kPer % 4 == 0, "Q chunks");
        if (st < NR) {
            const int m = w.b * NR + st;
            long long off = -1;
            if (m < p.M) {
                const int wr = m / p.G;
                const int hq = w.kh * p.G + (m - wr * p.G);
                off = (((long long)w.s * p.W + wr) * p.Hq + hq) * D;
            }
            sm.rowoff[jj & 1u][st] = off;
        }
        {
            uint4 qv[kPer];
#pragma unroll
            for (int c = 0; c < kPer; ++c) {
                const int f = st + NT * c;
                const int r = f / (D / 8), k = f % (D / 8);
                const int m = w.b * NR + r;
                qv[c] = make_uint4(0, 0, 0, 0);
                if (m < p.M) {
                    const int wr = m / p.G;
                    const int hq = w.kh * p.G + (m - wr * p.G);
                    qv[c] = __ldg(reinterpret_cast<const uint4 *>(
                                      p.q + (((size_t)w.s * p.W + wr) * p.Hq + hq) * D) +
                                  k);
                }
            }
            // the Q tile is free once the previous segment's last QK completed
            ok = pwait(sm, &sm.q_free, (jj & 1u) ^ 1u, p.flags, kWaitQEmpty) && ok;
#pragma unroll
            for (int c = 0; c < kPer; ++c) {
                const int f = st + NT * c;
                const int r = f / (D / 8), k = f % (D / 8);
                *reinterpret_cast<uint4 *>(sm.q + (k >> 3) * (NR * 128) + sw128_off(r, k & 7)) =
                    qv[c];
            }
        }
        // the following segment's query rows into L2 (128-byte lines)
        SegCursor ahead = after;
        WorkItem nx2;
        if (ahead.next(p, nx2)) {
            constexpr int kLines = NR * D * 2 / 128;
            for (int f = st; f < kLines; f += NT) {
                const int r = f / (D / 64), k = f % (D / 64);
                const int m = nx2.b * NR + r;
                if (m < p.M) {
                    const int wr = m / p.G;
                    const int hq = nx2.kh * p.G + (m - wr * p.G);
                    const __nv_bfloat16 *src =
                        p.q + (((size_t)nx2.s * p.W + wr) * p.Hq + hq) * D + k * 64;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(src));
                }
            }
        }
        if (kTree && st < NR / 32 * 8) {
            // the block's rows that see window row c, from the stream's masks
            // (every thread read the previous segment's masks before its last
            // tile's vote)
            const int hh = st >> 3, c = st & 7;
            uint32_t wv = 0;
            if (c < p.W) {
                const uint8_t *tm = p.tree + (size_t)w.s * p.W;
                for (int r = 0; r < 32; ++r) {
                    const int m = w.b * NR + 32 * hh + r;
                    if (m < p.M && ((__ldg(tm + m / p.G) >> c) & 1))
                        wv |= 1u << r;
                }
            }
            sm.rowvis[hh][c] = wv;
        }
        fence_async_smem();
        named_barrier(1, NT);
        if (st == 0)
            mbar_arrive(&sm.q_full);
    };

    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t j = 0, u0 = 0;
    bool have = cur.next(p, it);
    if (have)
        load_q(it, 0, cur);
    for (; have; ++j) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        float l[32];
#pragma unroll
        for (int r = 0; r < 32; ++r)
            l[r] = 0.f;
        // the block's first row sees the fewest positions (under tree masks,
        // every row sees the positions before the window)
        const int lim_lo = kTree ? it.len - p.W : row_lim(p, it.len, it.b * NR);
        for (int t = 0; t < n; ++t) {
            const uint32_t u = u0 + t;
            const int tpos = it.key0 + t * PT;
            const uint32_t tS = lane_base + C::kColS + (u & 1u) * NR + R0;
            // a tile every row of the block sees whole needs no mask
            const bool whole = tpos + PT <= lim_lo && tpos + PT <= it.key1;
            // causal: rows R0 + r, r >= rvis, see this thread's position;
            // tree: row R0 + r sees it when bit r of vis is set
            const int pos = tpos + tid;
            const int rvis = kTree || pos >= it.key1 || pos >= it.len
                                 ? 32
                                 : p.G * max(0, pos - (it.len - p.W)) - it.b * NR - R0;
            const uint32_t vis = !kTree || pos >= it.key1 || pos >= it.len ? 0u
                                 : pos < it.len - p.W                     ? 0xffffffffu
                                                       : sm.rowvis[h][pos - (it.len - p.W)];
            ok = pwait(sm, &sm.s_full[u & 1u], (u >> 1) & 1u, p.flags, kWaitFull) && ok;
            tc_fence_after();

            float x[32];
            bool slow = t == 0;
            if (!slow) {
                load_scores<32>(tS, x);
                float mx = NEG_INF;
#pragma unroll
                for (int r = 0; r < 32; r += 4) {
                    const float4 nm = *reinterpret_cast<const float4 *>(&sm.negm[R0 + r]);
                    x[r] = fmaf(x[r], sl, nm.x);
                    x[r + 1] = fmaf(x[r + 1], sl, nm.y);
                    x[r + 2] = fmaf(x[r + 2], sl, nm.z);
                    x[r + 3] = fmaf(x[r + 3], sl, nm.w);
                }
                if (!whole) {
#pragma unroll
                    for (int r = 0; r < 32; ++r)
                        x[r] = pm_sees<kTree>(r, rvis, vis) ? x[r] : NEG_INF;
                }
                mx = max_tree(x);
                slow = block_any<NT>(mx > kRescaleLog2);
            }
            if (slow) {
                // --- a new reference max for rows whose max grew past it ---
                float y[32];
                load_scores<32>(tS, y);
#pragma unroll
                for (int r = 0; r < 32; ++r)
                    y[r] = (whole || pm_sees<kTree>(r, rvis, vis)) ? y[r] * sl : NEG_INF;
                xpose_reduce<32, true>(y, lane);
                sm.red[wq][R0 + lane] = y[0];
                named_barrier(1, NT);
                bool moved = false;
                if (st < NR) {
                    const float tmax = fmaxf(fmaxf(sm.red[0][st], sm.red[1][st]),
                                             fmaxf(sm.red[2][st], sm.red[3][st]));
                    const float m_old = t == 0 ? NEG_INF : sm.mref[st];
                    const bool grow =
                        tmax != NEG_INF && (m_old == NEG_INF || tmax > m_old + kRescaleLog2);
                    const float m_new = grow ? tmax : m_old;
                    sm.mref[st] = m_new;
                    sm.negm[st] = m_new == NEG_INF ? POS_INF : -m_new;
                    sm.alpha[st] = !grow ? 1.f : (m_old == NEG_INF ? 0.f : fast_exp2(m_old - m_new));
                    moved = t > 0 && grow && m_old != NEG_INF;
                }
                moved = block_any<NT>(moved);  // also publishes mref / negm / alpha
                if (moved) {
                    // PV(u - 1) must be done before O^T is touched; this warp
                    // rescales its rows' hi and lo columns of every dim block
                    ok = pwait(sm, &sm.o_done[(u - 1) & 1u], ((u - 1) >> 1) & 1u, p.flags,
                               kWaitEmpty) && ok;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 2 * C::DB; ++c) {
                        const uint32_t ta =
                            lane_base + C::kColO + (c >> 1) * 2 * NR + (c & 1) * NR + R0;
                        uint32_t r[32];
                        tmem_ld32(ta, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(__uint_as_float(r[e]) * sm.alpha[R0 + e]);
                        tmem_st32(ta, r);
                    }
                    tmem_wait_st();
                }
                load_scores<32>(tS, x);
#pragma unroll
                for (int r = 0; r < 32; r += 4) {
                    const float4 nm = *reinterpret_cast<const float4 *>(&sm.negm[R0 + r]);
                    const float4 al = *reinterpret_cast<const float4 *>(&sm.alpha[R0 + r]);
                    x[r] = fmaf(x[r], sl, nm.x);
                    x[r + 1] = fmaf(x[r + 1], sl, nm.y);
                    x[r + 2] = fmaf(x[r + 2], sl, nm.z);
                    x[r + 3] = fmaf(x[r + 3], sl, nm.w);
                    l[r] *= al.x;
                    l[r + 1] *= al.y;
                    l[r + 2] *= al.z;
                    l[r + 3] *= al.w;
                }
                if (!whole) {
#pragma unroll
                    for (int r = 0; r < 32; ++r)
                        x[r] = pm_sees<kTree>(r, rvis, vis) ? x[r] : NEG_INF;
                }
            }
            // --- V rows past the stream's end: zero them (0 * NaN = NaN) ----
            const int nvalid = it.len - tpos;
            if (!C::kDual && nvalid < PT) {
                // The ring slots of this tile's V units last held units of
                // V(t - 1) or earlier (at head dim 512 the ring is shorter than
                // a tile): wait for PV(u - 1) first, so each full-barrier wait
                // below names its own phase, not the one before it.
                if (u >= 1)
                    ok = pwait(sm, &sm.o_done[(u - 1) & 1u], ((u - 1) >> 1) & 1u, p.flags,
                               kWaitEmpty) && ok;
                // the V units of this tile: K(0), then per tile K(t + 1) if any, V(t)
                uint32_t uv = ring_v_unit(C::DB, u0, t, n);
#pragma unroll 1
                for (int vb = 0; vb < C::DB; ++vb, ++uv) {
                    const int sl8 = (int)(uv % C::NU);
                    ok = pwait(sm, &sm.full[sl8], (uv / C::NU) & 1u, p.flags, kWaitFull) && ok;
                    if (tid >= nvalid) {
                        // the NW / 4 threads of a position split the unit's two boxes
#pragma unroll 1
                        for (int bx = h; bx < 2; bx += NR / 32) {
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                *reinterpret_cast<uint4 *>(sm.ring[sl8] + bx * kBox + sw128_off(tid, c)) =
                                    make_uint4(0, 0, 0, 0);
                        }
                    }
                }
            }
            // --- P^T(u) -----------------------------------------------------
            uint32_t hw[16], lw[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float p0 = fast_exp2(x[2 * e]);
                const float p1 = fast_exp2(x[2 * e + 1]);
                l[2 * e] += p0;
                l[2 * e + 1] += p1;
                // P = hi + lo, both bf16 by truncation: |p - hi - lo| < 2^-14 p
                const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
                hw[e] = __byte_perm(b0, b1, 0x7632);
                const float r0 = p0 - __uint_as_float(b0 & 0xffff0000u);
                const float r1 = p1 - __uint_as_float(b1 & 0xffff0000u);
                lw[e] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
            }
            // buffer u % kPBufs is free once PV(u - kPBufs) completed
            if (u >= (uint32_t)C::kPBufs) {
                const uint32_t v = u - C::kPBufs;
                ok = pwait(sm, &sm.o_done[v & 1u], (v >> 1) & 1u, p.flags, kWaitEmpty) && ok;
            }
            uint8_t *pr = sm.pt[u % C::kPBufs] + prow;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                // hi of rows R0 + 8g .. + 7 is 16-byte chunk R0 / 8 + g of the
                // position's row; lo is chunk (NR + R0) / 8 + g
                const int ch = R0 / 8 + g, cl = (NR + R0) / 8 + g;
                *reinterpret_cast<uint4 *>(pr + (ch >> 3) * kBox + (((ch & 7) ^ sw) << 4)) =
                    make_uint4(hw[4 * g], hw[4 * g + 1], hw[4 * g + 2], hw[4 * g + 3]);
                *reinterpret_cast<uint4 *>(pr + (cl >> 3) * kBox + (((cl & 7) ^ sw) << 4)) =
                    make_uint4(lw[4 * g], lw[4 * g + 1], lw[4 * g + 2], lw[4 * g + 3]);
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            // (the test switch: every CTA withholds its first tile's arrival)
            if (lane == 0 && !(p.withhold && u == 0))
                mbar_arrive(&sm.p_full[u & 1u]);
        }

        // --- the next segment's query rows, so that the issuer runs its first QK
        // while this segment's rows are written (the Q tile is free once this
        // segment's last QK completed; the next segment's first PV, which
        // overwrites O^T, waits for its P, written after this epilogue) ----------
        WorkItem nx;
        SegCursor ahead = cur;
        const bool have_nx = ahead.next(p, nx);
        if (have_nx)
            load_q(nx, j + 1, ahead);

        // --- the segment's last PV, then the rows' results ------------------------
        const uint32_t ulast = u0 + n - 1;
        ok = pwait(sm, &sm.o_done[ulast & 1u], (ulast >> 1) & 1u, p.flags, kWaitEmpty) && ok;
        tc_fence_after();
        const bool fin = it.fin;
        xpose_reduce<32, false>(l, lane);
        sm.red[wq][R0 + lane] = l[0];
        named_barrier(1, NT);
        if (st < NR) {
            const float s = sm.red[0][st] + sm.red[1][st] + sm.red[2][st] + sm.red[3][st];
            sm.lsum[st] = fin ? 1.f / s : s;
        }
        named_barrier(1, NT);
        const bool write = ok && !sm.abort_flag;
        float *slot = fin ? nullptr
                          : p.part + (size_t)it.slot * part_slot_floats(p);
#pragma unroll 1
        for (int vb = 0; vb < C::DB; ++vb) {
            uint32_t hi[32], lo[32];
            tmem_ld32(lane_base + C::kColO + vb * 2 * NR + R0, hi);
            tmem_ld32(lane_base + C::kColO + vb * 2 * NR + NR + R0, lo);
            tmem_wait_ld();
            if (write) {
                const int d = 128 * vb + tid;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int r = R0 + e;
                    const float o = __uint_as_float(hi[e]) + __uint_as_float(lo[e]);
                    if (fin) {
                        const long long off = sm.rowoff[j & 1u][r];
                        if (off >= 0)
                            p.out[off + d] = o * sm.lsum[r];
                    } else if (r < p.SR) {
                        slot[(size_t)r * D + d] = o;
                    }
                }
            }
        }
        if (write && !fin && st < p.SR) {
            slot[(size_t)p.SR * D + st] = sm.mref[st];
            slot[(size_t)p.SR * D + p.SR + st] = sm.lsum[st];
        }
        tc_fence_before();
        u0 += n;
        cur = ahead;
        it = nx;
        have = have_nx;
    }
}

template <int D, int NR, bool kTree, bool kG>
__global__ void __launch_bounds__(PmCfg<D, NR>::kThreads, 1)
    attn_pm_kernel(const __grid_constant__ PmArgs<kG> a)
{
    using C = PmCfg<D, NR>;
    extern __shared__ uint8_t smem_raw[];
    PmSmem<D, NR> &sm = *reinterpret_cast<PmSmem<D, NR> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    allow_dependent_launch();
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NU; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_free, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_full[b], C::kSoftThreads / 32);
            mbar_init(&sm.o_done[b], 1);
        }
        mbar_init(&sm.fin, 1);
        mbar_init(&sm.fin_pv, 1);
        sm.abort_flag = 0;
        sm.wait_limit = a.p.wait_limit;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&sm.tmem_base)), "r"(C::kTmemCols)
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
            if constexpr (C::kDual)
                pm_producer_dual_pieces<D, NR>(a, sm, lane);
            else
                ring_producer_pieces<C::DB, C::NU>(a.p, a.kmap, a.vmap, sm, lane);
        } else {
            if (lane == 0) {
                if constexpr (C::kDual)
                    pm_producer_dual<D, NR>(a, sm);
                else
                    ring_producer<C::DB, C::NU>(a.p, a.kmap, a.vmap, sm);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        if (lane == 0) {
            if constexpr (C::kDual)
                pm_qk_issuer<D, NR>(a, sm);
            else
                pm_issuer<D, NR>(a, sm);
        }
        __syncwarp();
    } else if (C::kDual && warp == C::kPvWarp) {
        pm_pv_issuer<D, NR>(a, sm, lane);
    } else {
        pm_softmax<D, NR, kTree>(a, sm, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sm.tmem_base),
                     "r"(C::kTmemCols)
                     : "memory");
    }
}

template <int D, int NR, bool kTree, bool kG>
cudaError_t launch_pm(const AttnParams &p, int grid, cudaStream_t stream)
{
    PmArgs<kG> a;
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
    constexpr size_t bytes = pm_smem_bytes<D, NR>();
    const cudaError_t e = set_smem_limit_once(attn_pm_kernel<D, NR, kTree, kG>, bytes, configured);
    if (e != cudaSuccess)
        return e;
    return launch_dependent(attn_pm_kernel<D, NR, kTree, kG>, dim3(grid),
                            dim3(PmCfg<D, NR>::kThreads), bytes, stream, a);
}

}  // namespace

// Rows per row block, or 0 when this kernel does not take the call: causal
// blocks of more than 64 rows at head dim 128 go to the row-major tensor-core
// kernel (tree calls run here with several row blocks), and pool rows are
// addressed by 32-bit coordinates.  Any page size: tiles that straddle pages
// are gathered row by row.
int pm_rows(const AttnParams &p)
{
    if (!pool_rows_fit(p))
        return 0;
    if (p.D == 128)
        return p.M <= 32 ? 32 : (p.M <= 64 || p.has_tree) ? 64 : 0;
    if (p.D == 256 || p.D == 512)
        return 32;
    return 0;
}

template <bool kTree, bool kG>
cudaError_t launch_attn_pm_t(const AttnParams &p, int grid, cudaStream_t stream)
{
    if (p.D == 128 && p.RB == 32)
        return launch_pm<128, 32, kTree, kG>(p, grid, stream);
    if (p.D == 128 && p.RB == 64)
        return launch_pm<128, 64, kTree, kG>(p, grid, stream);
    if (p.D == 256 && p.RB == 32)
        return launch_pm<256, 32, kTree, kG>(p, grid, stream);
    if (p.D == 512 && p.RB == 32)
        return launch_pm<512, 32, kTree, kG>(p, grid, stream);
    return cudaErrorInvalidValue;
}

// Pages that are a multiple of 128 positions hold whole tiles (TMA boxes);
// any other page size is gathered.
cudaError_t launch_attn_pm(const AttnParams &p, int grid, cudaStream_t stream)
{
    const bool gather = p.P % PT != 0;
    if (p.has_tree)
        return gather ? launch_attn_pm_t<true, true>(p, grid, stream)
                      : launch_attn_pm_t<true, false>(p, grid, stream);
    return gather ? launch_attn_pm_t<false, true>(p, grid, stream)
                  : launch_attn_pm_t<false, false>(p, grid, stream);
}

}  // namespace tfp
